// Status strings and the build identity of the C ABI.
#include "../../include/dflash.h"

#ifndef DFLASH_SOURCE_HASH
#define DFLASH_SOURCE_HASH "unhashed"
#endif

extern "C" const char* dflash_build_id(void) { return DFLASH_SOURCE_HASH; }

extern "C" const char* dflash_status_string(int status) {
  switch (status) {
    case DFLASH_OK: return "ok";
    case DFLASH_ERR_INVALID_ARG: return "invalid argument";
    case DFLASH_ERR_UNSUPPORTED: return "unsupported configuration";
    case DFLASH_ERR_CUDA: return "CUDA error";
    case DFLASH_ERR_WORKSPACE: return "workspace too small";
    case DFLASH_ERR_TIMEOUT: return "device wait timed out";
    case DFLASH_ERR_BAD_INDEX: return "token index out of range";
    default: return "unknown status";
  }
}
