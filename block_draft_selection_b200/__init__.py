"""Block-draft hot path on B200 (sm_100a): two-tap conv, fused LM-head top-16,
pair-score path selection, greedy verification.

The compute lives in libdflash.so (C ABI in include/dflash.h); this package is
the thin ctypes binding over it.  Importing it fails loudly when the library
has not been built: there is no CPU fallback.
"""
import numpy as np
import torch

from ._binding import (  # noqa: F401
    DFLASH_ERR_BAD_INDEX,
    DFLASH_ERR_TIMEOUT,
    DFlashError,
    K_TOP,
    LIB_PATH,
    dflash_conv2tap,
    dflash_conv2tap_dynamic,
    dflash_conv2tap_dynamic_workspace,
    dflash_ctx_gate,
    dflash_ctx_table,
    dflash_ctx_walk,
    dflash_gemm_bf16,
    dflash_lmhead_logits_debug,
    dflash_lmhead_topk,
    dflash_lmhead_topk_workspace,
    dflash_path_select,
    dflash_path_walk,
    dflash_select_verify,
    dflash_lmhead_topk_static,
    dflash_lmhead_topk_merge,
    dflash_lmhead_topk_partial,
    dflash_lmhead_topk_records,
    dflash_status_string,
    dflash_build_id,
    dflash_verify,
    dflash_verify_rejection,
    dflash_verify_rejection_workspace,
    lib,
    workspace,
)
from .cycle import DraftCycle, DraftPipeline  # noqa: F401,E402
from .parallel import VocabParallelLMHead, vocab_shard  # noqa: F401,E402


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """Wrap bf16 bit patterns (np.uint16) as a torch.bfloat16 tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t
