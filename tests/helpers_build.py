"""Build libdflash.so from the tests without importing the package first (the
package loads the library on import)."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def build_module():
    path = os.path.join(ROOT, "block_draft_selection_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_dflash_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def build_library():
    return build_module().build_library()
