"""speculative_decoding_step_pspec_b200 -- the per-step hot path of speculative decoding
with P-EAGLE parallel drafting on one B200 (sm_100a).

libpspec.so (hand-written CUDA, C ABI in ``include/pspec.h``) does all the work; this
package is its thin ctypes binding (``_binding``, the C names), allocation helpers
(``api``) and the seeded synthetic input generators (``inputs``).

The binding is loaded on first use of any of its names (``ps.verify_greedy``,
``ps.pspec_set_verify_path``, ``ps._binding`` ...), so that importing only the input
generators (``from speculative_decoding_step_pspec_b200 import inputs``) does not map the
library.  That first use raises ImportError when libpspec.so has not been built: there is
no CPU fallback.
"""
from __future__ import annotations

import importlib

_API_NAMES = ("Workspace", "build_draft_batch", "sample_drafts", "step", "verify_greedy",
              "verify_rejection")


def __getattr__(name):
    if name in ("_binding", "api"):
        return importlib.import_module(f".{name}", __name__)
    if name in _API_NAMES:
        return getattr(importlib.import_module(".api", __name__), name)
    if name in ("EXPORTED", "LIB", "PspecError", "library_path") or name.startswith("pspec_"):
        b = importlib.import_module("._binding", __name__)
        if hasattr(b, name):
            return getattr(b, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def load():
    """Map libpspec.so now (raises ImportError when it has not been built)."""
    return importlib.import_module("._binding", __name__).LIB
