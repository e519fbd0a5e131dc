"""speculative_decoding_step_pspec_b200 -- the per-step hot path of speculative decoding
with P-EAGLE parallel drafting on one B200 (sm_100a).

libpspec.so (hand-written CUDA, C ABI in ``include/pspec.h``) does all the work; this
package is its thin ctypes binding (``_binding``, the C names), allocation helpers
(``api``) and the seeded synthetic input generators (``inputs``).  Importing it fails if
the library has not been built: there is no CPU fallback.
"""
from ._binding import (  # noqa: F401
    EXPORTED, LIB, PspecError, library_path, pspec_build_draft_batch,
    pspec_last_launches, pspec_set_segment_elems, pspec_set_split_event,
    pspec_set_verify_path, pspec_last_verify_path, pspec_set_cluster_size,
    pspec_status_string,
    pspec_verify_greedy, pspec_verify_rejection, pspec_verify_workspace_bytes,
)
from ._binding import pspec_sample_drafts, pspec_sample_workspace_bytes  # noqa: F401
from ._binding import pspec_set_step_fusion, pspec_step_greedy, pspec_step_rejection  # noqa: F401
from ._binding import pspec_last_cluster_size, pspec_set_ee_stream, pspec_set_tail_split  # noqa: F401
from ._binding import pspec_set_wait_limit  # noqa: F401
from .api import (  # noqa: F401
    Workspace, build_draft_batch, sample_drafts, step, verify_greedy, verify_rejection,
)
