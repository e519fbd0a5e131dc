"""The no-allocation greedy entry point against the workspace one.

pspec_verify_greedy_noalloc exists for callers that cannot give the library device
memory (their HBM is reserved up front for the KV cache, or they have no allocator at
all): it runs the full-sweep greedy kernel with scratch that lives inside the library.
Here it must produce the same outputs as pspec_verify_greedy, on two calls in a row (the
second call finds the first call's leftovers in the shared scratch), report its own
launch count and path to the last-call queries, and refuse requests larger than its fixed
scratch without launching anything.

This file is collected last, so a run that stops at the first failure has already run
every other test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import speculative_decoding_step_pspec_b200 as ps
from speculative_decoding_step_pspec_b200 import _binding as b
from speculative_decoding_step_pspec_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"
RTOL = 1e-5


def _outputs(B, K):
    return dict(out_tokens=torch.full((B, K + 1), -7, dtype=torch.int32, device=DEV),
                accepted_len=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                bonus=torch.full((B,), -7, dtype=torch.int32, device=DEV),
                target_lse=torch.zeros((B, K + 1), dtype=torch.float32, device=DEV),
                err=torch.zeros((1,), dtype=torch.int32, device=DEV))


@pytest.mark.parametrize("name,B,K,V,dtype", [
    ("tiny", 4, 3, 32, torch.float32),
    ("ragged", 5, 4, 70001, torch.bfloat16),
    ("c1", 1, 7, 201088, torch.bfloat16),
    ("c64", 64, 7, 151936, torch.bfloat16),
    ("b1024", 1024, 7, 201088, torch.bfloat16),
])
def test_noalloc_matches_workspace_entry_point(name, B, K, V, dtype):
    w = I.Workload(name, B, K, V, 16, 4, dtype, seed=B + K, sigma_t=3.0, sigma_d=0.7)
    target, draft = I.logits(w, DEV)
    _, greedy = I.draft_tokens(w, draft)
    del draft
    ref = ps.verify_greedy(target, greedy, want_lse=True)
    torch.cuda.synchronize()
    for call in range(2):
        o = _outputs(B, K)
        if V % 8 == 0:             # leave an early-exit path in the last-call record first
            ps.verify_greedy(target, greedy, options={"verify_path": 2})
            assert ps.pspec_last_verify_path() == 2
        b.pspec_verify_greedy_noalloc(target_logits=target, draft_tokens=greedy, **o)
        assert ps.pspec_last_launches() == 1 and ps.pspec_last_verify_path() == 1
        torch.cuda.synchronize()
        for k in ("out_tokens", "accepted_len", "bonus"):
            assert torch.equal(o[k], ref[k]), (name, call, k)
        g, r = o["target_lse"].cpu().numpy(), ref["target_lse"].cpu().numpy()
        assert np.all(np.abs(g - r) <= RTOL * np.abs(r)), (name, call)
        assert o["err"].item() == 0


def test_noalloc_refuses_oversized_requests():
    # needs B*(K+1) partials of 16 bytes: 16384 * 32 * 16 = 8 MiB > 4 MiB of scratch.
    # Real buffers of the full size, so that nothing could read out of bounds anyway.
    B, K, V = 16384, 31, 8
    need = ps.pspec_verify_workspace_bytes(B, K, V, False)
    assert need > 4 << 20
    target = torch.zeros((B, K + 1, V), dtype=torch.bfloat16, device=DEV)
    drafts = torch.zeros((B, K), dtype=torch.int32, device=DEV)
    o = _outputs(B, K)
    with pytest.raises(b.PspecError) as ei:
        b.pspec_verify_greedy_noalloc(target_logits=target, draft_tokens=drafts, **o)
    assert ei.value.status == b.PSPEC_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (o["accepted_len"] == -7).all()          # nothing was launched
    # an empty batch launches nothing and says so
    e = _outputs(0, K)
    b.pspec_verify_greedy_noalloc(target_logits=target[:0], draft_tokens=drafts[:0], **e)
    assert ps.pspec_last_launches() == 0 and ps.pspec_last_verify_path() == 0
