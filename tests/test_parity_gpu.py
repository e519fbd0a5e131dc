"""GPU parity: libpspec's kernels (through the C ABI) against the CPU oracle.

Every workload runs at its full size in the launch configuration the benchmark uses, and
the oracle checks every sequence of every workload (the large batch's 1024 sequences on
both early-exit launches, every point of the depth sweep), besides invariants that hold at
any size.  Smaller cases cover several segments and tiles with ragged tails, padded row
strides, the edge cases (K = 1, K = 31, V < one vector, -inf rows, out-of-range tokens,
empty batches) and determinism.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_step_pspec_b200 as ps
from speculative_decoding_step_pspec_b200 import inputs as I
from tests import parity_util as U

pytestmark = pytest.mark.gpu
DEV = "cuda"


class verify_path:
    """Force the full sweep (1) or the early-exit path (2) inside a with-block."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        ps.pspec_set_verify_path(self.path)

    def __exit__(self, *a):
        ps.pspec_set_verify_path(0)


class tail_split:
    """Inside a with-block, n > 0 hands the last n sequences of an early-exit batch to a
    second launch (4-CTA clusters forced for the first)."""

    def __init__(self, n):
        self.n = n

    def __enter__(self):
        if self.n:
            ps.pspec_set_cluster_size(4)
            ps.pspec_set_tail_split(self.n)

    def __exit__(self, *a):
        ps.pspec_set_cluster_size(0)
        ps.pspec_set_tail_split(0)


def early_exit_allowed(t):
    return t.shape[2] % 8 == 0 and t.data_ptr() % 16 == 0 and (t.stride(1) * t.element_size()) % 16 == 0


def _verify_both(target, draft, sampled, greedy_drafts, u, diag=True):
    """Both verify rules, on both paths, against the oracle on every sequence: the full
    sweep with every diagnostic, then (where its shape rules allow) the early-exit path in
    its automatic launch configuration, which reads rows only up to the first rejection and
    must give the same tokens."""
    V = target.shape[2]
    with verify_path(1):
        gr = ps.verify_greedy(target, greedy_drafts, want_lse=diag)
        rj = ps.verify_rejection(target, draft, sampled, u, diagnostics=diag)
    torch.cuda.synchronize()
    U.check_verify_invariants(gr, greedy_drafts, V)
    U.check_verify_invariants(rj, sampled, V)
    og = U.oracle_greedy(target, greedy_drafts)
    U.compare_greedy(gr, og)
    orj = U.oracle_rejection(target, draft, sampled, u)
    U.compare_rejection(rj, orj)
    for path in (2,):
        if not early_exit_allowed(target):
            continue
        with verify_path(path):
            # the early-exit path may hand the batch's last sequences to a second launch
            ge = ps.verify_greedy(target, greedy_drafts)
            assert ps.pspec_last_launches() in (1, 2)
            assert ps.pspec_last_verify_path() == path
            re = ps.verify_rejection(target, draft, sampled, u, residual_mass=True)
            assert ps.pspec_last_launches() in (1, 2)
            assert ps.pspec_last_verify_path() == path
        torch.cuda.synchronize()
        assert ge["err"].item() == 0 and re["err"].item() == 0, path
        U.check_verify_invariants(ge, greedy_drafts, V)
        U.check_verify_invariants(re, sampled, V)
        U.compare_greedy(ge, og)
        U.compare_rejection(re, orj)
    return gr, rj, orj


# --------------------------------------------------------------------------- workloads
def test_tiny_workload():
    t = I.tiny_verify_numpy()
    target = torch.from_numpy(t["target"]).to(DEV)
    draft = torch.from_numpy(t["draft"]).to(DEV)
    d = torch.from_numpy(t["draft_tokens"]).to(DEV)
    u = torch.from_numpy(t["uniforms"]).to(DEV)
    _verify_both(target, draft, d, d, u)
    inp = I.build_inputs(I.TINY, DEV, ctx=t["ctx"], a_prev=t["a_prev"])
    _build_and_compare(inp)


@pytest.mark.parametrize("name", ["c1", "c64"])
def test_workload_all_sequences(name):
    w = I.WORKLOADS[name]
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    _verify_both(target, draft, sampled, greedy, u)
    if name == "c64":   # the stated drafts are sampled for both modes at c=64
        gr = ps.verify_greedy(target, sampled)
        U.compare_greedy(gr, U.oracle_greedy(target, sampled, want_lse=False))
    inp = I.build_inputs(w, DEV, drafts=sampled)
    _build_and_compare(inp)


def test_b1024_all_sequences():
    """The large batch at full size: all 1024 sequences of both rules against the oracle, on
    the full sweep and on the early exit's automatic two launches (the batch's last
    sequences in the second, wider launch)."""
    w = I.B1024
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    _, rj, _ = _verify_both(target, draft, sampled, greedy, u)
    # the step chains: this verify's accepted counts and bonus tokens feed the build
    inp = I.build_inputs(w, DEV, drafts=sampled)
    inp["accepted_len"] = rj["accepted_len"].clone()
    inp["bonus"] = rj["bonus"].clone()
    _build_and_compare(inp)


@pytest.mark.parametrize("K", I.DEPTH_K)
@pytest.mark.parametrize("sigma", I.DEPTH_SIGMA)
def test_depth_sweep_all_sequences(K, sigma):
    w = I.depth(K, sigma)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    _verify_both(target, draft, sampled, greedy, u)
    _build_and_compare(I.build_inputs(w, DEV, drafts=sampled))


# --------------------------------------------------------------------------- shapes
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("V,seg", [(1, 0), (7, 0), (8, 0), (2047, 0), (5003, 1024), (70001, 4096),
                                   (70001, 0), (5000, 1024), (70000, 0), (262144, 0)])
@pytest.mark.parametrize("K", [1, 4])
def test_ragged_multi_segment(dtype, V, seg, K):
    B = 5
    w = I.Workload("t", B, K, V, 16, 4, dtype, seed=V + K, sigma_t=2.0, sigma_d=0.6)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    ps.pspec_set_segment_elems(seg)
    try:
        _verify_both(target, draft, sampled, greedy, u)
    finally:
        ps.pspec_set_segment_elems(0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_padded_row_stride(dtype):
    B, K, V = 6, 3, 3001
    ld = 3008 if dtype == torch.bfloat16 else 3004
    w = I.Workload("t", B, K, V, 16, 4, dtype, seed=3, sigma_t=2.0, sigma_d=0.6)
    t0, q0 = I.logits(w, DEV)
    tb = torch.full((B, K + 1, ld), 99.0, dtype=dtype, device=DEV)
    qb = torch.full((B, K, ld), -99.0, dtype=dtype, device=DEV)
    tb[:, :, :V] = t0
    qb[:, :, :V] = q0
    target, draft = tb[:, :, :V], qb[:, :, :V]            # views: row stride ld > V
    sampled, greedy = I.draft_tokens(w, q0)
    u = I.uniforms(w, DEV)
    gr = ps.verify_greedy(target, greedy, want_lse=True)
    rj = ps.verify_rejection(target, draft, sampled, u, diagnostics=True)
    U.compare_greedy(gr, U.oracle_greedy(t0, greedy))
    U.compare_rejection(rj, U.oracle_rejection(t0, q0, sampled, u))


def test_max_K():
    w = I.Workload("t", 3, 31, 300, 16, 4, torch.bfloat16, seed=31, sigma_t=1.0, sigma_d=0.05)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    _verify_both(target, draft, sampled, greedy, u)
    # identical drafts pass all 31 positions
    rj = ps.verify_rejection(target, target[:, :31].contiguous(), sampled, u)
    assert (rj["accepted_len"].cpu() == 31).all()
    gr = ps.verify_greedy(target, target[:, :31].float().argmax(-1).int())
    assert (gr["accepted_len"].cpu() == 31).all()


def test_neg_inf_rows_and_entries():
    B, K, V = 6, 2, 4000
    g = torch.Generator(device=DEV).manual_seed(9)
    target = torch.randn((B, K + 1, V), generator=g, device=DEV) * 2
    draft = target[:, :K] + torch.randn((B, K, V), generator=g, device=DEV)
    target[0, 0, :] = -float("inf")                       # a row with no mass at all
    target[1, :, ::3] = -float("inf")                     # masked vocabulary entries
    draft[1, :, 1::3] = -float("inf")
    draft[2, 1, :] = -float("inf")
    target[3, 0, 17] = -float("inf")
    d = torch.randint(0, V, (B, K), generator=g, device=DEV, dtype=torch.int32)
    d[3, 0] = 17                                          # p(d) = 0: always rejected
    u = torch.rand((B, K + 1), generator=g, device=DEV)
    gr = ps.verify_greedy(target, d, want_lse=True)
    rj = ps.verify_rejection(target, draft, d, u, diagnostics=True)
    U.compare_greedy(gr, U.oracle_greedy(target, d))
    o = U.oracle_rejection(target, draft, d, u)
    U.compare_rejection(rj, o)
    assert rj["accepted_len"][3].item() == 0
    with verify_path(2):
        ge = ps.verify_greedy(target, d)
        re = ps.verify_rejection(target, draft, d, u, residual_mass=True)
    U.compare_greedy(ge, U.oracle_greedy(target, d, want_lse=False))
    U.compare_rejection(re, o)


def test_out_of_range_draft_tokens():
    w = I.Workload("t", 4, 3, 1000, 16, 4, torch.bfloat16, seed=4, sigma_t=2.0, sigma_d=0.1)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    bad = greedy.clone()
    bad[0, 0] = -1
    bad[2, 1] = w.V
    gr = ps.verify_greedy(target, bad)
    rj = ps.verify_rejection(target, draft, bad, u, diagnostics=True)
    assert gr["err"].item() == ps._binding.PSPEC_DEVERR_TOKEN_RANGE
    assert rj["err"].item() == ps._binding.PSPEC_DEVERR_TOKEN_RANGE
    U.compare_greedy(gr, U.oracle_greedy(target, bad, want_lse=False))
    o = U.oracle_rejection(target, draft, bad, u)
    U.compare_rejection(rj, o)
    assert gr["accepted_len"][0].item() == 0 and rj["accepted_len"][0].item() == 0
    for path in (2,):
        with verify_path(path):
            ge = ps.verify_greedy(target, bad)
            re = ps.verify_rejection(target, draft, bad, u)
        assert ge["err"].item() == ps._binding.PSPEC_DEVERR_TOKEN_RANGE
        assert re["err"].item() == ps._binding.PSPEC_DEVERR_TOKEN_RANGE
        U.compare_greedy(ge, U.oracle_greedy(target, bad, want_lse=False))
        U.compare_rejection(re, o)


@pytest.mark.parametrize("B", [1, 4, 63, 64, 159, 160, 200])
def test_automatic_path_selection(B):
    """Automatic selection with no per-row diagnostic requested: the early exit from 160
    sequences on for the rejection rule and from 64 on for the greedy rule (two launches
    from 128 sequences on), the full sweep below (two launches for the rejection rule, one
    for the greedy rule); a diagnostic always takes the full sweep; same tokens whichever
    path runs."""
    w = I.Workload("t", B, 5, 4096, 16, 4, torch.bfloat16, seed=B, sigma_t=2.0, sigma_d=0.6)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    a = ps.verify_rejection(target, draft, sampled, u)
    path_auto = ps.pspec_last_verify_path()
    b = ps.verify_rejection(target, draft, sampled, u, diagnostics=True)
    assert ps.pspec_last_launches() == 2 and ps.pspec_last_verify_path() == 1
    assert path_auto == (2 if B >= 160 else 1)
    g = ps.verify_greedy(target, greedy)
    if B >= 64:
        # from 128 sequences on the last sequences go to a second launch (tail split)
        assert ps.pspec_last_verify_path() == 2 and ps.pspec_last_launches() == (2 if B >= 128 else 1)
    else:
        assert ps.pspec_last_verify_path() == 1 and ps.pspec_last_launches() == 1
    gl = ps.verify_greedy(target, greedy, want_lse=True)
    assert ps.pspec_last_verify_path() == 1
    o = U.oracle_rejection(target, draft, sampled, u)
    U.compare_rejection(a, o)
    U.compare_rejection(b, o)
    og = U.oracle_greedy(target, greedy)
    U.compare_greedy(g, og)
    U.compare_greedy(gl, og)


def test_early_exit_refuses_what_it_cannot_take():
    w = I.Workload("t", 4, 3, 1001, 16, 4, torch.bfloat16, seed=5, sigma_t=2.0, sigma_d=0.6)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    with verify_path(2):
        with pytest.raises(ps.PspecError):
            ps.verify_rejection(target, draft, sampled, u)          # V not a multiple of 8
    w = I.Workload("t", 4, 3, 1000, 16, 4, torch.bfloat16, seed=5, sigma_t=2.0, sigma_d=0.6)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    with verify_path(2):
        with pytest.raises(ps.PspecError):
            ps.verify_rejection(target, draft, sampled, I.uniforms(w, DEV), diagnostics=True)


def test_determinism_and_workspace_reuse():
    w = I.scaled(I.C64, B=16, V=50000)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    ws = ps.Workspace(w.B, w.K, w.V, True)
    outs = [ps.verify_rejection(target, draft, sampled, u, diagnostics=True, workspace=ws)
            for _ in range(3)]
    for o in outs[1:]:
        for k in o:
            assert torch.equal(o[k], outs[0][k]), k
    # the counters left at zero serve a smaller batch next
    r = ps.verify_rejection(target[:5], draft[:5], sampled[:5], u[:5], workspace=ws)
    for k in ("out_tokens", "accepted_len", "bonus"):
        assert torch.equal(r[k], outs[0][k][:5]), k
    with verify_path(2):
        e1 = ps.verify_rejection(target, draft, sampled, u, residual_mass=True, workspace=ws)
        e2 = ps.verify_rejection(target, draft, sampled, u, residual_mass=True, workspace=ws)
    for k in e1:
        assert torch.equal(e1[k], e2[k]), k
    # the paths take turns on one workspace: sweep, early exit, sweep on a smaller batch
    with verify_path(1):
        s1 = ps.verify_rejection(target, draft, sampled, u, diagnostics=True, workspace=ws)
    with verify_path(2):
        e3 = ps.verify_rejection(target, draft, sampled, u, residual_mass=True, workspace=ws)
    with verify_path(1):
        s2 = ps.verify_rejection(target[:5], draft[:5], sampled[:5], u[:5], workspace=ws)
    for k in ("out_tokens", "accepted_len", "bonus"):
        assert torch.equal(s1[k], e1[k]), k
        assert torch.equal(e3[k], e1[k]), k
        assert torch.equal(s2[k], e1[k][:5]), k
    # residual mass is summed in a different order on each path: fp32 within 1e-5
    assert torch.allclose(s1["residual_mass"], e1["residual_mass"], rtol=1e-5, atol=0)
    wsg = ps.Workspace(w.B, w.K, w.V, False)
    g1 = ps.verify_greedy(target, greedy, want_lse=True, workspace=wsg)
    g2 = ps.verify_greedy(target, greedy, want_lse=True, workspace=wsg)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k
    with verify_path(2):
        h1 = ps.verify_greedy(target, greedy, workspace=wsg)
        h2 = ps.verify_greedy(target, greedy, workspace=wsg)
    g3 = ps.verify_greedy(target, greedy, want_lse=True, workspace=wsg)
    for k in ("out_tokens", "accepted_len", "bonus"):
        assert torch.equal(h1[k], g1[k]) and torch.equal(h2[k], g1[k]) and torch.equal(g3[k], g1[k]), k


def test_empty_batch():
    t = torch.empty((0, 4, 100), dtype=torch.bfloat16, device=DEV)
    q = torch.empty((0, 3, 100), dtype=torch.bfloat16, device=DEV)
    d = torch.empty((0, 3), dtype=torch.int32, device=DEV)
    u = torch.empty((0, 4), dtype=torch.float32, device=DEV)
    ps.verify_greedy(t, d)
    ps.verify_rejection(t, q, d, u)
    torch.cuda.synchronize()


# --------------------------------------------------------------------------- exactness
@pytest.mark.parametrize("K", [1, 2, 3])
def test_threshold_probing_exact_rule(K):
    """The kernel's accept decisions flip exactly at tau = min(1, p/q) and its draws follow
    the residual's CDF: u = tau - 2e-6 accepts, tau + 2e-6 rejects, and u at the middle of
    each CDF interval returns that interval's token (V = 8, all 8^K draft tuples of K = 1,
    2, 3, with target and draft rows that depend on the drafted prefix): together with the
    accept probabilities min(1, p/q) and the residual law this fixes, the emitted tokens
    follow the target's autoregressive law exactly."""
    from tests.oracle_pins import _prefix_logits
    import itertools
    import scipy.special as sps
    V = 8
    tuples = list(itertools.product(range(V), repeat=K))
    t = np.stack([np.stack([_prefix_logits(tp[:k], V, 1) for k in range(K + 1)]) for tp in tuples])
    q = np.stack([np.stack([_prefix_logits(tp[:k], V, 2) for k in range(K)]) for tp in tuples])
    d = np.array(tuples, np.int32)
    P = sps.softmax(t.astype(np.float64), axis=2)
    Q = sps.softmax(q.astype(np.float64), axis=2)
    rows_t, rows_q, rows_d, rows_u, expect_a, expect_tok = [], [], [], [], [], []
    for n in range(len(tuples)):
        for k in range(K):
            tau = min(1.0, P[n, k, d[n, k]] / Q[n, k, d[n, k]])
            for du, acc in ((-2e-6, True), (2e-6, False)):
                uu = tau + du
                if not (0.0 <= uu < 1.0):
                    continue
                u = np.zeros(K + 1, np.float32)
                u[k] = uu
                rows_t.append(t[n]); rows_q.append(q[n]); rows_d.append(d[n]); rows_u.append(u)
                expect_a.append((k, acc)); expect_tok.append(-1)
            # draws after a rejection at k
            if tau < 1.0 - 1e-5:
                r = np.maximum(P[n, k] - Q[n, k], 0.0)
                F = np.concatenate([[0.0], np.cumsum(r) / r.sum()])
                for tok in range(V):
                    if F[tok + 1] - F[tok] < 1e-5:
                        continue
                    u = np.zeros(K + 1, np.float32)
                    u[k] = np.nextafter(np.float32(1), np.float32(0))
                    u[K] = (F[tok] + F[tok + 1]) / 2
                    rows_t.append(t[n]); rows_q.append(q[n]); rows_d.append(d[n]); rows_u.append(u)
                    expect_a.append((k, False)); expect_tok.append(tok)
        # the bonus draw after K acceptances follows p_K
        F = np.concatenate([[0.0], np.cumsum(P[n, K])])
        for tok in range(V):
            if F[tok + 1] - F[tok] < 1e-5:
                continue
            u = np.zeros(K + 1, np.float32)
            u[K] = (F[tok] + F[tok + 1]) / 2
            rows_t.append(t[n]); rows_q.append(q[n]); rows_d.append(d[n]); rows_u.append(u)
            expect_a.append((K, None)); expect_tok.append(tok)
    T = torch.from_numpy(np.stack(rows_t)).to(DEV)
    Qd = torch.from_numpy(np.stack(rows_q)).to(DEV)
    D = torch.from_numpy(np.stack(rows_d)).to(DEV)
    Uu = torch.from_numpy(np.stack(rows_u)).to(DEV)
    o = oracle.verify_rejection(np.stack(rows_t), np.stack(rows_q), np.stack(rows_d), np.stack(rows_u))
    print(f"[probing] K={K}: {len(tuples)} tuples, {len(expect_a)} probes")
    for path in (1, 2):
        with verify_path(path):
            r = ps.verify_rejection(T, Qd, D, Uu)
        a = r["accepted_len"].cpu().numpy()
        bonus = r["bonus"].cpu().numpy()
        for n, ((k, acc), tok) in enumerate(zip(expect_a, expect_tok)):
            if acc is True:
                assert a[n] > k, (path, n)
            elif acc is False:
                assert a[n] == k, (path, n)
            else:
                assert a[n] == K, (path, n)
            if tok >= 0:
                assert bonus[n] == tok, (path, n, bonus[n], tok)
                assert o["bonus"][n] == tok
        assert np.array_equal(a, o["accepted_len"]), path


# --------------------------------------------------------------------------- build
def _build_and_compare(inp, check_hidden=True):
    dh = U.hidden_sentinel(inp["T_cap"], inp["H"], inp["verify_hidden"].dtype, DEV)
    init = dh.view(torch.int16).cpu().numpy() if dh.dtype == torch.bfloat16 else dh.cpu().numpy()
    out = ps.api.build_outputs(inp["B"], inp["K"], inp["H"], inp["T_cap"], dh.dtype, DEV)
    out["draft_hidden"] = dh
    g = ps.build_draft_batch(
        K=inp["K"], block_size=inp["block_size"], mask_id=inp["mask_id"], pad_id=inp["pad_id"],
        T_cap=inp["T_cap"], qsl_in=inp["qsl_in"], verify_tokens=inp["verify_tokens"],
        verify_pos=inp["verify_pos"], accepted_len=inp["accepted_len"], bonus=inp["bonus"],
        block_table=inp["block_table"], verify_hidden=inp["verify_hidden"],
        h_shared=inp["h_shared"], out=out, k_len=inp.get("k_len"))
    torch.cuda.synchronize()
    o = U.oracle_build(inp, init)
    U.compare_build(g, o, check_hidden)
    return g, o


def _torchify(case, dtype=torch.bfloat16):
    def i32(x):
        return torch.as_tensor(np.asarray(x, np.int32), device=DEV)
    B = len(case["qsl_in"]) - 1
    extra = {} if case.get("k_len") is None else {"k_len": i32(case["k_len"])}
    return dict(**extra, B=B, K=case["K"], H=case["verify_hidden"].shape[1], block_size=case["block_size"],
                mask_id=case["mask_id"], pad_id=case["pad_id"], T_cap=case["T_cap"],
                qsl_in=i32(case["qsl_in"]), verify_tokens=i32(case["verify_tokens"]),
                verify_pos=i32(case["verify_pos"]), accepted_len=i32(case["accepted_len"]),
                bonus=i32(case["bonus"]), block_table=i32(case["block_table"]),
                verify_hidden=torch.from_numpy(case["verify_hidden"]).to(DEV).to(dtype),
                h_shared=torch.from_numpy(case["h_shared"]).to(DEV).to(dtype))


@pytest.mark.parametrize("K,L_extra,bs,H", [(1, 0, 4, 8), (3, 0, 4, 16), (7, 0, 16, 64),
                                            (4, 5, 8, 24), (31, 2, 16, 8), (7, 40, 16, 2880)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_build_random_layouts(K, L_extra, bs, H, dtype):
    from tests.oracle_pins import random_build_case
    rng = np.random.default_rng(K * 100 + L_extra)
    case = random_build_case(rng, B=37, K=K, H=H, bs=bs, L_extra=L_extra)
    _build_and_compare(_torchify(case, dtype))


def test_build_worked_example_on_gpu():
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "build_worked_example.json")))
    case = dict(g, verify_hidden=np.arange(8 * 8, dtype=np.float32).reshape(8, 8),
                h_shared=np.full(8, -1.0, np.float32))
    out, _ = _build_and_compare(_torchify(case, torch.float32))
    for k, v in g["expect"].items():
        assert out[k].cpu().numpy().tolist() == v, k


def test_build_invalid_values():
    from tests.oracle_pins import random_build_case
    rng = np.random.default_rng(22)
    case = random_build_case(rng, B=6, K=3, H=8, bs=4)
    _build_and_compare(_torchify(dict(case, accepted_len=np.array([-2, 0, 1, 9, 3, 2]))))
    t = case["block_table"].copy()
    t[2, :] = -1
    _build_and_compare(_torchify(dict(case, block_table=t)))
    p = case["verify_pos"].copy()
    p[5] = -4
    p[9] = 10 ** 6
    _build_and_compare(_torchify(dict(case, verify_pos=p)))
    q = np.array(case["qsl_in"]).copy()
    q[2] = q[1] + 2                  # a sequence with fewer than K+1 rows
    _build_and_compare(_torchify(dict(case, qsl_in=q)))
    q = np.array(case["qsl_in"]).copy()
    q[3] = q[2] - 1                  # not an offset array: only the error bit is defined
    inp = _torchify(dict(case, qsl_in=q))
    out = ps.build_draft_batch(K=3, block_size=4, mask_id=inp["mask_id"], pad_id=inp["pad_id"],
                               T_cap=inp["T_cap"], qsl_in=inp["qsl_in"],
                               verify_tokens=inp["verify_tokens"], verify_pos=inp["verify_pos"],
                               accepted_len=inp["accepted_len"], bonus=inp["bonus"],
                               block_table=inp["block_table"], verify_hidden=inp["verify_hidden"],
                               h_shared=inp["h_shared"])
    assert out["err"].item() & ps._binding.PSPEC_DEVERR_LAYOUT


def test_build_empty_batch_pads():
    inp = dict(B=0, K=3, H=8, block_size=4, mask_id=5, pad_id=6, T_cap=10,
               qsl_in=torch.zeros(1, dtype=torch.int32, device=DEV),
               verify_tokens=torch.zeros(0, dtype=torch.int32, device=DEV),
               verify_pos=torch.zeros(0, dtype=torch.int32, device=DEV),
               accepted_len=torch.zeros(0, dtype=torch.int32, device=DEV),
               bonus=torch.zeros(0, dtype=torch.int32, device=DEV),
               block_table=torch.zeros((1, 1), dtype=torch.int32, device=DEV),
               verify_hidden=torch.zeros((0, 8), dtype=torch.float32, device=DEV),
               h_shared=torch.zeros(8, dtype=torch.float32, device=DEV))
    _build_and_compare(inp)


# --------------------------------------------------------------------------- draft sampling
def _sample_both(logits, u, seqs=None):
    """Inverse-CDF sampling and argmax of drafter rows [B, K, V] against the oracle."""
    B, K, V = logits.shape
    s = ps.sample_drafts(logits, u, want_probs=True)
    g = ps.sample_drafts(logits, None, want_probs=True)
    torch.cuda.synchronize()
    assert s["err"].item() == 0 and g["err"].item() == 0
    idx = slice(None) if seqs is None else torch.as_tensor(seqs, device=logits.device)
    host = U.host_logits(logits[idx])
    os_ = oracle.sample_rows(host, u[idx].cpu().numpy(), threads=U.THREADS)
    og = oracle.sample_rows(host, None, threads=U.THREADS)
    sel = slice(None) if seqs is None else np.asarray(seqs)
    st = s["draft_tokens"].cpu().numpy()[sel]
    gt = g["draft_tokens"].cpu().numpy()[sel]
    assert np.array_equal(gt, og["tokens"]), np.argwhere(gt != og["tokens"])[:5]
    clean = os_["flags"] == 0
    bad = np.argwhere((st != os_["tokens"]) & clean)
    assert bad.size == 0, (bad[:5], st[tuple(bad[:5].T)], os_["tokens"][tuple(bad[:5].T)])
    for out, o in ((s, os_), (g, og)):
        pr = out["q_at_draft"].cpu().numpy()[sel]
        same = out["draft_tokens"].cpu().numpy()[sel] == o["tokens"]
        ok = U._rel_ok(pr, o["probs"]) | ~same
        assert ok.all(), (pr[~ok][:5], o["probs"][~ok][:5])
    x = logits.float()
    tok = s["draft_tokens"].long()
    live = torch.isfinite(x).any(-1)                  # rows with some mass never pick -inf
    assert torch.isfinite(torch.gather(x, 2, tok[..., None]))[..., 0][live].all()
    print(f"[sampling] {clean.size} rows, {int((~clean).sum())} flagged near-ties")


@pytest.mark.parametrize("name", ["tiny", "c1", "c64"])
def test_sampling_workloads(name):
    if name == "tiny":
        t = I.tiny_verify_numpy()
        logits = torch.from_numpy(t["draft"]).to(DEV)
        u = torch.from_numpy(t["uniforms"][:, :logits.shape[1]].copy()).to(DEV)
    else:
        w = I.WORKLOADS[name]
        _, logits = I.logits(w, DEV)
        u = I.uniforms(w, DEV)[:, :w.K].contiguous()
    _sample_both(logits, u)


def test_sampling_b1024_all_rows():
    """All 7168 drafter rows of the large batch against the oracle."""
    w = I.B1024
    _, logits = I.logits(w, DEV)
    u = I.uniforms(w, DEV)[:, :w.K].contiguous()
    _sample_both(logits, u)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("V", [1, 7, 8, 255, 257, 2047, 5003, 70001, 262144])
def test_sampling_ragged(dtype, V):
    w = I.Workload("t", 3, 4, V, 16, 4, dtype, seed=V, sigma_t=2.0, sigma_d=0.6)
    _, logits = I.logits(w, DEV)
    _sample_both(logits, I.uniforms(w, DEV)[:, :4].contiguous())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sampling_padded_stride_and_neg_inf(dtype):
    B, K, V, ld = 4, 3, 3001, 3016
    g = torch.Generator(device=DEV).manual_seed(3)
    buf = torch.full((B, K, ld), 77.0, dtype=dtype, device=DEV)
    buf[:, :, :V] = (torch.randn((B, K, V), generator=g, device=DEV) * 2).to(dtype)
    buf[0, 0, :V:2] = -float("inf")
    buf[1, 2, :] = -float("inf")                     # a row with no mass: token 0, p 0
    logits = buf[:, :, :V]
    u = torch.rand((B, K), generator=g, device=DEV)
    _sample_both(logits, u)


def test_sampling_threshold_probing():
    """The token at the middle of every CDF interval is that interval's token."""
    import scipy.special as sps
    rng = np.random.default_rng(8)
    rows = rng.normal(0, 1.5, size=(5, 8)).astype(np.float32)
    P = sps.softmax(rows.astype(np.float64), axis=1)
    F = np.concatenate([np.zeros((5, 1)), np.cumsum(P, axis=1)], axis=1)
    lg, uu, want = [], [], []
    for n in range(5):
        for t in range(8):
            if F[n, t + 1] - F[n, t] < 1e-5:
                continue
            lg.append(rows[n]); uu.append((F[n, t] + F[n, t + 1]) / 2); want.append(t)
    L = torch.from_numpy(np.stack(lg)[:, None, :]).to(DEV)
    U_ = torch.tensor(np.array(uu, np.float32)[:, None], device=DEV)
    got = ps.sample_drafts(L, U_)["draft_tokens"][:, 0].cpu().numpy()
    assert np.array_equal(got, np.array(want))


def test_sampling_empty_and_errors():
    L = torch.empty((0, 3, 100), dtype=torch.bfloat16, device=DEV)
    ps.sample_drafts(L, None)
    with pytest.raises(ps.PspecError):
        ws = torch.zeros(256, dtype=torch.uint8, device=DEV)       # too small
        ps.sample_drafts(torch.zeros((2, 3, 100), device=DEV), None, workspace=ws)


def test_sampling_workspace_serves_smaller_batches():
    """One workspace sized for the largest batch: large, small, large again give the same
    tokens as fresh workspaces (the tickets sit at addresses independent of B)."""
    w = I.Workload("t", 24, 5, 30011, 16, 4, torch.bfloat16, seed=21, sigma_t=2.0, sigma_d=0.6)
    _, logits = I.logits(w, DEV)
    u = I.uniforms(w, DEV)[:, :w.K].contiguous()
    ws = torch.zeros(ps._binding.pspec_sample_workspace_bytes(w.B, w.K, w.V), dtype=torch.uint8,
                     device=DEV)
    ref = ps.sample_drafts(logits, u, want_probs=True)
    a = ps.sample_drafts(logits, u, want_probs=True, workspace=ws)
    b = ps.sample_drafts(logits[:7], u[:7], want_probs=True, workspace=ws)
    c = ps.sample_drafts(logits, u, want_probs=True, workspace=ws)
    for k in ("draft_tokens", "q_at_draft"):
        assert torch.equal(a[k], ref[k]) and torch.equal(c[k], ref[k]), k
        assert torch.equal(b[k], ref[k][:7]), k


# --------------------------------------------------------------------------- whole step
def _step_check(target, draft, drafts, u, binp, path, expect_fused):
    """ps.step (verify + build, one launch when the early-exit path takes it) equals the
    verify call followed by the build call, bit for bit, on every output including the
    hidden rows it must leave untouched."""
    rej = u is not None
    H, dt = binp["verify_hidden"].shape[1], binp["verify_hidden"].dtype

    def bout():
        o = ps.api.build_outputs(binp["B"], binp["K"], H, binp["T_cap"], dt, DEV)
        o["draft_hidden"] = U.hidden_sentinel(binp["T_cap"], H, dt, DEV)
        return o
    with verify_path(path):
        if rej:
            v1 = ps.verify_rejection(target, draft, drafts, u, residual_mass=True)
        else:
            v1 = ps.verify_greedy(target, drafts)
        n_verify = ps.pspec_last_launches()
        b1 = ps.build_draft_batch(
            K=binp["K"], block_size=binp["block_size"], mask_id=binp["mask_id"],
            pad_id=binp["pad_id"], T_cap=binp["T_cap"], qsl_in=binp["qsl_in"],
            verify_tokens=binp["verify_tokens"], verify_pos=binp["verify_pos"],
            accepted_len=v1["accepted_len"], bonus=v1["bonus"], block_table=binp["block_table"],
            verify_hidden=binp["verify_hidden"], h_shared=binp["h_shared"], out=bout())
        v2, b2 = ps.step(target, drafts, binp, draft_logits=draft if rej else None, uniforms=u,
                         residual_mass=rej, build_out=bout())
        n_step = ps.pspec_last_launches()
    torch.cuda.synchronize()
    for k in v1:
        assert torch.equal(v1[k], v2[k]), k
    for k in b1:
        assert torch.equal(b1[k], b2[k]), k
    # fused: the verify's own launches (one, or two when the batch is split) also build
    assert n_step == (n_verify if expect_fused else n_verify + 1), (n_step, n_verify)
    return v2, b2


@pytest.mark.parametrize("rule", ["greedy", "rejection"])
@pytest.mark.parametrize("path", [0, 2])
def test_step_c64_fused(rule, path):
    # automatic at 64 sequences: the greedy rule takes the early exit, the rejection rule the
    # full sweep; either way the build runs inside the verify's last launch
    w = I.C64
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    binp = I.build_inputs(w, DEV, drafts=sampled)
    rej = rule == "rejection"
    # below 256 sequences the build runs inside the verify's last launch on either path
    _step_check(target, draft, sampled if rej else greedy, u if rej else None, binp, path, True)


@pytest.mark.parametrize("path", [0, 1, 2])
@pytest.mark.parametrize("rule", ["greedy", "rejection"])
def test_step_tiny_every_path(rule, path):
    # automatic at 5 sequences: both rules take the full sweep; on every path the build runs
    # inside the verify's last launch (fewer than 256 sequences)
    fused = True
    w = I.scaled(I.C64, B=5, V=4096, H=64)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    binp = I.build_inputs(w, DEV, drafts=sampled)
    rej = rule == "rejection"
    _step_check(target, draft, sampled if rej else greedy, u if rej else None, binp, path, fused)


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("K,L_extra", [(1, 0), (3, 2), (7, 5)])
def test_step_random_layouts_fused(K, L_extra, path):
    """Spans with more verify rows than K+1 (the drafts are each span's last K rows), the
    build fused into the full sweep's deciding CTAs (path 1) or the early exit's clusters."""
    from tests.oracle_pins import random_build_case
    rng = np.random.default_rng(500 + K)
    case = random_build_case(rng, B=37, K=K, H=32, bs=4, L_extra=L_extra)
    binp = _torchify(case)
    g = torch.Generator(device=DEV).manual_seed(K)
    V = 3000
    target = (torch.randn((37, K + 1, V), generator=g, device=DEV) * 2).to(torch.bfloat16)
    draft = (target[:, :K].float() + torch.randn((37, K, V), generator=g, device=DEV) * 0.5).to(torch.bfloat16)
    d = torch.argmax(draft.float(), dim=2).to(torch.int32)
    u = torch.rand((37, K + 1), generator=g, device=DEV)
    _step_check(target, draft, d, u, binp, path, True)
    _step_check(target, draft, d, None, binp, path, True)


@pytest.mark.parametrize("path", [1, 2])
def test_step_fused_invalid_layout_sets_bit(path):
    from tests.oracle_pins import random_build_case
    rng = np.random.default_rng(31)
    case = random_build_case(rng, B=6, K=3, H=8, bs=4)
    q = case["qsl_in"].copy()
    q[3] = q[2] - 1                      # not an offset array: only the error bit is defined
    binp = _torchify(dict(case, qsl_in=q))
    target = torch.randn((6, 4, 512), device=DEV).to(torch.bfloat16)
    d = torch.argmax(target[:, :3].float(), dim=2).to(torch.int32)
    with verify_path(path):
        _, bo = ps.step(target, d, binp)
        assert ps.pspec_last_launches() == 1
    torch.cuda.synchronize()
    assert bo["err"].item() & ps._binding.PSPEC_DEVERR_LAYOUT


def test_step_b1024_fused():
    """Full size with fusion forced on (the automatic choice at 1024 sequences is two
    launches), then forced off; every sequence against the oracle."""
    w = I.B1024
    target, draft = I.logits(w, DEV)
    sampled, _ = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    binp = I.build_inputs(w, DEV, drafts=sampled)
    try:
        ps.pspec_set_step_fusion(1)
        v, _ = _step_check(target, draft, sampled, u, binp, 0, True)
        ps.pspec_set_step_fusion(2)
        _step_check(target, draft, sampled, u, binp, 2, False)
    finally:
        ps.pspec_set_step_fusion(0)
    U.compare_rejection(v, U.oracle_rejection(target, draft, sampled, u))


@pytest.mark.parametrize("path,tail", [(0, 0), (2, 20), (1, 0)])
def test_step_cuda_graph_replay(path, tail):
    """One step captured in a CUDA graph and replayed with new uniforms and drafts copied
    into the captured buffers gives what the eager calls give for those inputs (the
    kernels leave their workspace counters at zero, so replays need no reset); `tail`
    splits the early-exit launch in two (4-CTA clusters, then 8-CTA clusters queued with
    programmatic dependent launch)."""
    w = I.scaled(I.C64, B=96, V=20000, H=64)
    target, draft = I.logits(w, DEV)
    sampled, _ = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    binp = I.build_inputs(w, DEV, drafts=sampled)
    ws = ps.Workspace(w.B, w.K, w.V, True)
    vout = ps.api.verify_outputs(w.B, w.K, DEV, False, True, True)
    bout = ps.api.build_outputs(w.B, w.K, 64, binp["T_cap"], binp["verify_hidden"].dtype, DEV)
    d_in, u_in = sampled.clone(), u.clone()
    with verify_path(path), tail_split(tail):
        ps.step(target, d_in, binp, draft_logits=draft, uniforms=u_in, residual_mass=True,
                workspace=ws, out=vout, build_out=bout)           # warm-up outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g):
                ps.step(target, d_in, binp, draft_logits=draft, uniforms=u_in, residual_mass=True,
                        workspace=ws, out=vout, build_out=bout)
        torch.cuda.current_stream().wait_stream(side)
        gen = torch.Generator(device=DEV).manual_seed(7)
        for rep in range(3):
            u_new = torch.rand(u.shape, generator=gen, device=DEV).clamp_(max=I.LAST_BELOW_ONE)
            d_new = torch.where(torch.rand(sampled.shape, generator=gen, device=DEV) < 0.2,
                                torch.randint_like(sampled, 0, w.V), sampled)
            u_in.copy_(u_new)
            d_in.copy_(d_new)
            g.replay()
            ref_v, ref_b = ps.step(target, d_new, binp, draft_logits=draft, uniforms=u_new,
                                   residual_mass=True)
            torch.cuda.synchronize()
            for k in ("out_tokens", "accepted_len", "bonus", "residual_mass"):
                assert torch.equal(vout[k], ref_v[k]), (rep, k)
            for k in ("draft_tokens", "draft_pos", "slot_mapping", "row_kind", "hidden_src",
                      "qsl_out", "seq_lens_out", "sample_idx"):
                assert torch.equal(bout[k], ref_b[k]), (rep, k)
    del g


# --------------------------------------------------------------------------- per-sequence K_i
def _k_len_case(B, K, V, seed, with_bad=False):
    w = I.Workload("t", B, K, V, 64, 16, torch.bfloat16, seed=seed, sigma_t=2.0, sigma_d=0.5)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    g = np.random.default_rng(seed)
    kl = g.integers(0, K + 1, size=B).astype(np.int32)
    kl[:4] = [0, K, 1, 0]
    if with_bad:
        kl[4], kl[5] = -3, K + 2                 # clamped to 0 and K, error bit set
    klt = torch.as_tensor(kl, device=DEV)
    kc = np.clip(kl, 0, K)
    for t in (sampled, greedy):                  # unused draft slots hold -1
        m = torch.as_tensor(np.arange(K)[None, :] >= kc[:, None], device=DEV)
        t.masked_fill_(m, -1)
    return w, target, draft, sampled, greedy, u, klt


@pytest.mark.parametrize("path", [1, 2])
def test_k_len_verify_every_path(path):
    """Per-sequence draft counts on every path against the oracle (reading R14): counts
    0..K, -1 in the unused draft slots (no range error), out-of-range counts clamped with
    PSPEC_DEVERR_KLEN_RANGE."""
    w, target, draft, sampled, greedy, u, klt = _k_len_case(96, 7, 20000, 61, with_bad=True)
    with verify_path(path):
        g = ps.verify_greedy(target, greedy, k_len=klt)
        r = ps.verify_rejection(target, draft, sampled, u, k_len=klt, residual_mass=True)
    torch.cuda.synchronize()
    assert g["err"].item() == ps._binding.PSPEC_DEVERR_KLEN_RANGE
    assert r["err"].item() == ps._binding.PSPEC_DEVERR_KLEN_RANGE
    og = U.oracle_greedy(target, greedy, want_lse=False, k_len=klt)
    orj = U.oracle_rejection(target, draft, sampled, u, k_len=klt)
    assert og["err"] == 0x20 and orj["err"] == 0x20
    g["err"].zero_()
    r["err"].zero_()
    U.compare_greedy(g, og)
    U.compare_rejection(r, orj)
    kc = klt.clamp(0, 7)
    assert (g["accepted_len"] <= kc).all() and (r["accepted_len"] <= kc).all()


def test_k_len_all_k_equals_fixed_k():
    """k_len = K for every sequence gives the fixed-K outputs bit for bit."""
    w = I.scaled(I.C64, B=70, V=30000)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    kl = torch.full((w.B,), w.K, dtype=torch.int32, device=DEV)
    for path in (1, 2):
        with verify_path(path):
            a = ps.verify_rejection(target, draft, sampled, u, residual_mass=True)
            b = ps.verify_rejection(target, draft, sampled, u, residual_mass=True, k_len=kl)
            c = ps.verify_greedy(target, greedy)
            d = ps.verify_greedy(target, greedy, k_len=kl)
        for k in a:
            assert torch.equal(a[k], b[k]), (path, k)
        for k in c:
            assert torch.equal(c[k], d[k]), (path, k)


def test_k_len_b1024_all_sequences():
    w = I.B1024
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    kl = torch.as_tensor(np.random.default_rng(3).integers(0, w.K + 1, size=w.B).astype(np.int32),
                         device=DEV)
    r = ps.verify_rejection(target, draft, sampled, u, k_len=kl)
    g = ps.verify_greedy(target, greedy, k_len=kl)
    U.compare_rejection(r, U.oracle_rejection(target, draft, sampled, u, k_len=kl))
    U.compare_greedy(g, U.oracle_greedy(target, greedy, want_lse=False, k_len=kl))


@pytest.mark.parametrize("K,L_extra", [(1, 0), (3, 2), (7, 0), (7, 4)])
def test_k_len_build(K, L_extra):
    """The draft batch with per-sequence K_i (spans as short as K_i + 1 rows) against the
    oracle, and the whole step (fused and not) equal to verify + build."""
    from tests.oracle_pins import random_build_case
    rng = np.random.default_rng(700 + K)
    kl = rng.integers(0, K + 1, size=37)
    case = random_build_case(rng, B=37, K=K, H=32, bs=4, L_extra=L_extra, k_len=kl)
    binp = _torchify(case)
    _build_and_compare(binp)
    g = torch.Generator(device=DEV).manual_seed(K)
    V = 3000
    target = (torch.randn((37, K + 1, V), generator=g, device=DEV) * 2).to(torch.bfloat16)
    draft = (target[:, :K].float() + torch.randn((37, K, V), generator=g, device=DEV) * 0.5).to(torch.bfloat16)
    d = torch.argmax(draft.float(), dim=2).to(torch.int32)
    u = torch.rand((37, K + 1), generator=g, device=DEV)
    klt = binp["k_len"]
    # 37 sequences: the build runs inside the verify's last launch on either path (automatic
    # fusion), and after it when fusion is switched off
    try:
        for fusion, fused in ((0, True), (2, False)):
            ps.pspec_set_step_fusion(fusion)
            for path in (2, 1):
                for uu in (u, None):
                    v1, b1 = _step_check_k(target, draft, d, uu, binp, path, fused, klt)
                    assert b1["err"].item() == 0
    finally:
        ps.pspec_set_step_fusion(0)


def _step_check_k(target, draft, drafts, u, binp, path, expect_fused, klt):
    rej = u is not None
    H, dt = binp["verify_hidden"].shape[1], binp["verify_hidden"].dtype

    def bout():
        o = ps.api.build_outputs(binp["B"], binp["K"], H, binp["T_cap"], dt, DEV)
        o["draft_hidden"] = U.hidden_sentinel(binp["T_cap"], H, dt, DEV)
        return o
    with verify_path(path):
        if rej:
            v1 = ps.verify_rejection(target, draft, drafts, u, residual_mass=True, k_len=klt)
        else:
            v1 = ps.verify_greedy(target, drafts, k_len=klt)
        n_verify = ps.pspec_last_launches()
        b1 = ps.build_draft_batch(
            K=binp["K"], block_size=binp["block_size"], mask_id=binp["mask_id"],
            pad_id=binp["pad_id"], T_cap=binp["T_cap"], qsl_in=binp["qsl_in"],
            verify_tokens=binp["verify_tokens"], verify_pos=binp["verify_pos"],
            accepted_len=v1["accepted_len"], bonus=v1["bonus"], block_table=binp["block_table"],
            verify_hidden=binp["verify_hidden"], h_shared=binp["h_shared"], out=bout(), k_len=klt)
        v2, b2 = ps.step(target, drafts, binp, draft_logits=draft if rej else None, uniforms=u,
                         residual_mass=rej, build_out=bout(), k_len=klt)
        n_step = ps.pspec_last_launches()
    torch.cuda.synchronize()
    for k in v1:
        assert torch.equal(v1[k], v2[k]), k
    for k in b1:
        assert torch.equal(b1[k], b2[k]), k
    assert n_step == (n_verify if expect_fused else n_verify + 1)
    # the build against the oracle with the verify's own counts and tokens
    inp = dict(binp, accepted_len=v1["accepted_len"], bonus=v1["bonus"])
    dh = U.hidden_sentinel(binp["T_cap"], H, dt, DEV)
    init = dh.view(torch.int16).cpu().numpy() if dt == torch.bfloat16 else dh.cpu().numpy()
    U.compare_build(b2, U.oracle_build(inp, init))
    return v2, b2


@pytest.mark.parametrize("X", [1, 37, 150])
def test_early_exit_tail_split(X):
    """The batch split over two early-exit launches (the large-batch clusters, then the last
    X sequences in wider clusters queued with programmatic dependent launch) against the
    oracle, both rules, K_i included, and the step fused and unfused."""
    w = I.Workload("t", 300, 7, 40000, 64, 16, torch.bfloat16, seed=X, sigma_t=2.0, sigma_d=0.5)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    kl = torch.as_tensor(np.random.default_rng(X).integers(0, w.K + 1, size=w.B).astype(np.int32),
                         device=DEV)
    binp = I.build_inputs(w, DEV, drafts=sampled)
    try:
        ps.pspec_set_tail_split(X)
        with verify_path(2):
            g = ps.verify_greedy(target, greedy)
            assert ps.pspec_last_launches() == 2
            r = ps.verify_rejection(target, draft, sampled, u, residual_mass=True)
            assert ps.pspec_last_launches() == 2
            rk = ps.verify_rejection(target, draft, sampled, u, k_len=kl)
        torch.cuda.synchronize()
        assert g["err"].item() == 0 and r["err"].item() == 0 and rk["err"].item() == 0
        U.compare_greedy(g, U.oracle_greedy(target, greedy, want_lse=False))
        U.compare_rejection(r, U.oracle_rejection(target, draft, sampled, u))
        U.compare_rejection(rk, U.oracle_rejection(target, draft, sampled, u, k_len=kl))
        for fuse in (1, 2):
            ps.pspec_set_step_fusion(fuse)
            _step_check(target, draft, sampled, u, binp, 2, fuse == 1)
            _step_check(target, draft, greedy, None, binp, 2, fuse == 1)
    finally:
        ps.pspec_set_tail_split(0)
        ps.pspec_set_step_fusion(0)


@pytest.mark.parametrize("G", [2, 4, 8, 12, 16])
def test_early_exit_every_cluster_size(G):
    """The early-exit kernel with each cluster size (the automatic choice is fixed from 128
    sequences on, wider below) against the oracle, unfused and with the step fused, K_i
    included."""
    w = I.scaled(I.C64, B=40, V=40000, H=64)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    kl = torch.as_tensor(np.random.default_rng(G).integers(0, w.K + 1, size=w.B).astype(np.int32),
                         device=DEV)
    binp = I.build_inputs(w, DEV, drafts=sampled)
    try:
        ps.pspec_set_cluster_size(G)
        with verify_path(2):
            g = ps.verify_greedy(target, greedy)
            r = ps.verify_rejection(target, draft, sampled, u, residual_mass=True)
            rk = ps.verify_rejection(target, draft, sampled, u, k_len=kl)
        U.compare_greedy(g, U.oracle_greedy(target, greedy, want_lse=False))
        U.compare_rejection(r, U.oracle_rejection(target, draft, sampled, u))
        U.compare_rejection(rk, U.oracle_rejection(target, draft, sampled, u, k_len=kl))
        _step_check(target, draft, sampled, u, binp, 2, True)
        _step_check(target, draft, greedy, None, binp, 2, True)
    finally:
        ps.pspec_set_cluster_size(0)


# --------------------------------------------------------------------------- per-call options
def test_per_call_options_threads_and_streams():
    """Three host threads, each on a stream of its own, verify the same batch at the same time
    with different per-call options -- one forces the full sweep with short segments, one
    the early exit with 4-CTA clusters and a split batch, one the early exit with 8-CTA
    clusters in one launch -- while the process-wide
    defaults ask for something else again (early exit, 16-CTA clusters).  Each call runs
    with its own options (the per-thread last-call queries report its path, cluster width
    and launch count), and every output equals the oracle's; a call without options follows
    the defaults."""
    import threading
    w = I.scaled(I.C64, B=96, V=40000)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    u = I.uniforms(w, DEV)
    orj = U.oracle_rejection(target, draft, sampled, u)
    og = U.oracle_greedy(target, greedy, want_lse=False)
    opts = {"sweep": {"verify_path": 1, "segment_elems": 4096},
            "early": {"verify_path": 2, "cluster_size": 4, "tail_split": 16},
            "early8": {"verify_path": 2, "cluster_size": 8, "step_fusion": 2}}
    # (path, rejection launches, greedy path)
    want = {"sweep": (1, 2, 1), "early": (2, 2, 2), "early8": (2, 1, 2)}
    results, errors = {}, []
    start = threading.Barrier(len(opts))

    def worker(name):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                o = opts[name]
                wsr = ps.Workspace(w.B, w.K, w.V, True, DEV, o)
                wsg = ps.Workspace(w.B, w.K, w.V, False, DEV, o)
                start.wait()
                seen, outs = [], []
                for _ in range(10):
                    r = ps.verify_rejection(target, draft, sampled, u, residual_mass=True,
                                            workspace=wsr, options=o)
                    seen.append((ps.pspec_last_verify_path(), ps.pspec_last_launches(),
                                 ps.pspec_last_cluster_size()))
                    g = ps.verify_greedy(target, greedy, workspace=wsg, options=o)
                    seen.append((ps.pspec_last_verify_path(),))
                    outs.append((r, g))
                s.synchronize()
            results[name] = (seen, outs)
        except Exception as e:  # noqa: BLE001
            errors.append((name, repr(e)))

    ps.pspec_set_verify_path(2)
    ps.pspec_set_cluster_size(16)
    try:
        th = [threading.Thread(target=worker, args=(n,)) for n in opts]
        for t in th:
            t.start()
        for t in th:
            t.join()
        assert not errors, errors
        d = ps.verify_rejection(target, draft, sampled, u)
        assert ps.pspec_last_verify_path() == 2 and ps.pspec_last_cluster_size() == 16
    finally:
        ps.pspec_set_verify_path(0)
        ps.pspec_set_cluster_size(0)
    torch.cuda.synchronize()
    U.compare_rejection(d, orj)
    for name, (seen, outs) in results.items():
        path, launches, gpath = want[name]
        for j in range(0, len(seen), 2):
            assert seen[j][0] == path and seen[j][1] == launches, (name, seen[j])
            if name != "sweep":
                assert seen[j][2] == opts[name]["cluster_size"], (name, seen[j])
            assert seen[j + 1][0] == gpath, (name, seen[j + 1])
        for r, g in outs:
            assert r["err"].item() == 0 and g["err"].item() == 0
            U.compare_rejection(r, orj)
            U.compare_greedy(g, og)



# --------------------------------------------------------------------------- early exit, more shapes
def _ee_case(B, K, V, seed, sigma_d=0.6, dtype=torch.bfloat16, H=64):
    w = I.Workload("t", B, K, V, H, 16, dtype, seed=seed, sigma_t=3.0, sigma_d=sigma_d)
    target, draft = I.logits(w, DEV)
    sampled, greedy = I.draft_tokens(w, draft)
    return w, target, draft, sampled, greedy, I.uniforms(w, DEV)


@pytest.mark.parametrize("G", [4, 16])
@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 131072), (torch.float32, 40000),
                                     (torch.bfloat16, 200008)])
def test_early_exit_dtypes_and_ragged_slices(G, dtype, V):
    """The early exit with both dtypes and a last slice shorter than the others, against the
    oracle; K_i included; the step fused and not."""
    w, target, draft, sampled, greedy, u = _ee_case(40, 7, V, seed=V + G, dtype=dtype)
    kl = torch.as_tensor(np.random.default_rng(G).integers(0, w.K + 1, size=w.B).astype(np.int32),
                         device=DEV)
    opts = {"verify_path": 2, "cluster_size": G}
    g = ps.verify_greedy(target, greedy, options=opts)
    assert ps.pspec_last_verify_path() == 2 and ps.pspec_last_cluster_size() == G
    r = ps.verify_rejection(target, draft, sampled, u, residual_mass=True, options=opts)
    rk = ps.verify_rejection(target, draft, sampled, u, k_len=kl, options=opts)
    gk = ps.verify_greedy(target, greedy, k_len=kl, options=opts)
    torch.cuda.synchronize()
    for o in (g, r, rk, gk):
        assert o["err"].item() == 0
    U.compare_greedy(g, U.oracle_greedy(target, greedy, want_lse=False))
    U.compare_rejection(r, U.oracle_rejection(target, draft, sampled, u))
    U.compare_rejection(rk, U.oracle_rejection(target, draft, sampled, u, k_len=kl))
    U.compare_greedy(gk, U.oracle_greedy(target, greedy, want_lse=False, k_len=kl))
    binp = I.build_inputs(w, DEV, drafts=sampled)
    try:
        ps.pspec_set_cluster_size(G)
        _step_check(target, draft, sampled, u, binp, 2, True)
        _step_check(target, draft, greedy, None, binp, 2, True)
        ps.pspec_set_step_fusion(2)
        _step_check(target, draft, sampled, u, binp, 2, False)
    finally:
        ps.pspec_set_cluster_size(0)
        ps.pspec_set_step_fusion(0)


def test_early_exit_edge_decisions():
    """Sequences that accept every draft (draft rows equal to the target's), that reject at
    position 0 (a draft token with p = 0), with no drafts at all (K_i = 0) or one, and with
    out-of-range draft tokens, on the early exit against the oracle."""
    w, target, draft, sampled, greedy, u = _ee_case(12, 5, 131072, seed=77)
    draft[0] = target[0, :5]                              # identical rows: all accepted
    target[1, 0, 17] = -float("inf")
    sampled[1, 0] = 17                                    # p(d) = 0: rejected at once
    sampled[2, 3] = -5                                    # out of range
    greedy[2, 1] = w.V + 3
    kl = torch.full((w.B,), w.K, dtype=torch.int32, device=DEV)
    kl[3] = 0
    kl[4] = 1
    for k_len in (None, kl):
        r = ps.verify_rejection(target, draft, sampled, u, residual_mass=True, k_len=k_len,
                                options={"verify_path": 2})
        g = ps.verify_greedy(target, greedy, k_len=k_len, options={"verify_path": 2})
        torch.cuda.synchronize()
        assert r["err"].item() == ps._binding.PSPEC_DEVERR_TOKEN_RANGE
        assert g["err"].item() == ps._binding.PSPEC_DEVERR_TOKEN_RANGE
        r["err"].zero_()
        g["err"].zero_()
        U.compare_rejection(r, U.oracle_rejection(target, draft, sampled, u, k_len=k_len))
        U.compare_greedy(g, U.oracle_greedy(target, greedy, want_lse=False, k_len=k_len))
        if k_len is None:
            assert r["accepted_len"][0].item() == w.K and r["accepted_len"][1].item() == 0
