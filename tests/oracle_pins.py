"""Pins of the CPU oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` function takes an ``oracle.OracleLib`` and raises AssertionError when the
oracle disagrees with an independent source: hand-derived worked examples (tests/golden),
library routines (numpy argmax, scipy softmax / logsumexp, torch's bf16 conversion),
closed forms (sum max(0, p-q) = 1 - sum min(p, q)), special cases, and a brute-force
enumeration showing that the emitted tokens follow the target's autoregressive law
exactly.  The same pins run against deliberately broken copies of the oracle
(test_oracle_mutations.py) to show that each plausible mistake is caught.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np
import scipy.special as sps
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Raw bf16 bit patterns (round-to-nearest-even, torch's conversion)."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()


# ----------------------------------------------------------------------------- verify
def pin_worked_examples(o):
    """Hand-derived examples (tests/golden/verify_worked_examples.json)."""
    g = _load("verify_worked_examples.json")
    for c in g["cases"]:
        K = c["K"]
        t = np.log(np.array(c["p"], np.float64)).astype(np.float32)[None]
        q = np.log(np.array(c["q"], np.float64)).astype(np.float32)[None]
        d = np.array([c["drafts"]], np.int32)
        u = np.array([c["u"]], np.float32)
        r = o.verify_rejection(t, q, d, u)
        e = c["rejection"]
        assert r["out_tokens"][0].tolist() == e["out_tokens"], (c["name"], r["out_tokens"])
        assert int(r["accepted_len"][0]) == e["accepted_len"], c["name"]
        assert int(r["bonus"][0]) == e["bonus"], c["name"]
        np.testing.assert_allclose(r["residual_mass"][0], e["residual_mass"], rtol=1e-6)
        np.testing.assert_allclose(r["p_at_draft"][0], e["p_at_draft"], rtol=1e-6)
        np.testing.assert_allclose(r["q_at_draft"][0], e["q_at_draft"], rtol=1e-6)
        assert r["flags"][0] == 0
        gr = o.verify_greedy(t, d)
        e = c["greedy"]
        assert gr["out_tokens"][0].tolist() == e["out_tokens"], (c["name"], gr["out_tokens"])
        assert int(gr["accepted_len"][0]) == e["accepted_len"]
        assert int(gr["bonus"][0]) == e["bonus"]
        assert K == t.shape[1] - 1


def pin_greedy_matches_numpy_argmax(o):
    """Greedy choices equal numpy.argmax (first occurrence), ties included; the accepted
    prefix stops exactly at a planted mismatch."""
    rng = np.random.default_rng(11)
    B, K, V = 40, 5, 37
    t = rng.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    # plant ties: copy each row's max to a later and to an earlier position in half the rows
    for i in range(0, B, 2):
        for k in range(K + 1):
            j = int(np.argmax(t[i, k]))
            t[i, k, (j + 7) % V] = t[i, k, j]
            t[i, k, max(0, j - 3)] = t[i, k, j]
    g = np.argmax(t, axis=2).astype(np.int32)            # first occurrence
    d = g[:, :K].copy()
    r = o.verify_greedy(t, d, want_lse=True)
    assert (r["accepted_len"] == K).all()
    assert (r["out_tokens"] == g).all()
    assert (r["bonus"] == g[:, K]).all()
    np.testing.assert_allclose(r["target_lse"], sps.logsumexp(t.astype(np.float64), axis=2),
                               rtol=1e-13, atol=1e-13)
    m = rng.integers(0, K, size=B)
    for i in range(B):
        d[i, m[i]] = (g[i, m[i]] + 1) % V
    r = o.verify_greedy(t, d)
    assert (r["accepted_len"] == m).all()
    for i in range(B):
        a = m[i]
        assert r["out_tokens"][i, :a].tolist() == g[i, :a].tolist()
        assert r["out_tokens"][i, a] == g[i, a] == r["bonus"][i]
        assert (r["out_tokens"][i, a + 1:] == -1).all()


def pin_bf16_decoding(o):
    """bf16 logits arrive as raw bits; the oracle must decode them as torch does."""
    rng = np.random.default_rng(12)
    B, K, V = 6, 3, 300
    x = rng.normal(0, 3, size=(B, K + 1, V)).astype(np.float32)
    bits = bf16_bits(x)
    vals = bf16_values(bits)
    g = np.argmax(vals, axis=2).astype(np.int32)
    r = o.verify_greedy(bits, g[:, :K].copy(), want_lse=True)
    assert (r["out_tokens"] == g).all()
    np.testing.assert_allclose(r["target_lse"], sps.logsumexp(vals.astype(np.float64), axis=2),
                               rtol=1e-13, atol=1e-13)
    qbits = bf16_bits(x[:, :K] + rng.normal(0, 0.5, size=(B, K, V)).astype(np.float32))
    u = rng.random((B, K + 1), dtype=np.float32)
    r32 = o.verify_rejection(vals, bf16_values(qbits), g[:, :K].copy(), u)
    r16 = o.verify_rejection(bits, qbits, g[:, :K].copy(), u)
    for k in ("out_tokens", "accepted_len", "bonus", "p_at_draft", "q_at_draft", "residual_mass"):
        assert np.array_equal(r32[k], r16[k]), k


def pin_probabilities_match_scipy(o):
    """p(d_k), q(d_k) and both log-sum-exps against scipy.special (float64)."""
    rng = np.random.default_rng(13)
    B, K, V = 20, 4, 50
    t = rng.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    q = (t[:, :K] + rng.normal(0, 1, size=(B, K, V))).astype(np.float32)
    d = rng.integers(0, V, size=(B, K)).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    r = o.verify_rejection(t, q, d, u)
    pt = sps.softmax(t.astype(np.float64), axis=2)
    pq = sps.softmax(q.astype(np.float64), axis=2)
    ii, kk = np.meshgrid(np.arange(B), np.arange(K), indexing="ij")
    np.testing.assert_allclose(r["p_at_draft"], pt[ii, kk, d], rtol=1e-12)
    np.testing.assert_allclose(r["q_at_draft"], pq[ii, kk, d], rtol=1e-12)
    np.testing.assert_allclose(r["target_lse"], sps.logsumexp(t.astype(np.float64), axis=2), rtol=1e-13)
    np.testing.assert_allclose(r["draft_lse"], sps.logsumexp(q.astype(np.float64), axis=2), rtol=1e-13)
    # accepted drafts are the drafts; tokens after the emitted one are -1
    for i in range(B):
        a = r["accepted_len"][i]
        assert 0 <= a <= K
        assert r["out_tokens"][i, :a].tolist() == d[i, :a].tolist()
        assert r["out_tokens"][i, a] == r["bonus"][i]
        assert (r["out_tokens"][i, a + 1:] == -1).all()
        # the accept rule: every accepted position had u < p/q, the rejected one did not
        for k in range(a):
            assert u[i, k] < pt[i, k, d[i, k]] / pq[i, k, d[i, k]]
        if a < K:
            assert not (u[i, a] < pt[i, a, d[i, a]] / pq[i, a, d[i, a]])


def pin_residual_mass_closed_form(o):
    """sum_t max(0, p-q) = 1 - sum_t min(p, q) after a rejection (total-variation identity);
    the bonus row's mass is 1; a resampled token always has p > q."""
    rng = np.random.default_rng(14)
    B, K, V = 64, 3, 40
    t = rng.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    q = (t[:, :K] + rng.normal(0, 1.5, size=(B, K, V))).astype(np.float32)
    d = np.stack([[rng.choice(V, p=sps.softmax(q[i, k].astype(np.float64))) for k in range(K)]
                  for i in range(B)]).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    r = o.verify_rejection(t, q, d, u)
    pt = sps.softmax(t.astype(np.float64), axis=2)
    pq = sps.softmax(q.astype(np.float64), axis=2)
    saw_reject = saw_all = False
    for i in range(B):
        a = r["accepted_len"][i]
        if a < K:
            saw_reject = True
            z = 1.0 - np.minimum(pt[i, a], pq[i, a]).sum()
            np.testing.assert_allclose(r["residual_mass"][i], z, rtol=1e-9, atol=1e-14)
            tok = r["bonus"][i]
            assert pt[i, a, tok] > pq[i, a, tok]
        else:
            saw_all = True
            np.testing.assert_allclose(r["residual_mass"][i], 1.0, rtol=1e-12)
    assert saw_reject and saw_all


def pin_special_cases(o):
    """Special cases with known answers."""
    rng = np.random.default_rng(15)
    B, K, V = 16, 4, 24
    t = rng.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    d = rng.integers(0, V, size=(B, K)).astype(np.int32)
    # draft == target: p/q = 1 > u for every u in [0, 1): all K accepted
    u = rng.random((B, K + 1), dtype=np.float32)
    r = o.verify_rejection(t, t[:, :K].copy(), d, u)
    assert (r["accepted_len"] == K).all()
    # u = 0 accepts whenever p > 0; p(d) = 0 (a -inf target logit) rejects
    q = (t[:, :K] + rng.normal(0, 1, size=(B, K, V))).astype(np.float32)
    u0 = np.zeros((B, K + 1), np.float32)
    r = o.verify_rejection(t, q, d, u0)
    assert (r["accepted_len"] == K).all()
    tz = t.copy()
    kill = rng.integers(0, K, size=B)
    for i in range(B):
        tz[i, kill[i], d[i, kill[i]]] = -np.inf
    r = o.verify_rejection(tz, q, d, u0)
    assert (r["accepted_len"] == kill).all()
    # one-hot q on a token with p = 0: rejected at position 0; the residual is p itself,
    # so the draw's CDF boundaries are the cumulative sums of p (probed by bisection)
    t1 = t[:1].copy()
    t1[0, 0, 5] = -np.inf
    q1 = np.full((1, K, V), -np.inf, np.float32)
    q1[0, :, 5] = 0.0
    d1 = np.full((1, K), 5, np.int32)
    p0 = sps.softmax(t1[0, 0].astype(np.float64))
    cdf = np.cumsum(p0)
    for b in range(V - 1):
        if p0[b + 1] == 0.0:
            continue
        uu = np.array([[0.5] * K + [0.0]], np.float32)
        thr = _threshold(lambda x: o.verify_rejection(t1, q1, d1, _with(uu, K, x))["bonus"][0] > b)
        assert abs(thr - cdf[b]) < 2e-7, (b, thr, cdf[b])
        r = o.verify_rejection(t1, q1, d1, _with(uu, K, np.float32(thr)))
        assert r["accepted_len"][0] == 0
    # K = 1
    t2 = t[:, :2].copy()
    r = o.verify_rejection(t2, t2[:, :1].copy(), d[:, :1].copy(), u[:, :2].copy())
    assert (r["accepted_len"] == 1).all()


def _with(u, col, val):
    v = u.copy()
    v[0, col] = val
    return v


def _f32_from_bits(b):
    return np.array([b], np.uint32).view(np.float32)[0]


def _threshold(pred):
    """Smallest float32 u in [0, 1] with pred(u) true, found on the bit patterns (floats in
    [0, 1] are ordered like their bits).  pred must be monotone (false then true)."""
    lo, hi = 0, 0x3F800000                      # bits of 0.0 and 1.0
    if pred(np.float32(0.0)):
        return 0.0
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if pred(_f32_from_bits(mid)):
            hi = mid
        else:
            lo = mid
    return float(_f32_from_bits(hi))


def _thresholds_batched(o, t, q, d, base_u, col, pred):
    """Vectorised _threshold over a batch: for each sequence, the smallest float32 value of
    uniforms[:, col] (other columns from base_u) at which pred(result)[seq] becomes true."""
    B = t.shape[0]
    lo = np.zeros(B, np.int64)
    hi = np.full(B, 0x3F800000, np.int64)
    u = base_u.copy()
    u[:, col] = 0.0
    done0 = pred(o.verify_rejection(t, q, d, u))
    for _ in range(32):
        mid = (lo + hi) // 2
        u[:, col] = mid.astype(np.uint32).view(np.float32)
        p = pred(o.verify_rejection(t, q, d, u))
        hi = np.where(p, mid, hi)
        lo = np.where(p, lo, mid)
    th = hi.astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(done0, 0.0, th)


def _prefix_logits(prefix, V, salt):
    """Deterministic pseudo-random logits for a given token prefix (an autoregressive model)."""
    rng = np.random.default_rng([salt] + [int(x) for x in prefix])
    return rng.normal(0, 1.5, size=V).astype(np.float32)


def pin_exact_distribution(o, K=2, V=8):
    """Brute force over all V^K draft tuples: with accept probabilities and draw laws read
    off the oracle by bisection on the uniforms, the emitted token at every position, given
    the emitted prefix, follows the target's autoregressive law p(. | prefix) exactly (to
    the float32 resolution of the uniforms)."""
    tuples = list(itertools.product(range(V), repeat=K))
    B = len(tuples)
    d = np.array(tuples, np.int32).reshape(B, K)
    t = np.stack([np.stack([_prefix_logits(tp[:k], V, 1) for k in range(K + 1)]) for tp in tuples])
    q = np.stack([np.stack([_prefix_logits(tp[:k], V, 2) for k in range(K)]) for tp in tuples])
    P = sps.softmax(t.astype(np.float64), axis=2)
    Q = sps.softmax(q.astype(np.float64), axis=2)

    # accept probability tau_k(d) = the float32 threshold of u_k (earlier drafts forced in
    # with u = 0, which accepts whenever p > 0)
    tau = np.zeros((B, K))
    for k in range(K):
        base = np.zeros((B, K + 1), np.float32)
        tau[:, k] = _thresholds_batched(o, t, q, d, base, k, lambda r, k=k: r["accepted_len"] <= k)
    # the draw law after a rejection at k: CDF boundaries of u_K
    rho = np.zeros((B, K, V))
    for k in range(K):
        base = np.zeros((B, K + 1), np.float32)
        base[:, k] = np.nextafter(np.float32(1), np.float32(0))      # reject at k when possible
        rej = tau[:, k] < 1.0 - 1e-6
        F = np.zeros((B, V + 1))
        F[:, V] = 1.0
        for b in range(V - 1):
            F[:, b + 1] = _thresholds_batched(o, t, q, d, base, K, lambda r, b=b: r["bonus"] > b)
        rho[:, k] = np.diff(F, axis=1)
        rho[~rej, k] = np.nan
    # the bonus law when all K pass
    base = np.zeros((B, K + 1), np.float32)
    F = np.zeros((B, V + 1))
    F[:, V] = 1.0
    for b in range(V - 1):
        F[:, b + 1] = _thresholds_batched(o, t, q, d, base, K, lambda r, b=b: r["bonus"] > b)
    beta = np.diff(F, axis=1)

    index = {tp: n for n, tp in enumerate(tuples)}
    tol = 2e-6
    # position j < K, prefix x (length j): P(e_j = t | reached j with prefix x)
    for j in range(K):
        for x in itertools.product(range(V), repeat=j):
            rows = [index[x + (v,) + (0,) * (K - j - 1)] for v in range(V)]
            p = P[rows[0], j]
            qd = Q[rows[0], j]
            law = np.zeros(V)
            rej_mass = 0.0
            rho_j = None
            for v, n in enumerate(rows):
                law[v] += qd[v] * tau[n, j]
                rej_mass += qd[v] * (1.0 - tau[n, j])
                if not np.isnan(rho[n, j]).any():
                    rho_j = rho[n, j] if rho_j is None else rho_j
                    np.testing.assert_allclose(rho[n, j], rho_j, atol=tol)
            if rej_mass > 1e-9:
                assert rho_j is not None
                law += rej_mass * rho_j
            np.testing.assert_allclose(law, p, atol=tol, err_msg=f"position {j} prefix {x}")
    # position K: the bonus after K accepted drafts follows p_K(. | d)
    np.testing.assert_allclose(beta, P[:, K], atol=tol)


# ----------------------------------------------------------------------------- build
def pin_build_worked_example(o):
    g = _load("build_worked_example.json")
    r = o.build_draft_batch(
        K=g["K"], block_size=g["block_size"], mask_id=g["mask_id"], pad_id=g["pad_id"],
        T_cap=g["T_cap"], qsl_in=g["qsl_in"], verify_tokens=g["verify_tokens"],
        verify_pos=g["verify_pos"], accepted_len=g["accepted_len"], bonus=g["bonus"],
        block_table=np.array(g["block_table"]))
    for k, v in g["expect"].items():
        assert np.asarray(r[k]).tolist() == v, (k, np.asarray(r[k]).tolist(), v)
    assert r["err"] == 0


def random_build_case(rng, B, K, H, bs, V=1000, L_extra=0, permuted=True, k_len=None):
    """A random valid verify batch with disjoint block tables (a test input, not an oracle).
    With k_len [B], sequence i's span ends in its own K_i drafts (L_i >= K_i + 1)."""
    kn = np.full(B, K) if k_len is None else np.asarray(k_len)
    L = kn + 1 + rng.integers(0, L_extra + 1, size=B)
    qsl = np.zeros(B + 1, np.int64)
    qsl[1:] = np.cumsum(L)
    T_in = int(qsl[-1])
    ctx = rng.integers(0, 200, size=B)
    pos = np.concatenate([c + np.arange(l) for c, l in zip(ctx, L)])
    tok = rng.integers(0, V, size=T_in)
    a = rng.integers(0, kn + 1)
    bonus = rng.integers(0, V, size=B)
    nblk = -(-(ctx + L + K) // bs)
    mb = int(nblk.max())
    ids = rng.permutation(int(nblk.sum())) if permuted else np.arange(int(nblk.sum()))
    table = np.full((B, mb), -1, np.int64)
    off = 0
    for i in range(B):
        table[i, :nblk[i]] = ids[off:off + nblk[i]]
        off += nblk[i]
    hidden = rng.normal(size=(T_in, H)).astype(np.float32)
    hs = rng.normal(size=H).astype(np.float32)
    T_cap = T_in + B * (K - 1) + int(rng.integers(0, 9))
    case = dict(K=K, block_size=bs, mask_id=V, pad_id=V + 1, T_cap=T_cap, qsl_in=qsl,
                verify_tokens=tok, verify_pos=pos, accepted_len=a, bonus=bonus,
                block_table=table, verify_hidden=hidden, h_shared=hs)
    if k_len is not None:
        case["k_len"] = np.asarray(k_len, np.int32)
    return case


def check_build_invariants(case, r):
    """Properties that hold for any valid input (the method's statement, not its code)."""
    K, bs = case["K"], case["block_size"]
    qsl = np.asarray(case["qsl_in"])
    B = len(qsl) - 1
    T_in = int(qsl[-1])
    tok, pos, slot = r["draft_tokens"], r["draft_pos"], r["slot_mapping"]
    kind, src, qo = r["row_kind"], r["hidden_src"], r["qsl_out"]
    assert r["err"] == 0
    assert qo[0] == 0 and qo[B] == T_in + B * (K - 1)
    assert (np.diff(qo) > 0).all()
    vt, vp = np.asarray(case["verify_tokens"]), np.asarray(case["verify_pos"])
    table = np.asarray(case["block_table"])
    valid_slots = []
    kn = np.asarray(case["k_len"]) if case.get("k_len") is not None else np.full(B, K)
    for i in range(B):
        s, L = int(qsl[i]), int(qsl[i + 1] - qsl[i])
        a = int(case["accepted_len"][i])
        Ki = int(kn[i])                                              # R14
        c = L - Ki + a
        span = slice(qo[i], qo[i + 1])
        ks = kind[span]
        want = [0] * (c - 1) + [1] + [2] * (K - 1) + [3] * (Ki - a)
        assert ks.tolist() == want, (i, ks.tolist(), want)
        p = pos[span]
        live = p[: c + K - 1]
        assert (np.diff(live) == 1).all() and live[0] == vp[s]          # consecutive positions
        assert tok[span][c - 1] == case["bonus"][i]
        assert (tok[span][c:c + K - 1] == case["mask_id"]).all()
        assert (tok[span][c + K - 1:] == case["pad_id"]).all()
        assert (tok[span][: c - 1] == vt[s + 1: s + c]).all()         # EAGLE shift
        assert (src[span][:c] == np.arange(s, s + c)).all()
        assert (slot[span][c + K - 1:] == -1).all()                    # rejected: PADDING_SLOT_ID
        assert (p[c + K - 1:] == vp[s + c: s + L]).all()
        for j in range(c + K - 1):
            pp = int(p[j])
            assert slot[span][j] == table[i, pp // bs] * bs + pp % bs
            valid_slots.append(int(slot[span][j]))
        assert r["seq_lens_out"][i] == live[-1] + 1
        sidx = r["sample_idx"][i]
        assert (kind[sidx] == np.array([1] + [2] * (K - 1))).all()
    assert len(set(valid_slots)) == len(valid_slots)                  # disjoint tables
    tail = slice(qo[B], case["T_cap"])
    assert (kind[tail] == 4).all() and (slot[tail] == -1).all() and (pos[tail] == 0).all()
    # hidden rows: bit copies of their source or of h_shared; others untouched
    if r.get("draft_hidden") is not None:
        dh = r["draft_hidden"]
        vh = np.asarray(case["verify_hidden"])
        for row in range(case["T_cap"]):
            if kind[row] in (0, 1):
                assert np.array_equal(dh[row].view(np.uint32), vh[src[row]].view(np.uint32))
            elif kind[row] == 2:
                assert np.array_equal(dh[row].view(np.uint32),
                                      np.asarray(case["h_shared"]).view(np.uint32))
            else:
                assert np.isnan(dh[row]).all()


def pin_build_invariants(o):
    rng = np.random.default_rng(21)
    for K, L_extra, bs in ((1, 0, 4), (3, 0, 4), (7, 0, 16), (4, 5, 8), (31, 2, 16)):
        case = random_build_case(rng, B=13, K=K, H=8, bs=bs, L_extra=L_extra)
        init = np.full((case["T_cap"], 8), np.nan, np.float32)
        r = o.build_draft_batch(**case, draft_hidden_init=init)
        check_build_invariants(case, r)


def pin_build_invalid_values(o):
    """Invalid values: clamped counts, missing blocks, short spans, broken offsets."""
    rng = np.random.default_rng(22)
    case = random_build_case(rng, B=6, K=3, H=4, bs=4)
    c1 = dict(case, accepted_len=np.array([-2, 0, 1, 9, 3, 2]))
    r = o.build_draft_batch(**c1)
    assert r["err"] == 0x2
    c2 = dict(c1, accepted_len=np.array([0, 0, 1, 3, 3, 2]))
    r2 = o.build_draft_batch(**c2)
    for k in ("draft_tokens", "draft_pos", "slot_mapping", "row_kind", "hidden_src", "sample_idx"):
        assert np.array_equal(r[k], r2[k]), k
    t = case["block_table"].copy()
    t[2, :] = -1
    r = o.build_draft_batch(**dict(case, block_table=t))
    assert r["err"] == 0x4
    s = slice(r["qsl_out"][2], r["qsl_out"][3])
    assert (r["slot_mapping"][s] == -1).all()
    q = np.array(case["qsl_in"]).copy()
    q[2] = q[1] + 2                    # sequence 1 has 2 < K+1 rows, sequence 2 more
    r = o.build_draft_batch(**dict(case, qsl_in=q))
    assert r["err"] & 0x8
    s = slice(r["qsl_out"][1], r["qsl_out"][2])
    assert (r["row_kind"][s] == 4).all() and r["seq_lens_out"][1] == 0
    assert (r["sample_idx"][1] == -1).all()
    q = np.array(case["qsl_in"]).copy()
    q[3] = q[2] - 1                    # decreasing offsets: the batch is rejected
    r = o.build_draft_batch(**dict(case, qsl_in=q))
    assert r["err"] == 0x8


# ----------------------------------------------------------------------------- sampling
def pin_sampling(o):
    """Drafter-row sampling: the worked example, greedy = numpy argmax, never a zero-
    probability token, and the law read off by bisection equals the softmax."""
    g = _load("verify_worked_examples.json")["sampling"]
    x = np.log(np.array(g["p"], np.float64)).astype(np.float32)
    for u, tok in zip(g["u"], g["tokens"]):
        r = o.sample_rows(x[None], np.array([u], np.float32))
        assert int(r["tokens"][0]) == tok, (u, r["tokens"])
    rng = np.random.default_rng(31)
    L = rng.normal(0, 2, size=(50, 37)).astype(np.float32)
    L[::3, 5] = -np.inf
    r = o.sample_rows(L)
    assert (r["tokens"] == np.argmax(L, axis=1)).all()
    r = o.sample_rows(L, rng.random(50, dtype=np.float32))
    assert np.isfinite(L[np.arange(50), r["tokens"]]).all()
    P = sps.softmax(L.astype(np.float64), axis=1)
    np.testing.assert_allclose(r["probs"], P[np.arange(50), r["tokens"]], rtol=1e-12)
    # exact law: the CDF boundaries of the inverse-CDF draw are the softmax's cumulative sums
    rows = L[:6]
    Pc = np.cumsum(sps.softmax(rows.astype(np.float64), axis=1), axis=1)
    for n in range(rows.shape[0]):
        for t in range(rows.shape[1] - 1):
            if Pc[n, t + 1] - Pc[n, t] <= 0:
                continue
            thr = _threshold(lambda u, n=n, t=t: o.sample_rows(rows[n:n + 1], np.array([u], np.float32))["tokens"][0] > t)
            assert abs(thr - Pc[n, t]) < 2e-7, (n, t, thr, Pc[n, t])


# ----------------------------------------------------------------------------- K_i (R14)
def pin_k_len_worked_examples(o):
    """Hand-derived examples with per-sequence draft counts (the "k_len" entries of
    tests/golden/verify_worked_examples.json)."""
    g = _load("verify_worked_examples.json")
    for c in g["k_len_cases"]:
        t = np.log(np.array(c["p"], np.float64)).astype(np.float32)[None]
        q = np.log(np.array(c["q"], np.float64)).astype(np.float32)[None]
        d = np.array([c["drafts"]], np.int32)
        u = np.array([c["u"]], np.float32)
        kl = np.array([c["k_len"]], np.int32)
        r = o.verify_rejection(t, q, d, u, k_len=kl)
        e = c["rejection"]
        assert r["out_tokens"][0].tolist() == e["out_tokens"], (c["name"], r["out_tokens"])
        assert int(r["accepted_len"][0]) == e["accepted_len"], c["name"]
        np.testing.assert_allclose(r["residual_mass"][0], e["residual_mass"], rtol=1e-6)
        assert r["flags"][0] == 0 and r["err"] == 0
        gr = o.verify_greedy(t, d, k_len=kl)
        assert gr["out_tokens"][0].tolist() == c["greedy"]["out_tokens"], (c["name"], gr["out_tokens"])


def pin_k_len_reduces_to_truncation(o):
    """A sequence with K_i drafts gives exactly what the fixed-K oracle gives for that
    sequence alone cut to K = K_i (its first K_i+1 target rows, K_i draft rows and drafts,
    uniform columns 0..K_i); K_i = 0 draws the bonus from target row 0 with u_0 (the
    drafter-row sampler) or takes its numpy argmax.  Drafts past K_i are never read: -1
    there sets no error bit.  A count outside [0, K] sets bit 0x20 and is clamped."""
    rng = np.random.default_rng(41)
    B, K, V = 14, 5, 40
    t = rng.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    q = (t[:, :K] + rng.normal(0, 0.5, size=(B, K, V))).astype(np.float32)
    d = np.argmax(q, axis=2).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    kl = np.array([0, K, 1, 2, 3, 4, 5, 0, 1, 3, 2, 5, 4, 1], np.int32)
    for i in range(B):
        d[i, kl[i]:] = -1                                   # unused slots
    r = o.verify_rejection(t, q, d, u, k_len=kl)
    gr = o.verify_greedy(t, d, k_len=kl)
    assert r["err"] == 0 and gr["err"] == 0
    for i in range(B):
        Ki = int(kl[i])
        out, gout = r["out_tokens"][i], gr["out_tokens"][i]
        if Ki == 0:
            s = o.sample_rows(t[i, 0][None], u[i, :1])
            assert out.tolist() == [int(s["tokens"][0])] + [-1] * K
            assert gout.tolist() == [int(np.argmax(t[i, 0]))] + [-1] * K
            assert r["accepted_len"][i] == 0 and gr["accepted_len"][i] == 0
            continue
        ri = o.verify_rejection(t[i:i + 1, :Ki + 1], q[i:i + 1, :Ki], d[i:i + 1, :Ki],
                                u[i:i + 1, :Ki + 1])
        gi = o.verify_greedy(t[i:i + 1, :Ki + 1], d[i:i + 1, :Ki])
        assert out.tolist() == ri["out_tokens"][0].tolist() + [-1] * (K - Ki), i
        assert gout.tolist() == gi["out_tokens"][0].tolist() + [-1] * (K - Ki), i
        assert r["flags"][i] == ri["flags"][0]
        np.testing.assert_allclose(r["residual_mass"][i], ri["residual_mass"][0], rtol=1e-12)
        np.testing.assert_allclose(r["p_at_draft"][i, :Ki], ri["p_at_draft"][0], rtol=1e-12)
    bad = kl.copy()
    bad[3], bad[4] = -1, K + 2
    r2 = o.verify_rejection(t, q, np.where(d < 0, 0, d).astype(np.int32), u, k_len=bad)
    assert r2["err"] & 0x20
    assert r2["accepted_len"][3] == 0 and r2["accepted_len"][4] <= K


def pin_build_k_len(o):
    """Draft batch with per-sequence K_i: with spans of at least K+1 rows, K_i and accepted
    count a give the batch that fixed K gives for a + K - K_i (the same surviving rows);
    spans down to K_i + 1 rows keep the layout invariants (c_i context rows, K-1 masks,
    K_i - a rejected rows)."""
    rng = np.random.default_rng(43)
    K, B = 5, 12
    kl = rng.integers(0, K + 1, size=B).astype(np.int32)
    case = random_build_case(rng, B=B, K=K, H=8, bs=4, L_extra=3, k_len=np.full(B, K))
    case["k_len"] = kl                                      # spans hold >= K+1 rows
    case["accepted_len"] = rng.integers(0, kl + 1).astype(np.int32)
    r = o.build_draft_batch(**case)
    fixed = dict(case, accepted_len=case["accepted_len"] + (K - kl))
    del fixed["k_len"]
    rf = o.build_draft_batch(**fixed)
    assert r["err"] == 0 and rf["err"] == 0
    for k in ("draft_tokens", "draft_pos", "slot_mapping", "row_kind", "hidden_src", "qsl_out",
              "seq_lens_out", "sample_idx", "draft_hidden"):
        assert np.array_equal(r[k], rf[k]), k
    short = random_build_case(rng, B=B, K=K, H=8, bs=4, L_extra=0, k_len=kl)
    init = np.full((short["T_cap"], 8), np.nan, np.float32)
    check_build_invariants(short, o.build_draft_batch(**short, draft_hidden_init=init))
    over = dict(short, accepted_len=np.where(kl > 0, kl + 1, 0).astype(np.int32))
    assert o.build_draft_batch(**over)["err"] & 0x2     # a_i > K_i: clamped, bit set


ALL_PINS = [
    pin_worked_examples, pin_greedy_matches_numpy_argmax, pin_bf16_decoding,
    pin_probabilities_match_scipy, pin_residual_mass_closed_form, pin_special_cases,
    pin_exact_distribution, pin_build_worked_example, pin_build_invariants,
    pin_build_invalid_values, pin_sampling, pin_k_len_worked_examples,
    pin_k_len_reduces_to_truncation, pin_build_k_len,
]
