"""Helpers for the GPU parity tests: move inputs to the oracle, run both sides, compare.

Tolerances (floating-point outputs of the fp32 kernels against the double oracle):
  * p_at_draft, q_at_draft, target_lse, draft_lse: 1e-5 relative (the stated bar);
  * residual_mass Z: 1e-5 relative, no absolute floor.  Z = sum over t of
    max(0, p(t) - q(t)); the kernels form each term from fp32 probabilities, add a lane's few
    terms in fp32 and everything above that in double, so the error is about that of the
    terms (1e-7 of each p(t)), which stays below 1e-5 of Z on every workload measured.  Every comparison prints the largest
    relative error of Z.
Integer outputs (tokens, counts, offsets, slots) must be bit-exact, except for sequences
the oracle flags as near-ties (an accept decision with |u - p/q| < 1e-6, or a draw within
1e-6 * Z of a CDF boundary): those are excluded from the integer comparison and counted.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

THREADS = max(1, os.cpu_count() or 1)
RTOL = 1e-5


def host_logits(x: torch.Tensor) -> np.ndarray:
    """Logits for the oracle: fp32 as float32, bf16 as raw uint16 bits."""
    x = x.detach().contiguous()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).cpu().numpy().view(np.uint16)
    return x.float().cpu().numpy()


def np_i32(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().numpy().astype(np.int32)


def oracle_rejection(target, draft, drafts, u, seqs=None, k_len=None):
    idx = slice(None) if seqs is None else torch.as_tensor(seqs, device=target.device)
    return oracle.verify_rejection(host_logits(target[idx]), host_logits(draft[idx]),
                                   np_i32(drafts[idx]), u[idx].cpu().numpy(), threads=THREADS,
                                   k_len=None if k_len is None else np_i32(k_len[idx]))


def oracle_greedy(target, drafts, seqs=None, want_lse=True, k_len=None):
    idx = slice(None) if seqs is None else torch.as_tensor(seqs, device=target.device)
    return oracle.verify_greedy(host_logits(target[idx]), np_i32(drafts[idx]),
                                want_lse=want_lse, threads=THREADS,
                                k_len=None if k_len is None else np_i32(k_len[idx]))


def _rel_ok(a, b, rtol=RTOL, atol=0.0):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    ok = both_inf | (np.abs(a - b) <= rtol * np.abs(b) + atol)
    return ok


def compare_rejection(g: dict, o: dict, seqs=None, K=None):
    """Compare GPU rejection outputs (torch, all sequences) with oracle outputs (numpy, the
    sequences in `seqs`).  Unflagged sequences must match bit for bit.  Flagged ones (the
    oracle saw a near-tie the fp32 kernel may resolve either way) must still agree on the
    accepted prefix up to the first flagged decision and emit a valid token; they are
    counted.  Returns (flagged, flagged_but_identical)."""
    sel = slice(None) if seqs is None else np.asarray(seqs)
    G = {k: v.detach().cpu().numpy()[sel] for k, v in g.items()
         if isinstance(v, torch.Tensor) and k != "err"}
    flags = o["flags"]
    clean = flags == 0
    same = np.ones(len(flags), bool)
    for k in ("out_tokens", "accepted_len", "bonus"):
        eq = np.all((G[k] == o[k]).reshape(len(flags), -1), axis=1)
        same &= eq
        bad = np.nonzero(~eq & clean)[0]
        assert bad.size == 0, (k, bad[:10], G[k][bad[:3]], o[k][bad[:3]], flags[bad[:3]])
    for i in np.nonzero(~clean)[0]:
        if flags[i] == 2:              # only the draw was near a boundary: the prefix is exact
            assert G["accepted_len"][i] == o["accepted_len"][i], i
        a = int(G["accepted_len"][i])
        assert 0 <= G["bonus"][i] and G["out_tokens"][i, a] == G["bonus"][i]
    for k in ("p_at_draft", "q_at_draft", "target_lse", "draft_lse"):
        if k in G:
            ok = _rel_ok(G[k], o[k])
            assert ok.all(), (k, np.argwhere(~ok)[:5], G[k][~ok][:5], o[k][~ok][:5])
    if "residual_mass" in G:
        same_a = G["accepted_len"] == o["accepted_len"]
        gz = np.asarray(G["residual_mass"], np.float64)[same_a]
        oz = np.asarray(o["residual_mass"], np.float64)[same_a]
        nz = oz > 0
        worst = float(np.max(np.abs(gz - oz)[nz] / oz[nz])) if nz.any() else 0.0
        print(f"[parity] residual mass: {int(same_a.sum())} compared, max relative error "
              f"{worst:.2e}")
        ok = _rel_ok(gz, oz)
        assert ok.all(), ("residual_mass", gz[~ok][:5], oz[~ok][:5])
    flagged = int((~clean).sum())
    print(f"[parity] {len(flags)} sequences, {flagged} flagged near-ties, "
          f"{int((~clean & same).sum())} of those identical anyway")
    return flagged, int((~clean & same).sum())


def compare_greedy(g: dict, o: dict, seqs=None):
    sel = slice(None) if seqs is None else np.asarray(seqs)
    for k in ("out_tokens", "accepted_len", "bonus"):
        G = g[k].detach().cpu().numpy()[sel]
        assert np.array_equal(G, o[k]), (k, np.argwhere(G != o[k])[:5])
    if g.get("target_lse") is not None and o.get("target_lse") is not None:
        G = g["target_lse"].detach().cpu().numpy()[sel]
        ok = _rel_ok(G, o["target_lse"])
        assert ok.all(), ("target_lse", G[~ok][:5], o["target_lse"][~ok][:5])


def check_verify_invariants(g: dict, drafts: torch.Tensor, V: int):
    """Properties that hold for every sequence at any size."""
    out = g["out_tokens"].cpu().numpy()
    a = g["accepted_len"].cpu().numpy()
    bonus = g["bonus"].cpu().numpy()
    d = drafts.cpu().numpy()
    B, K1 = out.shape
    K = K1 - 1
    assert ((a >= 0) & (a <= K)).all()
    assert ((bonus >= 0) & (bonus < V)).all()
    cols = np.arange(K + 1)[None, :]
    m = np.arange(K)[None, :] < a[:, None]
    assert (out[:, :K][m] == d[m]).all()                 # accepted tokens are the drafts
    assert (out[np.arange(B), a] == bonus).all()
    assert (out[cols > a[:, None]] == -1).all()
    assert int(g["err"].item()) == 0


def oracle_build(inp: dict, hidden_init: np.ndarray | None):
    """The oracle on a build-input dict from speculative_decoding_step_pspec_b200.inputs."""
    vh = inp["verify_hidden"]
    hs = inp["h_shared"]
    if vh.dtype == torch.bfloat16:
        vh_np = vh.view(torch.int16).cpu().numpy()
        hs_np = hs.view(torch.int16).cpu().numpy()
    else:
        vh_np = vh.cpu().numpy()
        hs_np = hs.cpu().numpy()
    return oracle.build_draft_batch(
        K=inp["K"], block_size=inp["block_size"], mask_id=inp["mask_id"], pad_id=inp["pad_id"],
        T_cap=inp["T_cap"], qsl_in=np_i32(inp["qsl_in"]), verify_tokens=np_i32(inp["verify_tokens"]),
        verify_pos=np_i32(inp["verify_pos"]), accepted_len=np_i32(inp["accepted_len"]),
        bonus=np_i32(inp["bonus"]), block_table=np_i32(inp["block_table"]),
        verify_hidden=vh_np, h_shared=hs_np, draft_hidden_init=hidden_init,
        k_len=None if inp.get("k_len") is None else np_i32(inp["k_len"]))


def hidden_sentinel(T_cap, H, dtype, device):
    """A draft_hidden buffer filled with a byte pattern the method never writes."""
    t = torch.empty((T_cap, H), dtype=dtype, device=device)
    t.view(torch.uint8).fill_(0xA5)
    return t


def compare_build(g: dict, o: dict, check_hidden=True):
    for k in ("draft_tokens", "draft_pos", "slot_mapping", "row_kind", "hidden_src", "qsl_out",
              "seq_lens_out", "sample_idx"):
        G = g[k].detach().cpu().numpy()
        assert G.shape == o[k].shape, k
        assert np.array_equal(G, o[k]), (k, np.argwhere(G != o[k])[:5])
    assert int(g["err"].item()) == o["err"]
    if check_hidden:
        G = g["draft_hidden"]
        Gb = G.view(torch.int16).cpu().numpy() if G.dtype == torch.bfloat16 else G.cpu().numpy().view(np.int32)
        Ob = o["draft_hidden"].view(np.int16) if o["draft_hidden"].dtype.itemsize == 2 else o["draft_hidden"].view(np.int32)
        assert np.array_equal(Gb, Ob), np.argwhere(Gb != Ob)[:5]
