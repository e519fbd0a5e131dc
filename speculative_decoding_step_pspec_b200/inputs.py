"""Seeded synthetic inputs for the speculative-decoding step.

This module only draws random inputs: it holds none of the verify or batch-construction
arithmetic, and both the CUDA path and the CPU oracle receive exactly the arrays it
returns.  The workloads mirror the pages' deployment shapes (GPT-OSS / Qwen3 vocabularies
and hidden sizes, concurrency 1 / 64 / 1024 and draft depths 1..8 of "Eagle parallel
speculative decoding, vLLM, TorchSpec", sections "Production deployment" and
"Parallel architecture"); no benchmark suite item is reproduced.

Recipe (per workload, seed fixed per workload):
  * logits: target N(0, sigma_t) per element (plus a Zipf-shaped -s*ln(id+1) bias for the
    large-batch workload), draft = target row + N(0, sigma_d), stored bf16 (fp32 for the
    tiny workload);
  * sampled drafts are drawn from softmax(draft row) with torch's sampler, greedy drafts
    are torch.argmax of the draft row;
  * uniforms: torch.rand, float32, clamped below 1;
  * verify batch: K+1 rows per sequence at positions ctx_i + j, row 0 a random token and
    rows 1..K the sequence's drafts; hidden states N(0,1); h_shared N(0,1);
  * block tables: ceil((ctx_i + 2K) / block_size) blocks per sequence, from a global pool
    allocated in order or (mid-concurrency) as a random permutation; unused entries -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

LAST_BELOW_ONE = float(np.nextafter(np.float32(1.0), np.float32(0.0)))


@dataclass
class Workload:
    name: str
    B: int
    K: int
    V: int
    H: int
    block_size: int
    dtype: torch.dtype          # logits and hidden dtype
    seed: int
    sigma_t: float = 3.0
    sigma_d: float = 0.7
    zipf_s: float = 0.0
    ctx: str = "fixed"          # fixed | uniform | loguniform
    ctx_args: tuple = (4096,)
    a_prev: str = "uniform"     # uniform | geometric
    permuted_blocks: bool = False
    capture_pad: int = 16       # T_cap rounded up to a multiple of this
    extra: dict = field(default_factory=dict)


# The five workloads.  Sizes: (B, K, V, H).
TINY = Workload("tiny", 4, 3, 32, 16, 4, torch.float32, seed=0, sigma_t=2.0, sigma_d=0.5,
                ctx="uniform", ctx_args=(5, 20))
C1 = Workload("c1", 1, 7, 201088, 2880, 16, torch.bfloat16, seed=1, sigma_t=3.0, sigma_d=0.7,
              ctx="fixed", ctx_args=(4096,))
C64 = Workload("c64", 64, 7, 151936, 2048, 16, torch.bfloat16, seed=2, sigma_t=3.0,
               sigma_d=1.0, ctx="uniform", ctx_args=(512, 16384), a_prev="geometric",
               permuted_blocks=True)
B1024 = Workload("b1024", 1024, 7, 201088, 2880, 16, torch.bfloat16, seed=3, sigma_t=3.0,
                 sigma_d=0.8, zipf_s=1.1, ctx="loguniform", ctx_args=(128, 100000))
DEPTH_K = (1, 3, 5, 7, 8)
DEPTH_SIGMA = (0.3, 0.7, 1.5)


def depth(K: int, sigma: float) -> Workload:
    """Depth-sweep workload: B=256, V=128256, H=4096, K in DEPTH_K, sigma in DEPTH_SIGMA."""
    ki, si = DEPTH_K.index(K), DEPTH_SIGMA.index(sigma)
    return Workload(f"depth_K{K}_s{sigma}", 256, K, 128256, 4096, 16, torch.bfloat16,
                    seed=100 + 10 * ki + si, sigma_t=3.0, sigma_d=sigma, ctx="fixed",
                    ctx_args=(4096,))


WORKLOADS = {w.name: w for w in (TINY, C1, C64, B1024)}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller cases of the same recipe)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _ctx_lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.ctx == "fixed":
        return np.full(w.B, w.ctx_args[0], np.int64)
    if w.ctx == "uniform":
        lo, hi = w.ctx_args
        return rng.integers(lo, hi + 1, size=w.B)
    lo, hi = w.ctx_args
    return np.floor(np.exp(rng.uniform(math.log(lo), math.log(hi), size=w.B))).astype(np.int64)


def _a_prev(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.a_prev == "geometric":
        return np.minimum(rng.geometric(0.3, size=w.B) - 1, w.K)
    return rng.integers(0, w.K + 1, size=w.B)


def logits(w: Workload, device="cpu", chunk_rows: int = 256):
    """Target [B, K+1, V] and draft [B, K, V] logits in ``w.dtype`` on ``device``."""
    g = _gen(device, w.seed)
    B, K, V = w.B, w.K, w.V
    target = torch.empty((B, K + 1, V), dtype=w.dtype, device=device)
    draft = torch.empty((B, K, V), dtype=w.dtype, device=device)
    bias = None
    if w.zipf_s:
        bias = -w.zipf_s * torch.log(torch.arange(V, device=device, dtype=torch.float32) + 1.0)
    tflat = target.view(B * (K + 1), V)
    per = max(1, chunk_rows // (K + 1))
    for b0 in range(0, B, per):
        b1 = min(B, b0 + per)
        t = torch.randn((b1 - b0, K + 1, V), generator=g, device=device) * w.sigma_t
        if bias is not None:
            t += bias
        target[b0:b1] = t.to(w.dtype)
        n = torch.randn((b1 - b0, K, V), generator=g, device=device) * w.sigma_d
        draft[b0:b1] = (target[b0:b1, :K].float() + n).to(w.dtype)
        del t, n
    del tflat
    return target, draft


def draft_tokens(w: Workload, draft: torch.Tensor, chunk_rows: int = 512):
    """Sampled drafts (from softmax of each draft row) and greedy drafts (argmax), [B, K]."""
    device = draft.device
    g = _gen(device, w.seed + 7919)
    B, K, V = draft.shape
    rows = draft.view(B * K, V)
    sampled = torch.empty(B * K, dtype=torch.int32, device=device)
    greedy = torch.empty(B * K, dtype=torch.int32, device=device)
    for r0 in range(0, B * K, chunk_rows):
        r1 = min(B * K, r0 + chunk_rows)
        x = rows[r0:r1].float()
        sampled[r0:r1] = torch.multinomial(torch.softmax(x, dim=-1), 1, generator=g)[:, 0].int()
        greedy[r0:r1] = torch.argmax(x, dim=-1).int()
        del x
    return sampled.view(B, K), greedy.view(B, K)


def uniforms(w: Workload, device="cpu"):
    """Per-position uniforms [B, K+1] in [0, 1) (float32)."""
    g = _gen(device, w.seed + 104729)
    u = torch.rand((w.B, w.K + 1), generator=g, device=device, dtype=torch.float32)
    return u.clamp_(max=LAST_BELOW_ONE)


def tiny_verify_numpy(w: Workload = TINY):
    """The tiny workload drawn with numpy's default_rng(seed) in the stated order.

    Returns fp32 target [B, K+1, V], draft [B, K, V], sampled drafts [B, K] and uniforms
    [B, K+1], plus the context lengths and previous accepted counts."""
    rng = np.random.default_rng(w.seed)
    B, K, V = w.B, w.K, w.V
    ctx = rng.integers(w.ctx_args[0], w.ctx_args[1] + 1, size=B)
    a_prev = rng.integers(0, K + 1, size=B)
    target = rng.normal(0.0, w.sigma_t, size=(B, K + 1, V)).astype(np.float32)
    draft = (target[:, :K] + rng.normal(0.0, w.sigma_d, size=(B, K, V))).astype(np.float32)
    d = np.empty((B, K), np.int32)
    for i in range(B):
        for k in range(K):
            x = draft[i, k].astype(np.float64)
            p = np.exp(x - x.max())
            d[i, k] = rng.choice(V, p=p / p.sum())
    u = rng.random((B, K + 1), dtype=np.float32)
    return dict(target=target, draft=draft, draft_tokens=d, uniforms=u, ctx=ctx, a_prev=a_prev)


def build_inputs(w: Workload, device="cpu", ctx=None, a_prev=None, drafts=None):
    """Verify-batch, block-table and hidden-state inputs of the draft-batch construction.

    ``ctx`` / ``a_prev`` override the drawn context lengths and previous accepted counts;
    ``drafts`` [B, K] fills verify rows 1..K (random tokens when None)."""
    rng = np.random.default_rng(w.seed + 31337)
    B, K, H, bs = w.B, w.K, w.H, w.block_size
    ctx = np.asarray(ctx if ctx is not None else _ctx_lengths(w, rng), np.int64)
    a = np.asarray(a_prev if a_prev is not None else _a_prev(w, rng), np.int64)
    L = np.full(B, K + 1, np.int64)
    qsl_in = np.zeros(B + 1, np.int64)
    qsl_in[1:] = np.cumsum(L)
    T_in = int(qsl_in[-1])
    pos = np.concatenate([c + np.arange(K + 1) for c in ctx]) if B else np.zeros(0, np.int64)
    tok = rng.integers(0, w.V, size=T_in)
    if drafts is not None:
        dn = np.asarray(drafts.cpu() if torch.is_tensor(drafts) else drafts).reshape(B, K)
        tok.reshape(B, K + 1)[:, 1:] = dn
    bonus = rng.integers(0, w.V, size=B)
    nblk = -(-(ctx + 2 * K) // bs)
    max_blocks = int(nblk.max()) if B else 1
    pool = int(nblk.sum())
    ids = rng.permutation(pool) if w.permuted_blocks else np.arange(pool)
    table = np.full((B, max_blocks), -1, np.int64)
    off = 0
    for i in range(B):
        table[i, :nblk[i]] = ids[off:off + nblk[i]]
        off += nblk[i]
    T_cap = T_in + B * (K - 1)
    T_cap = -(-T_cap // w.capture_pad) * w.capture_pad if T_cap else w.capture_pad
    g = _gen(device, w.seed + 4242)
    hidden = torch.randn((T_in, H), generator=g, device=device).to(w.dtype)
    h_shared = torch.randn((H,), generator=g, device=device).to(w.dtype)

    def i32(x):
        return torch.as_tensor(np.ascontiguousarray(x, dtype=np.int32), device=device)

    return dict(
        B=B, K=K, H=H, block_size=bs, max_blocks=max_blocks, mask_id=w.V, pad_id=w.V + 1,
        T_in=T_in, T_cap=T_cap, ctx=ctx,
        qsl_in=i32(qsl_in), verify_tokens=i32(tok), verify_pos=i32(pos),
        accepted_len=i32(a), bonus=i32(bonus), block_table=i32(table),
        verify_hidden=hidden, h_shared=h_shared,
    )
