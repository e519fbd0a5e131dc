"""Allocation helpers around the C-ABI binding: output tensors and verify workspaces.

The functions here only allocate device memory with torch (plumbing) and forward to the
binding; every step of the method runs in libpspec's kernels.
"""
from __future__ import annotations

import torch

from . import _binding as _b


class Workspace:
    """Zero-initialised verify workspace for (B, K, V, mode) and the calls' tuning options
    (None: the process-wide defaults).  Reusable across calls on one stream: each call leaves
    its per-sequence counters back at zero."""

    def __init__(self, B: int, K: int, V: int, rejection: bool, device="cuda", options=None):
        n = _b.pspec_verify_workspace_bytes(B, K, V, rejection, options) if B > 0 else 0
        self.tensor = torch.zeros(max(n, 256), dtype=torch.uint8, device=device)

    def fits(self, B: int, K: int, V: int, rejection: bool, options=None) -> bool:
        return self.tensor.numel() >= _b.pspec_verify_workspace_bytes(B, K, V, rejection, options)


def verify_outputs(Bn: int, K: int, device, diagnostics: bool, rejection: bool,
                   residual_mass: bool = False) -> dict:
    i32 = dict(dtype=torch.int32, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    out = {
        "out_tokens": torch.empty((Bn, K + 1), **i32),
        "accepted_len": torch.empty((Bn,), **i32),
        "bonus": torch.empty((Bn,), **i32),
        "err": torch.zeros((1,), **i32),
    }
    if diagnostics:
        out["target_lse"] = torch.empty((Bn, K + 1), **f32)
        if rejection:
            out["draft_lse"] = torch.empty((Bn, K), **f32)
            out["p_at_draft"] = torch.empty((Bn, K), **f32)
            out["q_at_draft"] = torch.empty((Bn, K), **f32)
            out["residual_mass"] = torch.empty((Bn,), **f32)
    elif residual_mass and rejection:
        out["residual_mass"] = torch.empty((Bn,), **f32)
    return out


def verify_greedy(target_logits: torch.Tensor, draft_tokens: torch.Tensor, *,
                  want_lse: bool = False, workspace: Workspace | None = None, out=None,
                  k_len: torch.Tensor | None = None, options=None, stream=None) -> dict:
    """Greedy verify.  Returns out_tokens, accepted_len, bonus, err (+ target_lse).
    k_len [B] int32 (optional): each sequence's own draft count.  options (optional): a dict
    of pspec_options fields for this call alone."""
    Bn, K1, V = target_logits.shape
    K = K1 - 1
    o = out if out is not None else verify_outputs(Bn, K, target_logits.device, want_lse, False)
    ws = workspace if workspace is not None else Workspace(Bn, K, V, False, target_logits.device,
                                                           options)
    _b.pspec_verify_greedy(target_logits=target_logits, draft_tokens=draft_tokens,
                          out_tokens=o["out_tokens"], accepted_len=o["accepted_len"],
                          bonus=o["bonus"], err=o["err"], workspace=ws.tensor,
                          target_lse=o.get("target_lse") if want_lse else None, k_len=k_len,
                          options=options, stream=stream)
    return o


def verify_rejection(target_logits: torch.Tensor, draft_logits: torch.Tensor,
                     draft_tokens: torch.Tensor, uniforms: torch.Tensor, *,
                     diagnostics: bool = False, residual_mass: bool = False,
                     workspace: Workspace | None = None, out=None,
                     k_len: torch.Tensor | None = None, options=None, stream=None) -> dict:
    """Rejection-rule verify.  Returns out_tokens, accepted_len, bonus, err (+ fp32
    diagnostics target_lse, draft_lse, p_at_draft, q_at_draft, residual_mass; or only
    residual_mass).  options (optional): a dict of pspec_options fields for this call."""
    Bn, K1, V = target_logits.shape
    K = K1 - 1
    o = out if out is not None else verify_outputs(Bn, K, target_logits.device, diagnostics, True,
                                                   residual_mass)
    ws = workspace if workspace is not None else Workspace(Bn, K, V, True, target_logits.device,
                                                           options)
    _b.pspec_verify_rejection(target_logits=target_logits, draft_logits=draft_logits,
                             draft_tokens=draft_tokens, uniforms=uniforms,
                             out_tokens=o["out_tokens"], accepted_len=o["accepted_len"],
                             bonus=o["bonus"], err=o["err"], workspace=ws.tensor,
                             target_lse=o.get("target_lse"), draft_lse=o.get("draft_lse"),
                             p_at_draft=o.get("p_at_draft"), q_at_draft=o.get("q_at_draft"),
                             residual_mass=o.get("residual_mass"), k_len=k_len,
                             options=options, stream=stream)
    return o


def sample_drafts(logits: torch.Tensor, uniforms: torch.Tensor | None = None, *,
                  want_probs: bool = False, workspace: torch.Tensor | None = None,
                  out=None, stream=None) -> dict:
    """Draft tokens from drafter logits [B, K, V]: inverse-CDF sampling with uniforms
    [B, K], or the argmax when uniforms is None.  Returns draft_tokens, err (+ q_at_draft)."""
    Bn, K, V = logits.shape
    dev = logits.device
    o = out if out is not None else {
        "draft_tokens": torch.empty((Bn, K), dtype=torch.int32, device=dev),
        "err": torch.zeros((1,), dtype=torch.int32, device=dev),
    }
    if want_probs and "q_at_draft" not in o:
        o["q_at_draft"] = torch.empty((Bn, K), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else torch.zeros(
        max(256, _b.pspec_sample_workspace_bytes(Bn, K, V)), dtype=torch.uint8, device=dev)
    _b.pspec_sample_drafts(logits=logits, draft_tokens=o["draft_tokens"], err=o["err"],
                           workspace=ws, uniforms=uniforms, q_at_draft=o.get("q_at_draft"),
                           stream=stream)
    return o


def build_outputs(Bn: int, K: int, H: int, T_cap: int, hidden_dtype, device) -> dict:
    i32 = dict(dtype=torch.int32, device=device)
    return {
        "draft_tokens": torch.empty((T_cap,), **i32),
        "draft_pos": torch.empty((T_cap,), **i32),
        "slot_mapping": torch.empty((T_cap,), dtype=torch.int64, device=device),
        "row_kind": torch.empty((T_cap,), dtype=torch.uint8, device=device),
        "hidden_src": torch.empty((T_cap,), **i32),
        "qsl_out": torch.empty((Bn + 1,), **i32),
        "seq_lens_out": torch.empty((Bn,), **i32),
        "sample_idx": torch.empty((Bn, K), **i32),
        "draft_hidden": torch.zeros((T_cap, H), dtype=hidden_dtype, device=device),
        "err": torch.zeros((1,), **i32),
    }


def build_draft_batch(*, K: int, block_size: int, mask_id: int, pad_id: int, T_cap: int,
                      qsl_in, verify_tokens, verify_pos, accepted_len, bonus, block_table,
                      verify_hidden, h_shared, out=None, k_len=None, stream=None) -> dict:
    """P-EAGLE draft-batch construction.  Returns the per-row, per-sequence and hidden
    outputs (see ``include/pspec.h``)."""
    Bn = int(qsl_in.numel()) - 1
    o = out if out is not None else build_outputs(
        Bn, K, int(verify_hidden.shape[1]), T_cap, verify_hidden.dtype, verify_hidden.device)
    _b.pspec_build_draft_batch(K=K, block_size=block_size, mask_id=mask_id, pad_id=pad_id,
                              T_cap=T_cap, qsl_in=qsl_in, verify_tokens=verify_tokens,
                              verify_pos=verify_pos, accepted_len=accepted_len, bonus=bonus,
                              block_table=block_table, verify_hidden=verify_hidden,
                              h_shared=h_shared, draft_tokens=o["draft_tokens"],
                              draft_pos=o["draft_pos"], slot_mapping=o["slot_mapping"],
                              row_kind=o["row_kind"], hidden_src=o["hidden_src"],
                              qsl_out=o["qsl_out"], seq_lens_out=o["seq_lens_out"],
                              sample_idx=o["sample_idx"], draft_hidden=o["draft_hidden"],
                              err=o["err"], k_len=k_len, stream=stream)
    return o


def step(target_logits: torch.Tensor, draft_tokens: torch.Tensor, build: dict, *,
         draft_logits: torch.Tensor | None = None, uniforms: torch.Tensor | None = None,
         residual_mass: bool = False, workspace: Workspace | None = None, out=None,
         build_out=None, k_len: torch.Tensor | None = None, options=None, stream=None) -> tuple:
    """One step: verification (the rejection rule when `uniforms` is given, else greedy)
    and the draft-batch build from its accepted counts and bonus tokens, in one launch when
    the early-exit path takes the verification.  `build` holds the build inputs (K,
    block_size, mask_id, pad_id, T_cap, qsl_in, verify_tokens, verify_pos, block_table,
    verify_hidden, h_shared).  Returns (verify outputs, build outputs)."""
    rej = uniforms is not None
    Bn, K1, V = target_logits.shape
    K = K1 - 1
    dev = target_logits.device
    o = out if out is not None else verify_outputs(Bn, K, dev, False, rej, residual_mass)
    ws = workspace if workspace is not None else Workspace(Bn, K, V, rej, dev, options)
    vh = build["verify_hidden"]
    bo = build_out if build_out is not None else build_outputs(
        Bn, K, int(vh.shape[1]), build["T_cap"], vh.dtype, vh.device)
    bargs = dict(K=build["K"], block_size=build["block_size"], mask_id=build["mask_id"],
                 pad_id=build["pad_id"], T_cap=build["T_cap"], qsl_in=build["qsl_in"],
                 verify_tokens=build["verify_tokens"], verify_pos=build["verify_pos"],
                 accepted_len=None, bonus=None, block_table=build["block_table"],
                 verify_hidden=vh, h_shared=build["h_shared"], draft_tokens=bo["draft_tokens"],
                 draft_pos=bo["draft_pos"], slot_mapping=bo["slot_mapping"],
                 row_kind=bo["row_kind"], hidden_src=bo["hidden_src"], qsl_out=bo["qsl_out"],
                 seq_lens_out=bo["seq_lens_out"], sample_idx=bo["sample_idx"],
                 draft_hidden=bo["draft_hidden"], err=bo["err"])
    if rej:
        _b.pspec_step_rejection(target_logits=target_logits, draft_logits=draft_logits,
                               draft_tokens=draft_tokens, uniforms=uniforms,
                               out_tokens=o["out_tokens"], accepted_len=o["accepted_len"],
                               bonus=o["bonus"], err=o["err"], workspace=ws.tensor, build=bargs,
                               residual_mass=o.get("residual_mass"), k_len=k_len,
                               options=options, stream=stream)
    else:
        _b.pspec_step_greedy(target_logits=target_logits, draft_tokens=draft_tokens,
                             out_tokens=o["out_tokens"], accepted_len=o["accepted_len"],
                             bonus=o["bonus"], err=o["err"], workspace=ws.tensor, build=bargs,
                             k_len=k_len, options=options, stream=stream)
    return o, bo


def prepare_step(target_logits: torch.Tensor, draft_tokens: torch.Tensor, build: dict, *,
                 draft_logits: torch.Tensor | None = None, uniforms: torch.Tensor | None = None,
                 residual_mass: bool = False, workspace: Workspace | None = None, out=None,
                 build_out=None, k_len: torch.Tensor | None = None, options=None) -> tuple:
    """The arguments of ``step`` marshalled once: returns (call, verify outputs, build
    outputs), where ``call(stream=None)`` runs the step on the same tensors with no further
    Python-side marshalling (the buffers' contents may change between calls)."""
    rej = uniforms is not None
    Bn, K1, V = target_logits.shape
    K = K1 - 1
    dev = target_logits.device
    o = out if out is not None else verify_outputs(Bn, K, dev, False, rej, residual_mass)
    ws = workspace if workspace is not None else Workspace(Bn, K, V, rej, dev, options)
    vh = build["verify_hidden"]
    bo = build_out if build_out is not None else build_outputs(
        Bn, K, int(vh.shape[1]), build["T_cap"], vh.dtype, vh.device)
    bargs = dict(K=build["K"], block_size=build["block_size"], mask_id=build["mask_id"],
                 pad_id=build["pad_id"], T_cap=build["T_cap"], qsl_in=build["qsl_in"],
                 verify_tokens=build["verify_tokens"], verify_pos=build["verify_pos"],
                 accepted_len=None, bonus=None, block_table=build["block_table"],
                 verify_hidden=vh, h_shared=build["h_shared"], draft_tokens=bo["draft_tokens"],
                 draft_pos=bo["draft_pos"], slot_mapping=bo["slot_mapping"],
                 row_kind=bo["row_kind"], hidden_src=bo["hidden_src"], qsl_out=bo["qsl_out"],
                 seq_lens_out=bo["seq_lens_out"], sample_idx=bo["sample_idx"],
                 draft_hidden=bo["draft_hidden"], err=bo["err"], k_len=k_len)
    call = _b.prepare_step(target_logits=target_logits, draft_tokens=draft_tokens,
                           out_tokens=o["out_tokens"], accepted_len=o["accepted_len"],
                           bonus=o["bonus"], err=o["err"], workspace=ws.tensor, build=bargs,
                           draft_logits=draft_logits, uniforms=uniforms,
                           residual_mass=o.get("residual_mass"), k_len=k_len, options=options)
    return call, o, bo
