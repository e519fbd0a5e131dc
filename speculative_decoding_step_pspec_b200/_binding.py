"""Thin ctypes binding of libpspec (``include/pspec.h``): argument marshalling only.

Each function has the C entry point's name, takes torch tensors (device memory) for the
struct's pointer fields, fills the C argument struct, and calls the library on the given
stream (torch's current stream by default).  A non-OK status raises ``PspecError``.
Nothing here computes any part of the method; if ``libpspec.so`` is missing the import
fails (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpspec.so")

PSPEC_OK, PSPEC_ERR_INVALID_ARG, PSPEC_ERR_UNSUPPORTED, PSPEC_ERR_CUDA, PSPEC_ERR_WORKSPACE = range(5)
PSPEC_F32, PSPEC_BF16 = 0, 1
PSPEC_DEVERR_TOKEN_RANGE, PSPEC_DEVERR_ACCEPT_RANGE = 0x1, 0x2
PSPEC_DEVERR_BLOCK_RANGE, PSPEC_DEVERR_LAYOUT = 0x4, 0x8
PSPEC_DEVERR_KLEN_RANGE = 0x20
PSPEC_ROW_CTX, PSPEC_ROW_NTP, PSPEC_ROW_MASK, PSPEC_ROW_REJ, PSPEC_ROW_PAD = range(5)
PSPEC_PADDING_SLOT_ID = -1
PSPEC_MAX_K = 31

EXPORTED = (
    "pspec_verify_workspace_bytes", "pspec_verify_greedy", "pspec_verify_rejection",
    "pspec_build_draft_batch", "pspec_status_string", "pspec_last_launches",
    "pspec_set_verify_path", "pspec_last_verify_path", "pspec_set_cluster_size",
    "pspec_sample_workspace_bytes", "pspec_sample_drafts",
    "pspec_set_segment_elems", "pspec_set_split_event", "pspec_verify_greedy_noalloc",
    "pspec_step_greedy", "pspec_step_rejection", "pspec_set_step_fusion",
    "pspec_set_tail_split", "pspec_last_cluster_size", "pspec_get_options",
    "pspec_verify_workspace_bytes_opt",
)


class PspecError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {pspec_status_string(status)} ({status})")
        self.status = status


_P = ctypes.c_void_p
_I = ctypes.c_int


class pspec_options(ctypes.Structure):
    """Tuning of one call (0 = automatic in every field); see include/pspec.h."""
    _fields_ = [
        ("verify_path", _I), ("cluster_size", _I), ("tail_split", _I), ("step_fusion", _I),
        ("segment_elems", ctypes.c_longlong),
    ]


class pspec_verify_args(ctypes.Structure):
    _fields_ = [
        ("B", _I), ("K", _I), ("V", _I), ("ld", ctypes.c_longlong), ("dtype", _I),
        ("target_logits", _P), ("draft_logits", _P), ("draft_tokens", _P), ("uniforms", _P),
        ("out_tokens", _P), ("accepted_len", _P), ("bonus", _P),
        ("target_lse", _P), ("draft_lse", _P), ("p_at_draft", _P), ("q_at_draft", _P),
        ("residual_mass", _P), ("err", _P), ("k_len", _P),
        ("options", ctypes.POINTER(pspec_options)),
    ]


class pspec_sample_args(ctypes.Structure):
    _fields_ = [
        ("B", _I), ("K", _I), ("V", _I), ("ld", ctypes.c_longlong), ("dtype", _I),
        ("logits", _P), ("uniforms", _P), ("draft_tokens", _P), ("q_at_draft", _P), ("err", _P),
    ]


class pspec_build_args(ctypes.Structure):
    _fields_ = [
        ("B", _I), ("K", _I), ("H", _I), ("hidden_dtype", _I), ("block_size", _I),
        ("max_blocks", _I), ("mask_id", _I), ("pad_id", _I), ("T_in", _I), ("T_cap", _I),
        ("qsl_in", _P), ("verify_tokens", _P), ("verify_pos", _P), ("accepted_len", _P),
        ("bonus", _P), ("block_table", _P), ("verify_hidden", _P), ("h_shared", _P),
        ("draft_tokens", _P), ("draft_pos", _P), ("slot_mapping", _P), ("row_kind", _P),
        ("hidden_src", _P), ("qsl_out", _P), ("seq_lens_out", _P), ("sample_idx", _P),
        ("draft_hidden", _P), ("err", _P), ("k_len", _P),
    ]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libpspec.so not found at {_LIB_PATH}: build it with "
            "`python -m speculative_decoding_step_pspec_b200.build_lib` (there is no fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    lib.pspec_verify_workspace_bytes.argtypes = [_I, _I, _I, _I]
    lib.pspec_verify_workspace_bytes.restype = ctypes.c_size_t
    lib.pspec_verify_workspace_bytes_opt.argtypes = [_I, _I, _I, _I, ctypes.POINTER(pspec_options)]
    lib.pspec_verify_workspace_bytes_opt.restype = ctypes.c_size_t
    lib.pspec_get_options.argtypes = [ctypes.POINTER(pspec_options)]
    lib.pspec_get_options.restype = None
    for fn in ("pspec_verify_greedy", "pspec_verify_rejection"):
        getattr(lib, fn).argtypes = [ctypes.POINTER(pspec_verify_args), _P, ctypes.c_size_t, _P]
        getattr(lib, fn).restype = _I
    lib.pspec_sample_workspace_bytes.argtypes = [_I, _I, _I]
    lib.pspec_sample_workspace_bytes.restype = ctypes.c_size_t
    lib.pspec_sample_drafts.argtypes = [ctypes.POINTER(pspec_sample_args), _P, ctypes.c_size_t, _P]
    lib.pspec_sample_drafts.restype = _I
    lib.pspec_build_draft_batch.argtypes = [ctypes.POINTER(pspec_build_args), _P]
    lib.pspec_build_draft_batch.restype = _I
    for fn in (lib.pspec_step_greedy, lib.pspec_step_rejection):
        fn.argtypes = [ctypes.POINTER(pspec_verify_args), ctypes.POINTER(pspec_build_args), _P,
                       ctypes.c_size_t, _P]
        fn.restype = _I
    lib.pspec_status_string.argtypes = [_I]
    lib.pspec_status_string.restype = ctypes.c_char_p
    lib.pspec_last_launches.argtypes = []
    lib.pspec_last_launches.restype = _I
    lib.pspec_set_verify_path.argtypes = [_I]
    lib.pspec_set_verify_path.restype = None
    lib.pspec_set_step_fusion.argtypes = [_I]
    lib.pspec_set_step_fusion.restype = None
    lib.pspec_set_tail_split.argtypes = [_I]
    lib.pspec_set_tail_split.restype = None
    lib.pspec_set_cluster_size.argtypes = [_I]
    lib.pspec_set_cluster_size.restype = None
    lib.pspec_last_verify_path.argtypes = []
    lib.pspec_last_verify_path.restype = _I
    lib.pspec_last_cluster_size.argtypes = []
    lib.pspec_last_cluster_size.restype = _I
    lib.pspec_set_segment_elems.argtypes = [ctypes.c_longlong]
    lib.pspec_set_segment_elems.restype = None
    lib.pspec_set_split_event.argtypes = [_P]
    lib.pspec_set_split_event.restype = None
    return lib


LIB = _load()


def library_path() -> str:
    return _LIB_PATH


# --------------------------------------------------------------------------- helpers
_DT = {torch.float32: PSPEC_F32, torch.bfloat16: PSPEC_BF16}


def _ptr(t, dtype=None, name="tensor"):
    """Device pointer of a tensor (None -> NULL), with a dtype check."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _logits_layout(t: torch.Tensor, rows: int, name: str):
    """(B, V, ld, dtype) of a [B, rows, V] logits view whose rows may be padded to ld."""
    if t.dim() != 3 or t.shape[1] != rows:
        raise ValueError(f"{name} must be [B, {rows}, V], got {tuple(t.shape)}")
    if t.dtype not in _DT:
        raise TypeError(f"{name} must be float32 or bfloat16, got {t.dtype}")
    B, _, V = t.shape
    ld = t.stride(1) if rows > 1 else t.stride(0)      # one row per sequence: the batch stride
    if (V > 1 and t.stride(2) != 1) or (B > 1 and t.stride(0) != rows * ld) or ld < V:
        raise ValueError(f"{name} must be row-major with a uniform row stride")
    return B, V, ld, _DT[t.dtype]


# --------------------------------------------------------------------------- entry points
def pspec_status_string(status: int) -> str:
    return LIB.pspec_status_string(int(status)).decode()


def pspec_last_launches() -> int:
    """Kernel launches the most recent successful call on this thread issued."""
    return LIB.pspec_last_launches()


def pspec_set_cluster_size(G: int) -> None:
    """CTAs per cluster on the early-exit path: 2, 4, 8, 12, 16, or 0 for automatic."""
    LIB.pspec_set_cluster_size(int(G))


def pspec_last_verify_path() -> int:
    """1 full sweep, 2 early exit: the path of the most recent verify call on this thread."""
    return LIB.pspec_last_verify_path()


def pspec_last_cluster_size() -> int:
    """CTAs per cluster of the last early-exit verify on this thread (0 before any)."""
    return LIB.pspec_last_cluster_size()


def pspec_set_verify_path(path: int) -> None:
    """Process-wide default: 0 automatic, 1 full sweep, 2 early exit (see include/pspec.h)."""
    LIB.pspec_set_verify_path(int(path))


def pspec_set_step_fusion(mode: int) -> None:
    """Fusion of pspec_step_*'s two halves into one launch: 0 automatic, 1 always, 2 never."""
    LIB.pspec_set_step_fusion(int(mode))


def pspec_set_tail_split(n: int) -> None:
    """Early exit: sequences given to a second, wider launch (0 auto, -1 never)."""
    LIB.pspec_set_tail_split(int(n))


def pspec_get_options() -> dict:
    """The process-wide defaults of the tuning options, as a dict."""
    o = pspec_options()
    LIB.pspec_get_options(ctypes.byref(o))
    return {f: getattr(o, f) for f, _ in pspec_options._fields_}


def make_options(options) -> "pspec_options | None":
    """A pspec_options struct from a dict of its fields (missing fields 0), or None."""
    if options is None or isinstance(options, pspec_options):
        return options
    o = pspec_options()
    for k, v in dict(options).items():
        if k not in {f for f, _ in pspec_options._fields_}:
            raise KeyError(f"unknown pspec_options field {k!r}")
        setattr(o, k, int(v))
    return o


def pspec_set_segment_elems(elems: int) -> None:
    LIB.pspec_set_segment_elems(int(elems))


def pspec_set_split_event(event) -> None:
    """Record ``event`` (a torch.cuda.Event, or None to stop) between the two launches of
    every later pspec_verify_rejection call."""
    LIB.pspec_set_split_event(None if event is None else event.cuda_event)


def pspec_verify_workspace_bytes(B: int, K: int, V: int, rejection: bool, options=None) -> int:
    if options is None:
        return int(LIB.pspec_verify_workspace_bytes(int(B), int(K), int(V), int(bool(rejection))))
    o = make_options(options)
    return int(LIB.pspec_verify_workspace_bytes_opt(int(B), int(K), int(V), int(bool(rejection)),
                                                    ctypes.byref(o)))


def _verify_args(target_logits, draft_logits, draft_tokens, uniforms, out_tokens,
                 accepted_len, bonus, err, target_lse, draft_lse, p_at_draft, q_at_draft,
                 residual_mass, K, k_len=None, options=None):
    B, V, ld, dt = _logits_layout(target_logits, K + 1, "target_logits")
    a = pspec_verify_args()
    o = make_options(options)
    if o is not None:
        a.options = ctypes.pointer(o)          # kept alive by the struct until the call
    a.B, a.K, a.V, a.ld, a.dtype = B, K, V, ld, dt
    a.target_logits = target_logits.data_ptr()
    if draft_logits is not None:
        Bd, Vd, ldd, dtd = _logits_layout(draft_logits, K, "draft_logits")
        if (Bd, Vd, ldd, dtd) != (B, V, ld, dt):
            raise ValueError("draft_logits must match target_logits in B, V, stride and dtype")
        a.draft_logits = draft_logits.data_ptr()
    a.draft_tokens = _ptr(draft_tokens, torch.int32, "draft_tokens")
    a.uniforms = _ptr(uniforms, torch.float32, "uniforms")
    a.out_tokens = _ptr(out_tokens, torch.int32, "out_tokens")
    a.accepted_len = _ptr(accepted_len, torch.int32, "accepted_len")
    a.bonus = _ptr(bonus, torch.int32, "bonus")
    a.target_lse = _ptr(target_lse, torch.float32, "target_lse")
    a.draft_lse = _ptr(draft_lse, torch.float32, "draft_lse")
    a.p_at_draft = _ptr(p_at_draft, torch.float32, "p_at_draft")
    a.q_at_draft = _ptr(q_at_draft, torch.float32, "q_at_draft")
    a.residual_mass = _ptr(residual_mass, torch.float32, "residual_mass")
    a.err = _ptr(err, torch.int32, "err")
    a.k_len = _ptr(k_len, torch.int32, "k_len")
    return a


def pspec_verify_greedy(*, target_logits, draft_tokens, out_tokens, accepted_len, bonus, err,
                        workspace, target_lse=None, k_len=None, options=None, stream=None) -> None:
    K = int(target_logits.shape[1]) - 1
    a = _verify_args(target_logits, None, draft_tokens, None, out_tokens, accepted_len, bonus,
                     err, target_lse, None, None, None, None, K, k_len, options)
    st = LIB.pspec_verify_greedy(ctypes.byref(a), _ptr(workspace, torch.uint8, "workspace"),
                                 workspace.numel(), _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_verify_greedy", st)


def pspec_verify_rejection(*, target_logits, draft_logits, draft_tokens, uniforms, out_tokens,
                           accepted_len, bonus, err, workspace, target_lse=None, draft_lse=None,
                           p_at_draft=None, q_at_draft=None, residual_mass=None,
                           k_len=None, options=None, stream=None) -> None:
    K = int(target_logits.shape[1]) - 1
    a = _verify_args(target_logits, draft_logits, draft_tokens, uniforms, out_tokens,
                     accepted_len, bonus, err, target_lse, draft_lse, p_at_draft, q_at_draft,
                     residual_mass, K, k_len, options)
    st = LIB.pspec_verify_rejection(ctypes.byref(a), _ptr(workspace, torch.uint8, "workspace"),
                                    workspace.numel(), _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_verify_rejection", st)


def pspec_sample_workspace_bytes(B: int, K: int, V: int) -> int:
    return int(LIB.pspec_sample_workspace_bytes(int(B), int(K), int(V)))


def pspec_sample_drafts(*, logits, draft_tokens, err, workspace, uniforms=None, q_at_draft=None,
                        stream=None) -> None:
    K = int(logits.shape[1])
    Bn, V, ld, dt = _logits_layout(logits, K, "logits")
    a = pspec_sample_args()
    a.B, a.K, a.V, a.ld, a.dtype = Bn, K, V, ld, dt
    a.logits = logits.data_ptr()
    a.uniforms = _ptr(uniforms, torch.float32, "uniforms")
    a.draft_tokens = _ptr(draft_tokens, torch.int32, "draft_tokens")
    a.q_at_draft = _ptr(q_at_draft, torch.float32, "q_at_draft")
    a.err = _ptr(err, torch.int32, "err")
    st = LIB.pspec_sample_drafts(ctypes.byref(a), _ptr(workspace, torch.uint8, "workspace"),
                                 workspace.numel(), _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_sample_drafts", st)


def _build_args(*, K, block_size, mask_id, pad_id, T_cap, qsl_in, verify_tokens, verify_pos,
                accepted_len, bonus, block_table, verify_hidden, h_shared, draft_tokens,
                draft_pos, slot_mapping, row_kind, hidden_src, qsl_out, seq_lens_out,
                sample_idx, draft_hidden, err, k_len=None):
    a = pspec_build_args()
    a.B = int(qsl_in.numel()) - 1
    a.K = int(K)
    if verify_hidden is not None:
        if verify_hidden.dtype not in _DT:
            raise TypeError("hidden states must be float32 or bfloat16")
        a.H = int(verify_hidden.shape[1])
        a.hidden_dtype = _DT[verify_hidden.dtype]
        for t, nm in ((h_shared, "h_shared"), (draft_hidden, "draft_hidden")):
            if t is not None and t.dtype != verify_hidden.dtype:
                raise TypeError(f"{nm} must have the dtype of verify_hidden")
    else:
        a.H, a.hidden_dtype = 8, PSPEC_BF16
    a.block_size = int(block_size)
    a.max_blocks = int(block_table.shape[1]) if block_table.dim() == 2 else 1
    a.mask_id, a.pad_id = int(mask_id), int(pad_id)
    a.T_in = int(verify_tokens.numel())
    a.T_cap = int(T_cap)
    a.qsl_in = _ptr(qsl_in, torch.int32, "qsl_in")
    a.verify_tokens = _ptr(verify_tokens, torch.int32, "verify_tokens")
    a.verify_pos = _ptr(verify_pos, torch.int32, "verify_pos")
    a.accepted_len = _ptr(accepted_len, torch.int32, "accepted_len")
    a.bonus = _ptr(bonus, torch.int32, "bonus")
    a.block_table = _ptr(block_table, torch.int32, "block_table")
    a.verify_hidden = _ptr(verify_hidden, None, "verify_hidden")
    a.h_shared = _ptr(h_shared, None, "h_shared")
    a.draft_tokens = _ptr(draft_tokens, torch.int32, "draft_tokens")
    a.draft_pos = _ptr(draft_pos, torch.int32, "draft_pos")
    a.slot_mapping = _ptr(slot_mapping, torch.int64, "slot_mapping")
    a.row_kind = _ptr(row_kind, torch.uint8, "row_kind")
    a.hidden_src = _ptr(hidden_src, torch.int32, "hidden_src")
    a.qsl_out = _ptr(qsl_out, torch.int32, "qsl_out")
    a.seq_lens_out = _ptr(seq_lens_out, torch.int32, "seq_lens_out")
    a.sample_idx = _ptr(sample_idx, torch.int32, "sample_idx")
    a.draft_hidden = _ptr(draft_hidden, None, "draft_hidden")
    a.err = _ptr(err, torch.int32, "err")
    a.k_len = _ptr(k_len, torch.int32, "k_len")
    return a


def pspec_build_draft_batch(*, stream=None, **build) -> None:
    """Keyword arguments as the fields of pspec_build_args (tensors for the arrays)."""
    a = _build_args(**build)
    st = LIB.pspec_build_draft_batch(ctypes.byref(a), _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_build_draft_batch", st)


def pspec_step_greedy(*, target_logits, draft_tokens, out_tokens, accepted_len, bonus, err,
                      workspace, build: dict, k_len=None, options=None, stream=None) -> None:
    """Greedy verify followed by the draft-batch build (`build`: the keyword arguments of
    pspec_build_draft_batch, with accepted_len / bonus None or this call's outputs)."""
    K = int(target_logits.shape[1]) - 1
    v = _verify_args(target_logits, None, draft_tokens, None, out_tokens, accepted_len, bonus,
                     err, None, None, None, None, None, K, k_len, options)
    b = _build_args(**build)
    st = LIB.pspec_step_greedy(ctypes.byref(v), ctypes.byref(b),
                               _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                               _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_step_greedy", st)


def pspec_step_rejection(*, target_logits, draft_logits, draft_tokens, uniforms, out_tokens,
                         accepted_len, bonus, err, workspace, build: dict, residual_mass=None,
                         k_len=None, options=None, stream=None) -> None:
    """Rejection-rule verify followed by the draft-batch build (see pspec_step_greedy)."""
    K = int(target_logits.shape[1]) - 1
    v = _verify_args(target_logits, draft_logits, draft_tokens, uniforms, out_tokens,
                     accepted_len, bonus, err, None, None, None, None, residual_mass, K, k_len,
                     options)
    b = _build_args(**build)
    st = LIB.pspec_step_rejection(ctypes.byref(v), ctypes.byref(b),
                                  _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                  _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_step_rejection", st)


_NOALLOC_SIGNATURE_SET = False


def pspec_verify_greedy_noalloc(*, target_logits, draft_tokens, out_tokens, accepted_len, bonus,
                                err, target_lse=None, stream=None) -> None:
    """Greedy verify with the library's own fixed scratch: for callers that cannot hand the
    library a workspace (their device memory is all reserved up front, or they have no
    device allocator).  Same arguments and outputs as pspec_verify_greedy minus the
    workspace; raises PspecError (PSPEC_ERR_UNSUPPORTED) when the call needs more than the
    fixed scratch."""
    global _NOALLOC_SIGNATURE_SET
    if not _NOALLOC_SIGNATURE_SET:
        LIB.pspec_verify_greedy_noalloc.argtypes = [ctypes.POINTER(pspec_verify_args), _P]
        LIB.pspec_verify_greedy_noalloc.restype = _I
        _NOALLOC_SIGNATURE_SET = True
    K = int(target_logits.shape[1]) - 1
    a = _verify_args(target_logits, None, draft_tokens, None, out_tokens, accepted_len, bonus,
                     err, target_lse, None, None, None, None, K)
    st = LIB.pspec_verify_greedy_noalloc(ctypes.byref(a), _stream(stream))
    if st != PSPEC_OK:
        raise PspecError("pspec_verify_greedy_noalloc", st)


class PreparedStep:
    """A pspec_step_greedy / pspec_step_rejection call whose argument structs were filled
    once, for a decode loop that reuses the same buffers every step: calling it only issues
    the C entry point with the saved structs on the given stream (a torch.cuda.Stream, a raw
    cudaStream_t handle, or None for torch's current stream).  The tensors the structs point
    at are kept alive by this object and must keep their storage."""

    def __init__(self, rejection: bool, v, b, workspace, keep):
        self._name = "pspec_step_rejection" if rejection else "pspec_step_greedy"
        self._fn = getattr(LIB, self._name)
        self._v, self._b, self._keep = v, b, keep
        self._vp, self._bp = ctypes.byref(v), ctypes.byref(b)
        self._ws = _ptr(workspace, torch.uint8, "workspace")
        self._wsn = workspace.numel()

    def __call__(self, stream=None) -> None:
        st = self._fn(self._vp, self._bp, self._ws, self._wsn, _stream(stream))
        if st != PSPEC_OK:
            raise PspecError(self._name, st)


def prepare_step(*, target_logits, draft_tokens, out_tokens, accepted_len, bonus, err,
                 workspace, build: dict, draft_logits=None, uniforms=None, residual_mass=None,
                 k_len=None, options=None) -> PreparedStep:
    """The argument structs of a step call (the rejection rule when `uniforms` is given),
    filled once; see PreparedStep."""
    K = int(target_logits.shape[1]) - 1
    rej = uniforms is not None
    v = _verify_args(target_logits, draft_logits if rej else None, draft_tokens, uniforms,
                     out_tokens, accepted_len, bonus, err, None, None, None, None,
                     residual_mass if rej else None, K, k_len, options)
    b = _build_args(**build)
    keep = [target_logits, draft_logits, draft_tokens, uniforms, out_tokens, accepted_len, bonus,
            err, workspace, residual_mass, k_len, dict(build)]
    return PreparedStep(rej, v, b, workspace, keep)
