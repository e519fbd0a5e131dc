"""CPU oracle for the speculative-decoding step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg
may import this package.  The product path (the CUDA library and its binding) never does,
and the oracle imports nothing from it: the two share no code.

The arithmetic lives in ``pspec_oracle.c`` (plain C, double precision, one loop per
definition; its header comment lists the passages it follows and the readings taken where
the pages are silent).  This module compiles it with gcc on first use and marshals numpy
arrays to it.  Verify calls can be split over host threads by sequence: sequences are
independent and ctypes releases the GIL during the foreign call, so each thread runs the
same per-sequence loop on its own slice.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pspec_oracle.c")
_HDR = os.path.join(_HERE, "pspec_oracle.h")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

F32, BF16 = 0, 1
ROW_CTX, ROW_NTP, ROW_MASK, ROW_REJ, ROW_PAD = 0, 1, 2, 3, 4
ERR_TOKEN, ERR_ACCEPT, ERR_BLOCK, ERR_LAYOUT = 0x1, 0x2, 0x4, 0x8
TIE_EPS = 1e-6

_lock = threading.Lock()
_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` with gcc (plain C99)."""
    newest = max(os.path.getmtime(src), os.path.getmtime(_HDR))
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-Wall", "-fPIC", "-shared",
                           "-I", _HERE, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_longlong, ctypes.c_double
    lib.oracle_verify_greedy.argtypes = [i32, i32, i32, i64, i32, P, P, P, P, P, P, P, P]
    lib.oracle_verify_greedy.restype = i32
    lib.oracle_verify_rejection.argtypes = [i32, i32, i32, i64, i32] + [P] * 14 + [f64, P]
    lib.oracle_verify_rejection.restype = i32
    lib.oracle_build_draft_batch.argtypes = [i32] * 10 + [P] * 18
    lib.oracle_build_draft_batch.restype = i32
    lib.oracle_sample_rows.argtypes = [i32, i32, i64, i32, P, P, P, P, P, f64]
    lib.oracle_sample_rows.restype = i32
    return lib


def default() -> "OracleLib":
    """The oracle compiled from ``pspec_oracle.c`` (built on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = OracleLib(build())
    return _default


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _logits_dtype(x: np.ndarray) -> int:
    """fp32 arrays are fp32; bf16 arrives as its raw 16-bit patterns (uint16/int16)."""
    if x.dtype == np.float32:
        return F32
    if x.dtype in (np.uint16, np.int16):
        return BF16
    raise TypeError(f"logits must be float32 or raw bf16 bits (uint16), got {x.dtype}")


def _split(B: int, threads: int):
    threads = max(1, min(threads, B))
    step = (B + threads - 1) // threads
    return [(b, min(B, b + step)) for b in range(0, B, step)]


class OracleLib:
    """The three oracle entry points bound to one compiled copy of the C source."""

    def __init__(self, path: str):
        self.path = path
        self.lib = _bind(path)

    def verify_greedy(self, target: np.ndarray, draft_tokens: np.ndarray,
                      want_lse: bool = False, threads: int = 1, k_len=None) -> dict:
        """Greedy verify of target logits [B, K+1, V] against drafts [B, K] (int32);
        k_len [B] (optional): each sequence's own draft count (R14)."""
        lib = self.lib
        target = np.ascontiguousarray(target)
        draft_tokens = np.ascontiguousarray(draft_tokens, dtype=np.int32)
        k_len = None if k_len is None else np.ascontiguousarray(k_len, dtype=np.int32)
        B, K1, V = target.shape
        K = K1 - 1
        dt = _logits_dtype(target)
        out = {
            "out_tokens": np.empty((B, K + 1), np.int32),
            "accepted_len": np.empty(B, np.int32),
            "bonus": np.empty(B, np.int32),
            "target_lse": np.empty((B, K + 1), np.float64) if want_lse else None,
        }
        errs = []

        def run(b0, b1):
            e = ctypes.c_int(0)
            rc = lib.oracle_verify_greedy(
                b1 - b0, K, V, V, dt, _ptr(target[b0:b1]), _ptr(draft_tokens[b0:b1]),
                _ptr(k_len[b0:b1]) if k_len is not None else None,
                _ptr(out["out_tokens"][b0:b1]), _ptr(out["accepted_len"][b0:b1]),
                _ptr(out["bonus"][b0:b1]),
                _ptr(out["target_lse"][b0:b1]) if want_lse else None, ctypes.byref(e))
            if rc != 0:
                raise ValueError("oracle_verify_greedy rejected its arguments")
            errs.append(e.value)

        _run_parallel(run, B, threads)
        out["err"] = int(np.bitwise_or.reduce(np.array(errs or [0])))
        return out

    def verify_rejection(self, target: np.ndarray, draft: np.ndarray, draft_tokens: np.ndarray,
                         uniforms: np.ndarray, tie_eps: float = TIE_EPS,
                         threads: int = 1, k_len=None) -> dict:
        """Rejection-rule verify: target [B, K+1, V], draft [B, K, V], drafts [B, K],
        uniforms [B, K+1] (float32), k_len [B] (optional, R14).  Returns tokens, counts,
        flags and double diagnostics."""
        lib = self.lib
        target = np.ascontiguousarray(target)
        draft = np.ascontiguousarray(draft)
        draft_tokens = np.ascontiguousarray(draft_tokens, dtype=np.int32)
        uniforms = np.ascontiguousarray(uniforms, dtype=np.float32)
        k_len = None if k_len is None else np.ascontiguousarray(k_len, dtype=np.int32)
        B, K1, V = target.shape
        K = K1 - 1
        assert draft.shape == (B, K, V) and draft.dtype == target.dtype
        assert uniforms.shape == (B, K + 1) and draft_tokens.shape == (B, K)
        dt = _logits_dtype(target)
        out = {
            "out_tokens": np.empty((B, K + 1), np.int32),
            "accepted_len": np.empty(B, np.int32),
            "bonus": np.empty(B, np.int32),
            "p_at_draft": np.empty((B, K), np.float64),
            "q_at_draft": np.empty((B, K), np.float64),
            "target_lse": np.empty((B, K + 1), np.float64),
            "draft_lse": np.empty((B, K), np.float64),
            "residual_mass": np.empty(B, np.float64),
            "flags": np.empty(B, np.int32),
        }
        errs = []

        def run(b0, b1):
            e = ctypes.c_int(0)
            o = {k: v[b0:b1] for k, v in out.items()}
            rc = lib.oracle_verify_rejection(
                b1 - b0, K, V, V, dt, _ptr(target[b0:b1]), _ptr(draft[b0:b1]),
                _ptr(draft_tokens[b0:b1]), _ptr(uniforms[b0:b1]),
                _ptr(k_len[b0:b1]) if k_len is not None else None,
                _ptr(o["out_tokens"]), _ptr(o["accepted_len"]), _ptr(o["bonus"]),
                _ptr(o["p_at_draft"]), _ptr(o["q_at_draft"]), _ptr(o["target_lse"]),
                _ptr(o["draft_lse"]), _ptr(o["residual_mass"]), _ptr(o["flags"]),
                ctypes.c_double(tie_eps), ctypes.byref(e))
            if rc != 0:
                raise ValueError("oracle_verify_rejection rejected its arguments")
            errs.append(e.value)

        _run_parallel(run, B, threads)
        out["err"] = int(np.bitwise_or.reduce(np.array(errs or [0])))
        return out

    def sample_rows(self, logits: np.ndarray, uniforms=None, tie_eps: float = TIE_EPS,
                    threads: int = 1) -> dict:
        """Sample one token per row of logits [..., V] (float32 or raw bf16 bits) by inverse
        CDF at uniforms [...] (float32), or take the argmax when uniforms is None."""
        lib = self.lib
        logits = np.ascontiguousarray(logits)
        shape = logits.shape[:-1]
        V = logits.shape[-1]
        flat = logits.reshape(-1, V)
        N = flat.shape[0]
        u = None if uniforms is None else np.ascontiguousarray(uniforms, np.float32).reshape(-1)
        assert u is None or u.shape == (N,)
        dt = _logits_dtype(flat)
        out = {"tokens": np.empty(N, np.int32), "probs": np.empty(N, np.float64),
               "flags": np.empty(N, np.int32)}

        def run(b0, b1):
            rc = lib.oracle_sample_rows(
                b1 - b0, V, V, dt, _ptr(flat[b0:b1]), _ptr(u[b0:b1]) if u is not None else None,
                _ptr(out["tokens"][b0:b1]), _ptr(out["probs"][b0:b1]), _ptr(out["flags"][b0:b1]),
                ctypes.c_double(tie_eps))
            if rc != 0:
                raise ValueError("oracle_sample_rows rejected its arguments")

        _run_parallel(run, N, threads)
        return {k: v.reshape(shape) for k, v in out.items()}

    def build_draft_batch(self, *, K: int, block_size: int, mask_id: int, pad_id: int,
                          T_cap: int, qsl_in, verify_tokens, verify_pos, accepted_len, bonus,
                          block_table, verify_hidden=None, h_shared=None,
                          draft_hidden_init=None, k_len=None) -> dict:
        """P-EAGLE draft-batch construction (single-threaded: offsets are a running sum).

        ``verify_hidden`` [T_in, H] and ``h_shared`` [H] may be any dtype of equal element
        size; they are copied as bytes.  ``draft_hidden_init`` gives the initial contents of
        the output hidden buffer (rows the method does not write keep them)."""
        lib = self.lib
        qsl_in = np.ascontiguousarray(qsl_in, dtype=np.int32)
        verify_tokens = np.ascontiguousarray(verify_tokens, dtype=np.int32)
        verify_pos = np.ascontiguousarray(verify_pos, dtype=np.int32)
        accepted_len = np.ascontiguousarray(accepted_len, dtype=np.int32)
        bonus = np.ascontiguousarray(bonus, dtype=np.int32)
        block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        k_len = None if k_len is None else np.ascontiguousarray(k_len, dtype=np.int32)
        B = qsl_in.shape[0] - 1
        T_in = verify_tokens.shape[0]
        max_blocks = block_table.shape[1] if block_table.ndim == 2 else 1
        out = {
            "draft_tokens": np.empty(T_cap, np.int32),
            "draft_pos": np.empty(T_cap, np.int32),
            "slot_mapping": np.empty(T_cap, np.int64),
            "row_kind": np.empty(T_cap, np.uint8),
            "hidden_src": np.empty(T_cap, np.int32),
            "qsl_out": np.empty(B + 1, np.int32),
            "seq_lens_out": np.empty(B, np.int32),
            "sample_idx": np.empty((B, K), np.int32),
        }
        H, eb, dh = 1, 1, None
        if verify_hidden is not None:
            verify_hidden = np.ascontiguousarray(verify_hidden)
            h_shared = np.ascontiguousarray(h_shared)
            H = verify_hidden.shape[1]
            eb = verify_hidden.dtype.itemsize
            assert h_shared.shape == (H,) and h_shared.dtype.itemsize == eb
            if draft_hidden_init is not None:
                dh = np.array(draft_hidden_init, dtype=verify_hidden.dtype, copy=True)
                assert dh.shape == (T_cap, H)
            else:
                dh = np.zeros((T_cap, H), verify_hidden.dtype)
        e = ctypes.c_int(0)
        rc = lib.oracle_build_draft_batch(
            B, K, H, eb, block_size, max_blocks, mask_id, pad_id, T_in, T_cap,
            _ptr(qsl_in), _ptr(verify_tokens), _ptr(verify_pos), _ptr(accepted_len), _ptr(bonus),
            _ptr(k_len) if k_len is not None else None, _ptr(block_table), _ptr(verify_hidden), _ptr(h_shared),
            _ptr(out["draft_tokens"]), _ptr(out["draft_pos"]), _ptr(out["slot_mapping"]),
            _ptr(out["row_kind"]), _ptr(out["hidden_src"]), _ptr(out["qsl_out"]),
            _ptr(out["seq_lens_out"]), _ptr(out["sample_idx"]), _ptr(dh), ctypes.byref(e))
        if rc != 0:
            raise ValueError("oracle_build_draft_batch rejected its arguments")
        out["draft_hidden"] = dh
        out["err"] = e.value
        return out


def _run_parallel(fn, B: int, threads: int):
    if B == 0:
        return
    parts = _split(B, threads)
    if len(parts) == 1:
        fn(*parts[0])
        return
    with ThreadPoolExecutor(max_workers=len(parts)) as ex:
        for f in [ex.submit(fn, b0, b1) for b0, b1 in parts]:
            f.result()


def verify_greedy(*args, **kw) -> dict:
    """Greedy verify with the default oracle (see ``OracleLib.verify_greedy``)."""
    return default().verify_greedy(*args, **kw)


def verify_rejection(*args, **kw) -> dict:
    """Rejection-rule verify with the default oracle (see ``OracleLib.verify_rejection``)."""
    return default().verify_rejection(*args, **kw)


def sample_rows(*args, **kw) -> dict:
    """Draft sampling with the default oracle (see ``OracleLib.sample_rows``)."""
    return default().sample_rows(*args, **kw)


def build_draft_batch(**kw) -> dict:
    """Draft-batch construction with the default oracle (see ``OracleLib.build_draft_batch``)."""
    return default().build_draft_batch(**kw)
