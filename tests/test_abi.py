"""The C ABI without a GPU: the library loads, exports every symbol include/pspec.h
declares, and its host-side validation rejects malformed calls before any launch.

Every call made here fails a host check (or is a B = 0 no-op), so no kernel is ever
launched: the pointers are never dereferenced."""
import ctypes
import os
import re
import subprocess

import pytest

import speculative_decoding_step_pspec_b200 as ps
from speculative_decoding_step_pspec_b200 import _binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pspec.h")

FAKE = 0x10000          # 16- and 256-byte aligned, never dereferenced
FAKE_ODD = 0x10001      # not even 2-byte aligned


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"PSPEC_API\s+[\w\s\*]+?\**\s*(pspec_\w+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = declared()
    assert len(names) >= 8, names
    out = subprocess.run(["nm", "-D", "--defined-only", b.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (pspec_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(b.EXPORTED) == set(names)
    for n in names:
        assert getattr(b.LIB, n) is not None


def test_status_strings_and_launch_counts():
    assert ps.pspec_status_string(0) == "PSPEC_OK"
    assert ps.pspec_status_string(4) == "PSPEC_ERR_WORKSPACE"
    assert ps.pspec_status_string(99) == "PSPEC_ERR_UNKNOWN"
    assert ps.pspec_last_launches() == 0          # no successful call on this thread yet
    for path in (1, 2, 0, 7):
        ps.pspec_set_verify_path(path)                # setter only; 7 falls back to automatic
    ps.pspec_set_verify_path(0)


def test_tuning_setters_and_queries():
    """Every process-wide tuning setter changes the defaults pspec_get_options reports, takes
    its valid values and falls back to the automatic choice on others (setters only: nothing
    launches); the last-call queries start at zero on a thread that made no call."""
    assert ps.pspec_last_verify_path() == 0 and ps.pspec_last_cluster_size() == 0
    zero = dict(verify_path=0, cluster_size=0, tail_split=0, step_fusion=0, segment_elems=0)
    assert ps.pspec_get_options() == zero
    try:
        for path, want in ((1, 1), (2, 2), (3, 0), (4, 0), (9, 0), (-1, 0)):
            ps.pspec_set_verify_path(path)
            assert ps.pspec_get_options()["verify_path"] == want
        for G, want in ((1, 0), (2, 2), (4, 4), (8, 8), (12, 12), (16, 16), (5, 0), (0, 0)):
            ps.pspec_set_cluster_size(G)
            assert ps.pspec_get_options()["cluster_size"] == want
        for n, want in ((96, 96), (1, 1), (-1, -1), (-7, -1), (0, 0)):
            ps.pspec_set_tail_split(n)
            assert ps.pspec_get_options()["tail_split"] == want
        for mode, want in ((1, 1), (2, 2), (3, 0), (4, 0), (0, 0)):
            ps.pspec_set_step_fusion(mode)
            assert ps.pspec_get_options()["step_fusion"] == want
        ps.pspec_set_segment_elems(4096)
        assert ps.pspec_get_options()["segment_elems"] == 4096
    finally:
        ps.pspec_set_verify_path(0)
        ps.pspec_set_cluster_size(0)
        ps.pspec_set_tail_split(0)
        ps.pspec_set_step_fusion(0)
        ps.pspec_set_segment_elems(0)
    assert ps.pspec_get_options() == zero


def test_options_struct_layout_and_workspace():
    """The options struct the binding builds has the header's layout (four ints, then a
    64-bit count at offset 16), the verify argument struct ends with its pointer, and a
    call's own segment length changes the workspace size as the process-wide one does."""
    o = b.pspec_options
    assert [f for f, _ in o._fields_] == ["verify_path", "cluster_size", "tail_split",
                                          "step_fusion", "segment_elems"]
    assert o.segment_elems.offset == 16 and ctypes.sizeof(o) == 24
    assert b.pspec_verify_args._fields_[-1][0] == "options"
    f = b.pspec_verify_workspace_bytes
    base = f(64, 7, 151936, True)
    assert f(64, 7, 151936, True, {}) == base
    small = f(64, 7, 151936, True, {"segment_elems": 1024})
    assert small > base
    ps.pspec_set_segment_elems(1024)
    try:
        assert f(64, 7, 151936, True) == small
        assert f(64, 7, 151936, True, {}) == base     # a call's own options ignore the default
    finally:
        ps.pspec_set_segment_elems(0)
    with pytest.raises(KeyError):
        b.make_options({"no_such_field": 1})


def test_workspace_sizes():
    f = ps.pspec_verify_workspace_bytes
    assert f(0, 7, 1000, True) > 0 or f(0, 7, 1000, True) == 0
    assert f(-1, 7, 1000, True) == 0 and f(4, 0, 1000, True) == 0 and f(4, 32, 10, True) == 0
    assert f(4, 7, 0, False) == 0
    for rej in (False, True):
        prev = 0
        for B in (1, 8, 64, 1024):
            n = f(B, 7, 201088, rej)
            assert n % 256 == 0 and n >= prev
            prev = n
    assert f(1024, 7, 201088, True) > f(1024, 7, 201088, False)
    # the sweep's (m, s) partials of all 15 rows per sequence, SeqInfo and the draw's tile
    # sums, plus the two tickets per sequence at the end
    assert f(1024, 7, 201088, True) >= 1024 * 15 * 8 + 1024 * 48 + 1024 * 786 * 8 + 1024 * 8


def _vargs(**kw):
    a = b.pspec_verify_args()
    a.B, a.K, a.V, a.ld, a.dtype = 4, 3, 1000, 1000, b.PSPEC_BF16
    for f in ("target_logits", "draft_logits", "draft_tokens", "uniforms", "out_tokens",
              "accepted_len", "bonus", "err"):
        setattr(a, f, FAKE)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


WS_SMALL = 256


@pytest.mark.parametrize("fn", ["pspec_verify_greedy", "pspec_verify_rejection"])
@pytest.mark.parametrize("case,field,value,status", [
    ("null_target", "target_logits", None, b.PSPEC_ERR_INVALID_ARG),
    ("null_err", "err", None, b.PSPEC_ERR_INVALID_ARG),
    ("null_out", "out_tokens", None, b.PSPEC_ERR_INVALID_ARG),
    ("neg_B", "B", -1, b.PSPEC_ERR_INVALID_ARG),
    ("K0", "K", 0, b.PSPEC_ERR_INVALID_ARG),
    ("K32", "K", 32, b.PSPEC_ERR_UNSUPPORTED),
    ("V0", "V", 0, b.PSPEC_ERR_INVALID_ARG),
    ("ld_lt_V", "ld", 999, b.PSPEC_ERR_INVALID_ARG),
    ("base_unaligned", "target_logits", FAKE_ODD, b.PSPEC_ERR_INVALID_ARG),
    ("bad_dtype", "dtype", 7, b.PSPEC_ERR_INVALID_ARG),
])
def test_verify_host_checks(fn, case, field, value, status):
    a = _vargs(**{field: value})
    st = getattr(b.LIB, fn)(ctypes.byref(a), FAKE, 1 << 40, None)
    assert st == status, (case, b.pspec_status_string(st))


@pytest.mark.parametrize("fn", ["pspec_verify_greedy", "pspec_verify_rejection"])
def test_verify_workspace_checks(fn):
    a = _vargs()
    need = ps.pspec_verify_workspace_bytes(4, 3, 1000, fn.endswith("rejection"))
    L = getattr(b.LIB, fn)
    assert L(ctypes.byref(a), None, need, None) == b.PSPEC_ERR_WORKSPACE
    assert L(ctypes.byref(a), FAKE + 16, need, None) == b.PSPEC_ERR_WORKSPACE
    assert L(ctypes.byref(a), FAKE, need - 1, None) == b.PSPEC_ERR_WORKSPACE
    assert L(None, FAKE, need, None) == b.PSPEC_ERR_INVALID_ARG


def test_rejection_needs_draft_and_uniforms():
    for f in ("draft_logits", "uniforms"):
        a = _vargs(**{f: None})
        assert b.LIB.pspec_verify_rejection(ctypes.byref(a), FAKE, 1 << 40, None) == \
            b.PSPEC_ERR_INVALID_ARG
    a = _vargs(draft_logits=FAKE_ODD)
    assert b.LIB.pspec_verify_rejection(ctypes.byref(a), FAKE, 1 << 40, None) == \
        b.PSPEC_ERR_INVALID_ARG


@pytest.mark.parametrize("fn", ["pspec_verify_greedy", "pspec_verify_rejection"])
def test_empty_batch_is_a_noop(fn):
    a = _vargs(B=0, target_logits=None, out_tokens=None)
    assert getattr(b.LIB, fn)(ctypes.byref(a), None, 0, None) == b.PSPEC_OK


def _bargs(**kw):
    a = b.pspec_build_args()
    a.B, a.K, a.H, a.hidden_dtype, a.block_size, a.max_blocks = 4, 3, 64, b.PSPEC_BF16, 16, 8
    a.mask_id, a.pad_id, a.T_in, a.T_cap = 1, 2, 16, 24
    for f, _ in b.pspec_build_args._fields_[10:]:
        setattr(a, f, FAKE)
    a.k_len = None                       # optional: per-sequence draft counts
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("case,kw,status", [
    ("null_args", None, b.PSPEC_ERR_INVALID_ARG),
    ("cap_too_small", dict(T_cap=23), b.PSPEC_ERR_INVALID_ARG),
    ("K0", dict(K=0), b.PSPEC_ERR_INVALID_ARG),
    ("K32", dict(K=32, T_cap=1000), b.PSPEC_ERR_UNSUPPORTED),
    ("H0", dict(H=0), b.PSPEC_ERR_INVALID_ARG),
    ("bs0", dict(block_size=0), b.PSPEC_ERR_INVALID_ARG),
    ("mb0", dict(max_blocks=0), b.PSPEC_ERR_INVALID_ARG),
    ("neg_T_in", dict(T_in=-1), b.PSPEC_ERR_INVALID_ARG),
    ("row_not_16B", dict(H=60), b.PSPEC_ERR_INVALID_ARG),
    ("hidden_unaligned", dict(draft_hidden=FAKE_ODD), b.PSPEC_ERR_INVALID_ARG),
    ("h_shared_null", dict(h_shared=None), b.PSPEC_ERR_INVALID_ARG),
    ("null_qsl", dict(qsl_in=None), b.PSPEC_ERR_INVALID_ARG),
    ("null_slot", dict(slot_mapping=None), b.PSPEC_ERR_INVALID_ARG),
    ("null_err", dict(err=None), b.PSPEC_ERR_INVALID_ARG),
    ("null_table", dict(block_table=None), b.PSPEC_ERR_INVALID_ARG),
    ("bad_dtype", dict(hidden_dtype=5), b.PSPEC_ERR_INVALID_ARG),
])
def test_build_host_checks(case, kw, status):
    if kw is None:
        st = b.LIB.pspec_build_draft_batch(None, None)
    else:
        a = _bargs(**kw)
        st = b.LIB.pspec_build_draft_batch(ctypes.byref(a), None)
    assert st == status, (case, b.pspec_status_string(st))


def test_segment_override_changes_workspace():
    base = ps.pspec_verify_workspace_bytes(2, 3, 100000, True)
    ps.pspec_set_segment_elems(1024)
    try:
        assert ps.pspec_verify_workspace_bytes(2, 3, 100000, True) > base
    finally:
        ps.pspec_set_segment_elems(0)
    assert ps.pspec_verify_workspace_bytes(2, 3, 100000, True) == base


@pytest.mark.parametrize("case,vkw,bkw,ws,status", [
    ("batch_mismatch", {}, {"B": 5}, (FAKE, 1 << 30), b.PSPEC_ERR_INVALID_ARG),
    ("k_mismatch", {}, {"K": 2}, (FAKE, 1 << 30), b.PSPEC_ERR_INVALID_ARG),
    ("foreign_accepted_len", {}, {"accepted_len": FAKE + 256}, (FAKE, 1 << 30),
     b.PSPEC_ERR_INVALID_ARG),
    ("foreign_bonus", {}, {"bonus": FAKE + 256}, (FAKE, 1 << 30), b.PSPEC_ERR_INVALID_ARG),
    ("foreign_k_len", {}, {"k_len": FAKE + 512}, (FAKE, 1 << 30), b.PSPEC_ERR_INVALID_ARG),
    ("bad_build", {}, {"T_cap": 3}, (FAKE, 1 << 30), b.PSPEC_ERR_INVALID_ARG),
    ("bad_verify", {"ld": 10}, {}, (FAKE, 1 << 30), b.PSPEC_ERR_INVALID_ARG),
    ("short_workspace", {}, {}, (FAKE, 256), b.PSPEC_ERR_WORKSPACE),
    ("no_workspace", {}, {}, (None, 0), b.PSPEC_ERR_WORKSPACE),
])
@pytest.mark.parametrize("fn", ["pspec_step_greedy", "pspec_step_rejection"])
def test_step_host_checks(fn, case, vkw, bkw, ws, status):
    """The step calls check both halves before any launch: a build whose accepted counts or
    bonus tokens are not the verify's outputs, shapes that disagree, or either half's own
    argument errors return a status and launch nothing."""
    v = _vargs(**vkw)
    bb = _bargs(**bkw)
    ps.pspec_set_verify_path(1)          # full sweep: its workspace check runs before a launch
    try:
        st = getattr(b.LIB, fn)(ctypes.byref(v), ctypes.byref(bb), ws[0], ws[1], None)
    finally:
        ps.pspec_set_verify_path(0)
    assert st == status, (case, b.pspec_status_string(st))
    assert getattr(b.LIB, fn)(None, ctypes.byref(bb), FAKE, 1 << 30, None) == b.PSPEC_ERR_INVALID_ARG
    assert getattr(b.LIB, fn)(ctypes.byref(v), None, FAKE, 1 << 30, None) == b.PSPEC_ERR_INVALID_ARG
