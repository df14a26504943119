"""The C ABI loads without a GPU, exports what include/asffn.h declares, and
rejects bad arguments on the host before any launch."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O
from activation_sparse_ffn_predict_b200 import _lib as L
from activation_sparse_ffn_predict_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "asffn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ASF_API\s+[\w\s\*]*?\b(asf_\w+)\s*\(", text)))


def test_header_declares_the_expected_calls():
    names = declared_functions()
    for fn in ["asf_predict", "asf_sparse_ffn", "asf_dense_ffn", "asf_activation_counts",
               "asf_hot_permutation", "asf_permute_rows", "asf_workspace_bytes",
               "asf_workspace_init", "asf_read_error", "asf_status_string", "asf_version"]:
        assert fn in names
    assert sorted(L.PROTOTYPES) == names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for fn in declared_functions():
        assert fn in exported, fn
        assert hasattr(lib, fn)
    # nothing else leaks out of the C ABI
    assert {e for e in exported if e.startswith("asf_")} == set(declared_functions())


def test_version_and_status_strings(lib):
    assert lib.asf_version() == 106
    for code in range(8):
        assert lib.asf_status_string(code).decode() not in ("", "unknown status")
    assert lib.asf_status_string(99).decode() == "unknown status"


def test_struct_layout_matches_header():
    # int32 d, r, n; enum; then four pointers (8-byte aligned)
    assert ctypes.sizeof(L.asf_predictor) == 16 + 4 * 8
    assert L.asf_predictor.W1.offset == 16
    assert ctypes.sizeof(L.asf_ffn) == 16 + 4 * 8 + 8 + 2 * 8 + 2 * 8   # + hot_rows, row_stride, l2_next[2], l2_next_bytes[2]
    assert L.asf_ffn.Wg.offset == 16


@pytest.mark.parametrize("n", [0, 1, 7, 1376, 20000])
def test_hot_permutation_matches_oracle(lib, n):
    rng = np.random.default_rng(n)
    counts = rng.integers(0, 50, size=n).astype(np.int64)
    c = np.ascontiguousarray(counts)
    out = np.empty(n, dtype=np.int32)
    st = lib.asf_hot_permutation(c.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
                                 out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    assert st == L.ASF_OK
    np.testing.assert_array_equal(out, O.hot_permutation(counts))


# ----------------------------------------------------------- host checks --
FAKE = 1 << 20          # aligned, never dereferenced: every case fails validation first


def _pred(d=64, r=32, n=100, dt=L.ASF_F16, w1=FAKE, b1=FAKE, w2=FAKE, b2=FAKE):
    return L.asf_predictor(d, r, n, dt, w1, b1, w2, b2)


def _ffn(d=64, n=100, dt=L.ASF_F16, act=L.ASF_ACT_REGLU, wg=FAKE, wu=FAKE, wdt=FAKE, bias=FAKE):
    return L.asf_ffn(d, n, dt, act, wg, wu, wdt, bias)


def test_workspace_bytes(lib):
    p = _pred()
    f = _ffn()
    wp = lib.asf_workspace_bytes(ctypes.byref(p), None, 1)
    wf = lib.asf_workspace_bytes(None, ctypes.byref(f), 4)
    both = lib.asf_workspace_bytes(ctypes.byref(p), ctypes.byref(f), 4)
    assert wp >= 4096 + 100 // 32 * 4 + 32 * 4
    assert wf >= 4096 + 100 * 4 * 4
    # with both descriptors: the predictor's and the FFN's scratch side by side
    # (the combined call uses both at once); 4096 = the header
    assert both == lib.asf_workspace_bytes(ctypes.byref(p), None, 4) + wf - 4096
    assert lib.asf_workspace_bytes(None, None, 1) == 0
    assert lib.asf_workspace_bytes(ctypes.byref(p), None, 0) == 0
    assert lib.asf_workspace_bytes(ctypes.byref(p), None, L.ASF_MAX_BATCH + 1) == 0
    bad = _pred(d=60)    # not a multiple of 8 for fp16
    assert lib.asf_workspace_bytes(ctypes.byref(bad), None, 1) == 0


def _predict(lib, p, x=FAKE, B=1, tau=0.5, idx=FAKE, cnt=FAKE, ws=FAKE, wsb=0):
    return lib.asf_predict(ctypes.byref(p) if p is not None else None, x, B, tau, idx, cnt, ws, wsb, None)


def test_predict_rejects_bad_arguments(lib):
    p = _pred()
    assert _predict(lib, None) == L.ASF_ERR_INVALID_ARG
    assert _predict(lib, _pred(w1=0)) == L.ASF_ERR_INVALID_ARG
    assert _predict(lib, _pred(d=0)) == L.ASF_ERR_INVALID_ARG
    assert _predict(lib, _pred(d=60)) == L.ASF_ERR_MISALIGNED
    assert _predict(lib, _pred(r=12)) == L.ASF_ERR_MISALIGNED
    assert _predict(lib, _pred(w2=FAKE + 8)) == L.ASF_ERR_MISALIGNED
    assert _predict(lib, _pred(dt=7)) == L.ASF_ERR_UNSUPPORTED
    assert _predict(lib, p, x=0) == L.ASF_ERR_INVALID_ARG
    assert _predict(lib, p, B=0) == L.ASF_ERR_INVALID_ARG
    assert _predict(lib, p, B=33) == L.ASF_ERR_INVALID_ARG
    for tau in [0.0, 1.0, -0.5, 2.0, float("nan")]:
        assert _predict(lib, p, tau=tau) == L.ASF_ERR_INVALID_ARG
    assert _predict(lib, p, x=FAKE + 4) == L.ASF_ERR_MISALIGNED
    assert _predict(lib, p, idx=FAKE + 2) == L.ASF_ERR_MISALIGNED
    assert _predict(lib, p, ws=0) == L.ASF_ERR_WORKSPACE
    assert _predict(lib, p, ws=FAKE + 64, wsb=1 << 30) == L.ASF_ERR_WORKSPACE
    need = lib.asf_workspace_bytes(ctypes.byref(p), None, 1)
    assert _predict(lib, p, wsb=need - 1) == L.ASF_ERR_WORKSPACE


def _sparse(lib, f, x=FAKE, B=1, idx=FAKE, cnt=FAKE, y=FAKE, ws=FAKE, wsb=0):
    return lib.asf_sparse_ffn(ctypes.byref(f) if f is not None else None, x, B, idx, cnt, y, ws, wsb, None)


def test_sparse_ffn_rejects_bad_arguments(lib):
    f = _ffn()
    assert _sparse(lib, None) == L.ASF_ERR_INVALID_ARG
    assert _sparse(lib, _ffn(wg=0)) == L.ASF_ERR_INVALID_ARG           # ReGLU needs a gate
    assert _sparse(lib, _ffn(act=L.ASF_ACT_RELU, wg=0), wsb=0) == L.ASF_ERR_WORKSPACE
    assert _sparse(lib, _ffn(act=9)) == L.ASF_ERR_UNSUPPORTED
    assert _sparse(lib, _ffn(dt=L.ASF_F32, d=66)) == L.ASF_ERR_MISALIGNED
    assert _sparse(lib, _ffn(wdt=FAKE + 4)) == L.ASF_ERR_MISALIGNED
    assert _sparse(lib, _ffn(bias=FAKE + 2)) == L.ASF_ERR_MISALIGNED
    assert _sparse(lib, _ffn(d=1 << 20)) == L.ASF_ERR_UNSUPPORTED      # too wide to stage
    assert _sparse(lib, f, y=0) == L.ASF_ERR_INVALID_ARG
    assert _sparse(lib, f, cnt=0) == L.ASF_ERR_INVALID_ARG
    assert _sparse(lib, f, B=0) == L.ASF_ERR_INVALID_ARG
    assert _sparse(lib, f, y=FAKE + 8) == L.ASF_ERR_MISALIGNED
    need = lib.asf_workspace_bytes(None, ctypes.byref(f), 1)
    assert _sparse(lib, f, wsb=need - 1) == L.ASF_ERR_WORKSPACE
    hinted = _ffn()
    hinted.l2_next[1] = FAKE + 8
    hinted.l2_next_bytes[1] = 4096
    assert _sparse(lib, hinted) == L.ASF_ERR_MISALIGNED                # L2 hint not 16-byte aligned
    hinted.l2_next[1] = FAKE
    hinted.l2_next_bytes[1] = -16
    assert _sparse(lib, hinted) == L.ASF_ERR_INVALID_ARG
    assert lib.asf_dense_ffn(ctypes.byref(f), FAKE, 1, FAKE, FAKE, need - 1, None) == L.ASF_ERR_WORKSPACE
    assert lib.asf_dense_ffn(ctypes.byref(f), FAKE, 0, FAKE, FAKE, need, None) == L.ASF_ERR_INVALID_ARG


def _combined(lib, p, f, x=FAKE, B=1, tau=0.5, idx=FAKE, cnt=FAKE, y=FAKE, ws=FAKE, wsb=None,
              name="asf_predict_sparse_ffn"):
    if wsb is None:
        wsb = lib.asf_workspace_bytes(ctypes.byref(p), ctypes.byref(f), max(1, min(B, L.ASF_MAX_BATCH)))
    return getattr(lib, name)(ctypes.byref(p) if p is not None else None,
                              ctypes.byref(f) if f is not None else None, x, B, tau, idx, cnt, y,
                              ws, wsb, None)


@pytest.mark.parametrize("name", ["asf_predict_sparse_ffn", "asf_predict_sparse_ffn_begin",
                                  "asf_predict_sparse_ffn_end"])
def test_layer_calls_reject_bad_arguments(lib, name):
    """The combined call and its two halves validate the same way."""
    import functools
    _combined_ = functools.partial(_combined, name=name)
    p, f = _pred(), _ffn()
    assert _combined_(lib, None, f, wsb=1 << 30) == L.ASF_ERR_INVALID_ARG
    assert _combined_(lib, p, f, x=0) == L.ASF_ERR_INVALID_ARG
    assert _combined_(lib, p, f, tau=0.0) == L.ASF_ERR_INVALID_ARG
    assert _combined_(lib, p, f, B=33, wsb=1 << 30) == L.ASF_ERR_INVALID_ARG
    assert _combined_(lib, _pred(n=100), _ffn(n=101), wsb=1 << 30) == L.ASF_ERR_INVALID_ARG
    assert _combined_(lib, p, f, y=FAKE + 8) == L.ASF_ERR_MISALIGNED
    need = lib.asf_workspace_bytes(ctypes.byref(p), ctypes.byref(f), 1)
    assert _combined_(lib, p, f, wsb=need - 1) == L.ASF_ERR_WORKSPACE


def test_fault_injection_modes(lib):
    assert lib.asf_set_fault_injection(L.ASF_INJECT_WITHHOLD_FFN_COPIES) == L.ASF_OK
    assert lib.asf_set_fault_injection(L.ASF_INJECT_NONE) == L.ASF_OK
    for bad in (-1, 2, 99):
        assert lib.asf_set_fault_injection(bad) == L.ASF_ERR_INVALID_ARG


def test_combined_call_rejects_bad_arguments(lib):
    p, f = _pred(), _ffn()
    assert _combined(lib, None, f, wsb=1 << 30) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, p, None, wsb=1 << 30) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, _pred(d=64), _ffn(d=72), wsb=1 << 30) == L.ASF_ERR_INVALID_ARG   # d differs
    assert _combined(lib, _pred(n=100), _ffn(n=101), wsb=1 << 30) == L.ASF_ERR_INVALID_ARG  # n differs
    assert _combined(lib, _pred(dt=L.ASF_F32), _ffn(), wsb=1 << 30) == L.ASF_ERR_INVALID_ARG  # dtype differs
    assert _combined(lib, p, f, x=0) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, p, f, y=0) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, p, f, B=0) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, p, f, B=33, wsb=1 << 30) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, p, f, tau=1.0) == L.ASF_ERR_INVALID_ARG
    assert _combined(lib, p, f, y=FAKE + 8) == L.ASF_ERR_MISALIGNED
    assert _combined(lib, p, f, idx=FAKE + 2) == L.ASF_ERR_MISALIGNED
    need = lib.asf_workspace_bytes(ctypes.byref(p), ctypes.byref(f), 1)
    assert _combined(lib, p, f, wsb=need - 1) == L.ASF_ERR_WORKSPACE
    # the predictor-only size is not enough for the combined call
    assert _combined(lib, p, f, wsb=lib.asf_workspace_bytes(ctypes.byref(p), None, 1)) == L.ASF_ERR_WORKSPACE


def test_offline_calls_reject_bad_arguments(lib):
    f = _ffn()
    assert lib.asf_activation_counts(ctypes.byref(f), FAKE, -1, FAKE, FAKE, 1 << 20, None) == L.ASF_ERR_INVALID_ARG
    assert lib.asf_activation_counts(ctypes.byref(f), FAKE, 4, FAKE + 4, FAKE, 1 << 20, None) == L.ASF_ERR_MISALIGNED
    assert lib.asf_activation_counts(ctypes.byref(f), FAKE, 4, FAKE, FAKE + 1, 1 << 20, None) == L.ASF_ERR_WORKSPACE
    assert lib.asf_activation_counts(ctypes.byref(f), FAKE, 0, FAKE, FAKE, 1 << 20, None) == L.ASF_OK
    assert lib.asf_permute_rows(FAKE, FAKE, 4, 16, FAKE, None) == L.ASF_ERR_INVALID_ARG      # src == dst
    assert lib.asf_permute_rows(FAKE, FAKE * 2, 4, 0, FAKE, None) == L.ASF_ERR_INVALID_ARG
    assert lib.asf_permute_rows(FAKE, FAKE * 2, 4, 16, FAKE + 1, None) == L.ASF_ERR_MISALIGNED
    assert lib.asf_permute_rows(FAKE, FAKE * 2, 0, 16, FAKE, None) == L.ASF_OK
    assert lib.asf_hot_permutation(None, 3, None) == L.ASF_ERR_INVALID_ARG
    assert lib.asf_workspace_init(FAKE + 16, 8192, None) == L.ASF_ERR_WORKSPACE
    assert lib.asf_workspace_init(FAKE, 100, None) == L.ASF_ERR_WORKSPACE
    assert lib.asf_read_error(None, None, None) == L.ASF_ERR_INVALID_ARG
