"""The C-ABI library on the CPU: it loads without a GPU, exports every entry point that
include/sdm.h declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdm.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(sdm_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from sparse_state_linear_score_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


class Dims(ctypes.Structure):
    """sdm_dims as include/sdm.h lays it out (twelve int32 fields)."""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "T", "d_k", "n_sub", "d_v", "k_half", "W", "R", "x_dtype", "v_dtype",
                 "decay")]


def mid_dims(**kw):
    d = dict(B=2, H=4, T=4096, d_k=128, n_sub=256, d_v=128, k_half=32, W=32, R=32, x_dtype=1,
             v_dtype=1, decay=0)
    d.update(kw)
    return Dims(**d)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("sdm_score_topk", "sdm_forward", "sdm_decode_step", "sdm_prefill",
                 "sdm_state_reset", "sdm_state_materialize", "sdm_forward_workspace_bytes",
                 "sdm_device_error"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    lib.sdm_status_str.restype = ctypes.c_char_p
    for code in range(0, 9):
        s = lib.sdm_status_str(code)
        assert s and s.startswith(b"SDM_")
    assert lib.sdm_abi_version() >= 1


def test_workspace_and_state_sizes(lib):
    lib.sdm_forward_workspace_bytes.restype = ctypes.c_size_t
    d = mid_dims()
    ws = lib.sdm_forward_workspace_bytes(ctypes.byref(d))
    assert ws > 2 * 4 * 4096 * 64 * 8  # at least the per-occurrence plan records
    bad = mid_dims(W=65)
    assert lib.sdm_forward_workspace_bytes(ctypes.byref(bad)) == 0
    m, s, l = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.sdm_state_bytes(ctypes.byref(d), ctypes.byref(m), ctypes.byref(s), ctypes.byref(l)) == 0
    assert m.value == 2 * 4 * 65536 * 128 * 4
    assert s.value == 2 * 4 * 65536 * 8 and l.value == 2 * 4 * 8


def test_touched_decay_workspace(lib):
    """decay = touched adds two fp32 records per occurrence (its in-chunk decay products)."""
    lib.sdm_forward_workspace_bytes.restype = ctypes.c_size_t
    a = lib.sdm_forward_workspace_bytes(ctypes.byref(mid_dims(decay=0)))
    t = lib.sdm_forward_workspace_bytes(ctypes.byref(mid_dims(decay=1)))
    occ = 2 * 4 * 4096 * 64
    assert t - a == 2 * occ * 4  # both sizes are 256-byte multiples here
    assert ctypes.sizeof(Dims) == 48


@pytest.mark.parametrize("field,value,code", [
    ("x_dtype", 7, 3), ("v_dtype", -1, 3), ("B", 0, 2), ("T", -1, 2), ("d_k", 30, 2),
    ("d_k", 512, 2), ("n_sub", 0, 2), ("d_v", 6, 2), ("d_v", 512, 2), ("k_half", 65, 2),
    ("k_half", 300, 2), ("W", 0, 2), ("R", 65, 2), ("decay", 2, 1), ("decay", -1, 1),
])
def test_bad_dims_rejected_on_host(lib, field, value, code):
    d = mid_dims(**{field: value})
    p = ctypes.c_void_p(0x1000)
    assert lib.sdm_score_topk(ctypes.byref(d), p, p, 4, p, p, None) == code


def test_null_and_misaligned_pointers(lib):
    d = mid_dims()
    p = ctypes.c_void_p(0x1000)
    assert lib.sdm_score_topk(None, p, p, 4, p, p, None) == 1
    assert lib.sdm_score_topk(ctypes.byref(d), None, p, 4, p, p, None) == 1
    assert lib.sdm_score_topk(ctypes.byref(d), ctypes.c_void_p(0x1004), p, 4, p, p, None) == 4
    assert lib.sdm_score_topk(ctypes.byref(d), p, p, 0, p, p, None) == 2
    assert lib.sdm_score_topk(ctypes.byref(d), p, p, 65, p, p, None) == 2
    assert lib.sdm_device_error(None, 0, None) == 1
    assert lib.sdm_state_reset(ctypes.byref(d), None, None) == 1
    # decode needs T == 1
    assert lib.sdm_decode_step(ctypes.byref(d), p, p, p, p, p, p, p, None, p, p, p, p, p, None) == 2


def test_forward_rejects_small_workspace(lib):
    class State(ctypes.Structure):
        _fields_ = [("M", ctypes.c_void_p), ("stamp", ctypes.c_void_p), ("Lambda", ctypes.c_void_p),
                    ("M0", ctypes.c_void_p)]
    d = mid_dims()
    p = ctypes.c_void_p(0x1000)
    st = State(0x1000, 0x2000, 0x3000, 0x4000)
    assert lib.sdm_forward(ctypes.byref(d), p, p, p, p, p, p, p, ctypes.byref(st), p, p,
                           ctypes.c_size_t(64), None) == 7
    st_bad = State(0x1000, 0x2000, 0x3003, 0x4000)
    assert lib.sdm_forward(ctypes.byref(d), p, p, p, p, p, p, p, ctypes.byref(st_bad), p, p,
                           ctypes.c_size_t(1 << 40), None) == 4


def test_backward_host_checks(lib):
    """sdm_backward's workspace query covers the write log, the memory gradient and one
    private stamp copy pair per 4-column slice; bad arguments are refused on the host."""
    class State(ctypes.Structure):
        _fields_ = [("M", ctypes.c_void_p), ("stamp", ctypes.c_void_p), ("Lambda", ctypes.c_void_p),
                    ("M0", ctypes.c_void_p)]
    lib.sdm_backward_workspace_bytes.restype = ctypes.c_size_t
    d = mid_dims()
    ws = lib.sdm_backward_workspace_bytes(ctypes.byref(d))
    BH, T, N, W, dv = 2 * 4, 4096, 65536, 32, 128
    log_rows, dM = BH * T * W * dv * 4, BH * N * dv * 4
    stamps = 2 * (dv // 4) * BH * N * 8
    assert ws >= log_rows + dM + stamps
    assert lib.sdm_backward_workspace_bytes(ctypes.byref(mid_dims(W=65))) == 0
    # twice the columns: twice the slices' stamp copies
    ws2 = lib.sdm_backward_workspace_bytes(ctypes.byref(mid_dims(d_v=256)))
    assert ws2 - ws >= log_rows + dM + stamps
    p = ctypes.c_void_p(0x1000)
    st = State(0x1000, 0x2000, 0x3000, 0x4000)
    big = ctypes.c_size_t(1 << 44)

    def call(v=p, dout=p, ws_ptr=p, ws_bytes=big, dims=d):
        return lib.sdm_backward(ctypes.byref(dims), v, p, p, p, p, p, p, ctypes.byref(st), dout,
                                None, p, p, p, p, p, p, ws_ptr, ws_bytes, None)
    assert call(v=None) == 1                                  # SDM_ERR_ARG
    assert call(dout=ctypes.c_void_p(0x1008)) == 4            # SDM_ERR_ALIGN
    assert call(ws_bytes=ctypes.c_size_t(ws - 1)) == 7        # SDM_ERR_WORKSPACE
    assert call(ws_ptr=None) == 7
    assert call(dims=mid_dims(d_k=30)) == 2                   # SDM_ERR_SHAPE
    assert lib.sdm_backward(ctypes.byref(d), p, p, p, p, p, p, p, ctypes.byref(st), p,
                            ctypes.c_void_p(0x1004), p, p, p, p, p, p, p, big, None) == 4


def test_score_path_dispatch(lib):
    """Which scorer each workload's shape takes (host-side query): every bf16 prefill shape of
    the workloads, the long-context one (n = 1024, k = W = R = 64) included, goes to the
    tensor-core kernel; decode steps (T = 1) to the row scorer; fp32 to the CUDA-core paths."""
    import sparse_state_linear_score_b200 as sdm
    import sdm_synth as S
    for wl in (S.MID, S.HEADLINE, S.LONG):
        d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                     wl.x_dtype, wl.v_dtype)
        assert sdm.score_path(d, wl.W) == sdm.SCORE_TC, wl
        assert sdm.score_path(d, wl.R) == sdm.SCORE_TC, wl
        assert sdm.score_path(d.with_T(1), wl.W) == (sdm.SCORE_ROWS if wl.n_sub <= 512
                                                     else sdm.SCORE_WARP)
    wl = S.TINY
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                 wl.x_dtype, wl.v_dtype)
    assert sdm.score_path(d, wl.W) == sdm.SCORE_ROWS  # fp32


def test_decode_path_dispatch(lib):
    """The decode workload's step is one launch (scoring and recurrence steps in one cluster of
    two CTAs); shapes outside the fused kernel's limits (n = 64 or 1024, k = 64, fp32 keys,
    d_k = 64, d_v = 256 whose two steps' arrays exceed the sub-key buffers) take the scoring
    launch and the recurrence launch."""
    import sparse_state_linear_score_b200 as sdm
    import sdm_synth as S
    wl = S.DECODE
    d = sdm.Dims(wl.B, wl.H, 1, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype)
    assert sdm.decode_path(d) == sdm.DECODE_FUSED
    for kw in (dict(n_sub=64), dict(k_half=64, W=64, R=64), dict(x_dtype="f32"), dict(d_k=64),
               dict(n_sub=1024), dict(d_v=256)):
        w2 = wl.scaled(**kw)
        d2 = sdm.Dims(w2.B, w2.H, 1, w2.d_k, w2.n_sub, w2.d_v, w2.k_half, w2.W, w2.R,
                      w2.x_dtype, w2.v_dtype)
        assert sdm.decode_path(d2) == sdm.DECODE_TWO, kw
    for kw in (dict(n_sub=128, d_v=64), dict(n_sub=512, d_v=192, v_dtype="f32"),
               dict(W=16, R=8, k_half=16)):
        w2 = wl.scaled(**kw)
        d2 = sdm.Dims(w2.B, w2.H, 1, w2.d_k, w2.n_sub, w2.d_v, w2.k_half, w2.W, w2.R,
                      w2.x_dtype, w2.v_dtype)
        assert sdm.decode_path(d2) == sdm.DECODE_FUSED, kw


def test_call_log_host_checks(lib):
    """sdm_call_log_bytes covers the rows and stamps of every write occurrence and Lambda;
    save and restore refuse bad arguments on the host (nothing is launched)."""
    class State(ctypes.Structure):
        _fields_ = [("M", ctypes.c_void_p), ("stamp", ctypes.c_void_p), ("Lambda", ctypes.c_void_p),
                    ("M0", ctypes.c_void_p)]
    lib.sdm_call_log_bytes.restype = ctypes.c_size_t
    d = mid_dims()
    BH, T, W, dv = 2 * 4, 4096, 32, 128
    nb = lib.sdm_call_log_bytes(ctypes.byref(d))
    assert nb >= BH * T * W * (dv * 4 + 8) + BH * 8
    assert nb < BH * T * W * (dv * 4 + 8) + BH * 8 + 3 * 256  # three 256-byte aligned sections
    # the log grows with the write slots, not with N or R
    assert lib.sdm_call_log_bytes(ctypes.byref(mid_dims(n_sub=512, R=8))) == nb
    assert lib.sdm_call_log_bytes(ctypes.byref(mid_dims(W=16))) < nb
    assert lib.sdm_call_log_bytes(ctypes.byref(mid_dims(W=65))) == 0  # bad dims
    p = ctypes.c_void_p(0x1000)
    st = State(0x1000, 0x2000, 0x3000, 0x4000)
    small = ctypes.c_size_t(nb - 1)
    assert lib.sdm_call_log_save(ctypes.byref(d), None, ctypes.byref(st), p,
                                 ctypes.c_size_t(nb), None) == 1                  # SDM_ERR_ARG
    assert lib.sdm_call_log_save(ctypes.byref(d), p, ctypes.byref(st), p, small, None) == 7
    assert lib.sdm_call_log_restore(ctypes.byref(d), p, p, small, ctypes.byref(st), None) == 7
    assert lib.sdm_call_log_restore(ctypes.byref(d), p, ctypes.c_void_p(0x1008),
                                    ctypes.c_size_t(nb), ctypes.byref(st), None) == 4  # ALIGN
    st_bad = State(0x1000, 0x2000, 0x3003, 0x4000)
    assert lib.sdm_call_log_save(ctypes.byref(d), p, ctypes.byref(st_bad), p,
                                 ctypes.c_size_t(nb), None) == 4
