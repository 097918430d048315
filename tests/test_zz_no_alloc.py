"""sdm_forward_noalloc: the recurrence with the library's fixed device scratch array.

Some callers cannot allocate device memory at all — a custom operator inside a host
framework that owns the device allocator and forbids side allocations, or a loop whose
memory budget is fixed when the process starts — and cannot hand the library a
workspace either.  sdm_forward_noalloc serves them from one fixed 64 MiB array in
device memory.  These tests call it through the C ABI and check it against
sdm_forward (caller workspace) on two calls in a row with different shapes, so that
nothing left in the shared array by one call can leak into the next.  The file is
named to be collected last; it passes alone in a fresh process and after the others.
"""
import ctypes

import pytest
import torch

import sdm_synth as S
from tests.parity import TOL, f64, per_bh_rel_err


def _dims(sdm, wl):
    return sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                    wl.x_dtype, wl.v_dtype)


def _case(sdm, wl, seed):
    inp = {k: v.cuda() for k, v in S.generate(wl, seed=seed).items()}
    d = _dims(sdm, wl)
    g = torch.Generator().manual_seed(seed)
    widx = S.random_indices(wl.B, wl.H, wl.T, wl.N, wl.W, g, pool=min(wl.N, 4 * wl.W)).cuda()
    ridx = S.random_indices(wl.B, wl.H, wl.T, wl.N, wl.R, g, pool=min(wl.N, 4 * wl.R)).cuda()
    ww = S.random_weights(wl.B, wl.H, wl.T, wl.W, g).cuda()
    rw = S.random_weights(wl.B, wl.H, wl.T, wl.R, g).cuda()
    return inp, d, (widx, ww, ridx, rw)


@pytest.mark.gpu
def test_noalloc_matches_forward_two_calls():
    assert torch.cuda.is_available()
    import sparse_state_linear_score_b200 as sdm
    sdm.device_error(clear=True)
    cases = [(S.MID.scaled(B=1, H=2, T=600), 11), (S.TINY.scaled(B=2, H=3, T=150), 12)]
    for wl, seed in cases:
        inp, d, (widx, ww, ridx, rw) = _case(sdm, wl, seed)
        assert 0 < sdm.forward_workspace_bytes(d) <= 64 << 20
        st_ref = sdm.State(d, inp["M0"])
        st_new = sdm.State(d, inp["M0"])
        sdm.state_reset(d, st_ref)
        sdm.state_reset(d, st_new)
        ref = sdm.forward(d, inp["v"], inp["alpha"], inp["beta"], widx, ww, ridx, rw, st_ref)
        out = torch.full_like(ref, float("nan"))
        # through the C ABI directly
        status = sdm._lib.sdm_forward_noalloc(
            ctypes.byref(d), ctypes.c_void_p(inp["v"].data_ptr()),
            ctypes.c_void_p(inp["alpha"].data_ptr()), ctypes.c_void_p(inp["beta"].data_ptr()),
            ctypes.c_void_p(widx.data_ptr()), ctypes.c_void_p(ww.data_ptr()),
            ctypes.c_void_p(ridx.data_ptr()), ctypes.c_void_p(rw.data_ptr()),
            ctypes.byref(st_new.c), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert status == 0, sdm._lib.sdm_status_str(status)
        torch.cuda.synchronize()
        tol = TOL[wl.v_dtype]
        err = per_bh_rel_err(f64(out), f64(ref))
        assert err <= tol, f"outputs differ from sdm_forward: max rel err {err:.3e}"
        # the same deterministic kernels on the same inputs: equal bit for bit
        assert torch.equal(out, ref), f"outputs not bitwise equal (max rel err {err:.3e})"
        M_ref = sdm.state_materialize(d, st_ref)
        M_new = sdm.state_materialize(d, st_new)
        assert torch.equal(M_new, M_ref), \
            f"memory not bitwise equal (max rel err {per_bh_rel_err(f64(M_new), f64(M_ref)):.3e})"
        # stamps hold NaN for slots never written: compare their bits
        assert torch.equal(st_new.stamp.view(torch.int64), st_ref.stamp.view(torch.int64))
        assert torch.equal(st_new.Lambda, st_ref.Lambda)
    assert sdm.device_error() == 0


@pytest.mark.gpu
def test_noalloc_rejects_oversized_workspace():
    import sparse_state_linear_score_b200 as sdm
    wl = S.MID  # B=2 H=4 T=4096: workspace above 64 MiB? use a longer T to be sure
    d = sdm.Dims(wl.B, wl.H, 4 * wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R,
                 wl.x_dtype, wl.v_dtype)
    assert sdm.forward_workspace_bytes(d) > 64 << 20
    # small real device buffers for every pointer: were the size check ever moved behind a
    # launch, the kernels would get valid addresses (and the status would be wrong) rather
    # than arbitrary ones
    buf = [torch.zeros(64, dtype=torch.float32, device="cuda") for _ in range(12)]
    p = [ctypes.c_void_p(t.data_ptr()) for t in buf]
    st = sdm._CState(buf[8].data_ptr(), buf[9].data_ptr(), buf[10].data_ptr(), buf[11].data_ptr())
    status = sdm._lib.sdm_forward_noalloc(ctypes.byref(d), *p[:7], ctypes.byref(st), p[7], None)
    torch.cuda.synchronize()
    assert status == 7  # SDM_ERR_WORKSPACE, nothing enqueued
    assert all(int(torch.count_nonzero(t)) == 0 for t in buf)
