"""The allocation-free entry point against dust_head_grad and the oracle.

dust_head_grad_noalloc serves callers that cannot call cudaMalloc (their
device memory belongs to another allocator, or they cannot afford the
synchronisation an allocation may cause): it keeps all its scratch in a fixed
16 MiB device array. Its outputs must agree with the allocating entry point's
and with the oracle within the parity tolerances, on two calls in a row (the
array is shared and keeps the previous call's contents), and the device's
free memory must not move across its calls.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import zeroth_order_transformer_dust_b200 as dust
from _util import TOL_G, TOL_GW_BF16, TOL_GW_F32, TOL_LOSS, rel_fro

pytestmark = pytest.mark.gpu


def _entry():
    fn = dust.load_library().dust_head_grad_noalloc
    fn.restype = ctypes.c_int32
    fn.argtypes = ([ctypes.POINTER(dust.DustParams), ctypes.c_void_p] + [ctypes.c_void_p] * 7
                   + [ctypes.c_char_p, ctypes.c_int])
    return fn


WORKLOADS = [
    synth.CONFIGS["tiny_fp32"],
    synth.Workload("noalloc_subset", "head", T=64, d=96, V=3000, K=32, S=200, sigma=1e-2, seed=7,
                   dtype="bf16", targets="zipf"),
    synth.Workload("noalloc_full", "head", T=40, d=64, V=2000, K=12, S=0, sigma=2e-2, seed=9,
                   dtype="bf16", targets="zipf"),
    synth.Workload("noalloc_subset_f32", "head", T=48, d=40, V=1500, K=24, S=77, sigma=2e-2,
                   seed=11, dtype="f32", targets="zipf"),
]


def _dev_inputs(wl, y=None):
    inp = synth.make_head_inputs(wl)
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    H = torch.from_numpy(inp["H"]).to(tdt).cuda()
    W = torch.from_numpy(inp["W"]).to(tdt).cuda()
    yd = torch.from_numpy(inp["targets"] if y is None else y).to(torch.int32).cuda()
    return inp, H, W, yd


def _call(fn, wl, H, W, y, out):
    prm = dust.make_params(wl.T, wl.d, wl.V, wl.K, wl.sigma, S=wl.S, seed=wl.seed,
                           dtype=dust.DUST_F32 if wl.dtype == "f32" else dust.DUST_BF16)
    msg = ctypes.create_string_buffer(256)
    st = fn(ctypes.byref(prm), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
            ctypes.c_void_p(H.data_ptr()), ctypes.c_void_p(W.data_ptr()),
            ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(out["G"].data_ptr()),
            ctypes.c_void_p(out["loss"].data_ptr()), ctypes.c_void_p(out["rewards"].data_ptr()),
            ctypes.c_void_p(out["g"].data_ptr()), msg, 256)
    return st, msg.value


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
def test_noalloc_matches_head_grad_and_the_oracle(cuda_ok, wl):
    inp, H, W, y = _dev_inputs(wl)
    ctx = dust.Context(0)
    ref = ctx.head_grad(H, W, y, K=wl.K, sigma=wl.sigma, S=wl.S, seed=wl.seed,
                        want_rewards=True, want_g=True)
    torch.cuda.synchronize()
    ref = {k: v.double().cpu().numpy() for k, v in ref.items()}
    prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=wl.K, S=wl.S, sigma=wl.sigma, seed=wl.seed)
    orc = oracle.head_grad(inp["H"], inp["W"], inp["targets"], prm)
    gw_tol = TOL_GW_F32 if wl.dtype == "f32" else TOL_GW_BF16
    fn = _entry()
    outs = [{"G": torch.empty(wl.V, wl.d, device="cuda"), "loss": torch.empty(wl.T, device="cuda"),
             "rewards": torch.empty(wl.T, wl.K, device="cuda"),
             "g": torch.empty(wl.T, wl.V, device="cuda")} for _ in range(3)]
    st, msg = _call(fn, wl, H, W, y, outs[0])      # first call on the device: the set-up
    assert st == 0, msg
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for out in outs[1:]:                           # two more calls: nothing allocated
        st, msg = _call(fn, wl, H, W, y, out)
        assert st == 0, msg
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
    for out in outs:
        got = {k: v.double().cpu().numpy() for k, v in out.items()}
        for other in (ref, orc):
            assert np.abs(got["loss"] - other["loss"]).max() < TOL_LOSS
            assert np.abs(got["rewards"] - other["rewards"]).max() < TOL_LOSS
            assert rel_fro(got["g"], other["g"]) < TOL_G
            assert rel_fro(got["G"], other["G"]) < gw_tol
    ctx.close()


def test_noalloc_reports_a_bad_target(cuda_ok):
    wl = WORKLOADS[1]
    y = synth.make_head_inputs(wl)["targets"].copy()
    y[10] = wl.V
    _, H, W, yd = _dev_inputs(wl, y)
    out = {"G": torch.empty(wl.V, wl.d, device="cuda"), "loss": torch.empty(wl.T, device="cuda"),
           "rewards": torch.empty(wl.T, wl.K, device="cuda"),
           "g": torch.empty(wl.T, wl.V, device="cuda")}
    st, msg = _call(_entry(), wl, H, W, yd, out)
    assert st == 4 and b"target" in msg
    # the status word in the shared array is cleared by the next call
    _, H, W, yd = _dev_inputs(wl)
    st, msg = _call(_entry(), wl, H, W, yd, out)
    assert st == 0, msg


def test_noalloc_rejects_sizes_beyond_its_array(cuda_ok):
    fn = _entry()
    prm = dust.make_params(4096, 512, 50304, 64, 1e-2, dtype=dust.DUST_BF16)
    msg = ctypes.create_string_buffer(256)
    dummy = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = fn(ctypes.byref(prm), None, p, p, p, p, p, None, None, msg, 256)
    assert st == 6 and b"scratch" in msg.value
