"""The allocation-free entry point against dust_head_grad.

dust_head_grad_noalloc serves callers that cannot call cudaMalloc (their
device memory belongs to another allocator, or they cannot afford the
synchronisation an allocation may cause): it keeps all its scratch in a fixed
16 MiB device array. Its outputs must agree with the allocating entry point's
within the parity tolerances, on two calls in a row (the array is shared and
keeps the previous call's contents).
"""
import ctypes

import numpy as np
import pytest
import torch

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
]


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
def test_noalloc_matches_head_grad(cuda_ok, wl):
    inp = synth.make_head_inputs(wl)
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    H = torch.from_numpy(inp["H"]).to(tdt).cuda()
    W = torch.from_numpy(inp["W"]).to(tdt).cuda()
    y = torch.from_numpy(inp["targets"]).to(torch.int32).cuda()
    ctx = dust.Context(0)
    ref = ctx.head_grad(H, W, y, K=wl.K, sigma=wl.sigma, S=wl.S, seed=wl.seed,
                        want_rewards=True, want_g=True)
    torch.cuda.synchronize()
    ref = {k: v.double().cpu().numpy() for k, v in ref.items()}
    fn = _entry()
    for _ in range(2):
        out = {"G": torch.empty(wl.V, wl.d, device="cuda"), "loss": torch.empty(wl.T, device="cuda"),
               "rewards": torch.empty(wl.T, wl.K, device="cuda"),
               "g": torch.empty(wl.T, wl.V, device="cuda")}
        prm = dust.make_params(wl.T, wl.d, wl.V, wl.K, wl.sigma, S=wl.S, seed=wl.seed,
                               dtype=dust.DUST_F32 if wl.dtype == "f32" else dust.DUST_BF16)
        msg = ctypes.create_string_buffer(256)
        st = fn(ctypes.byref(prm), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                ctypes.c_void_p(H.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(out["G"].data_ptr()),
                ctypes.c_void_p(out["loss"].data_ptr()), ctypes.c_void_p(out["rewards"].data_ptr()),
                ctypes.c_void_p(out["g"].data_ptr()), msg, 256)
        assert st == 0, msg.value
        torch.cuda.synchronize()
        got = {k: v.double().cpu().numpy() for k, v in out.items()}
        assert np.abs(got["loss"] - ref["loss"]).max() < TOL_LOSS
        assert np.abs(got["rewards"] - ref["rewards"]).max() < TOL_LOSS
        assert rel_fro(got["g"], ref["g"]) < TOL_G
        assert rel_fro(got["G"], ref["G"]) < (TOL_GW_F32 if wl.dtype == "f32" else TOL_GW_BF16)
    ctx.close()


def test_noalloc_rejects_sizes_beyond_its_array(cuda_ok):
    fn = _entry()
    prm = dust.make_params(4096, 512, 50304, 64, 1e-2, dtype=dust.DUST_BF16)
    msg = ctypes.create_string_buffer(256)
    dummy = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = fn(ctypes.byref(prm), None, p, p, p, p, p, None, None, msg, 256)
    assert st == 6 and b"scratch" in msg.value
