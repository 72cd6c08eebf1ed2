"""The C-ABI library loads, exports every symbol the header declares, and
validates arguments on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest

import zeroth_order_transformer_dust_b200 as dust
from zeroth_order_transformer_dust_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dust.load_library()


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dust_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            names += _declared(h)
    assert "dust_head_grad" in names and "dust_mlp_grad" in names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(set(names)) == sorted(set(dust.EXPORTS)) or set(dust.EXPORTS) <= set(names)


def test_params_struct_layout_matches_header():
    # int64 x4, int32 x2, float, int32, uint64, int64 x3, uint32 x2
    assert ctypes.sizeof(dust.DustParams) == 88
    assert dust.DustParams.seed.offset == 48
    assert dust.DustParams.flags.offset == 84


def _p(**kw):
    base = dict(T=8, d=16, V=1000, K=4, sigma=0.01)
    base.update(kw)
    T, d, V, K, s = base.pop("T"), base.pop("d"), base.pop("V"), base.pop("K"), base.pop("sigma")
    return dust.make_params(T, d, V, K, s, **base)


@pytest.mark.parametrize("kw,frag", [
    (dict(T=0), "T must"), (dict(d=0), "d must"), (dict(V=0), "V must"), (dict(K=0), "K must"),
    (dict(sigma=-1.0), "sigma"), (dict(sigma=float("nan")), "sigma"),
    (dict(sigma=float("inf")), "sigma"), (dict(S=1001), "S must"),
    (dict(S=10, subset_a=500), "coprime"), (dict(S=10, subset_a=-3), "subset_a"),
    (dict(dtype=7), "dtype"), (dict(token_offset=-1), "token_offset"),
    (dict(token_offset=(1 << 32) - 4), "token_offset"), (dict(draw_offset=(1 << 32)), "draw_offset"),
    (dict(stream_id=1 << 24), "stream_id"),
])
def test_head_validation_rejects(lib, kw, frag):
    st, msg = dust.validate(_p(**kw), dust.VARIANT_HEAD)
    assert st == 1 and frag in msg


def test_head_validation_accepts(lib):
    for kw in (dict(), dict(S=1000), dict(S=1), dict(S=10, subset_a=7), dict(sigma=0.0),
               dict(token_offset=(1 << 32) - 8), dict(dtype=dust.DUST_F32)):
        st, msg = dust.validate(_p(**kw), dust.VARIANT_HEAD)
        assert st == 0, (kw, msg)


def test_mlp_validation(lib):
    ok = _p(d_ff=32)
    assert dust.validate(ok, dust.VARIANT_MLP)[0] == 0
    assert dust.validate(_p(d_ff=0), dust.VARIANT_MLP)[0] == 1
    assert dust.validate(_p(d_ff=32, S=4), dust.VARIANT_MLP)[0] == 1
    assert dust.validate(_p(d_ff=32, dtype=dust.DUST_F32), dust.VARIANT_MLP)[0] == 1
    assert dust.validate(ok, 7)[0] == 1


def test_attention_validation(lib):
    # the attention-internals variant ignores V and d_ff, perturbs every channel
    assert dust.validate(_p(V=0, d_ff=0), dust.VARIANT_ATTN)[0] == 0
    assert dust.validate(_p(dtype=dust.DUST_F32), dust.VARIANT_ATTN)[0] == 0
    assert dust.validate(_p(S=4), dust.VARIANT_ATTN)[0] == 1
    assert dust.validate(_p(K=0), dust.VARIANT_ATTN)[0] == 1
    assert dust.validate(_p(T=0), dust.VARIANT_ATTN)[0] == 1


def test_null_params_and_context(lib):
    assert lib.dust_validate(None, 0, None, 0) == 1
    p = _p()
    assert lib.dust_head_grad(None, ctypes.byref(p), None, None, None, None, None, None, None) == 1
    assert lib.dust_mlp_grad(None, ctypes.byref(p), *([None] * 9)) == 1
    assert lib.dust_check(None) == 1
    assert lib.dust_status_string(4) == b"DUST_ERR_BOUNDS"


def test_default_subset_stride_matches_the_documented_rule(lib):
    assert dust.subset_stride(_p(V=50304, S=512)) == 31091
    assert dust.subset_stride(_p(V=1024, S=8)) == 633
    assert dust.subset_stride(_p(V=1000, S=8, subset_a=1003)) == 3
    assert dust.subset_stride(_p(V=1000, S=0)) == 0


def test_binding_fails_loudly_without_the_library(tmp_path):
    with pytest.raises(FileNotFoundError):
        dust._lib_saved = dust._lib
        try:
            dust._lib = None
            dust.load_library(str(tmp_path / "nope.so"))
        finally:
            dust._lib = dust._lib_saved


def _noalloc(lib):
    fn = lib.dust_head_grad_noalloc
    fn.restype = ctypes.c_int32
    fn.argtypes = ([ctypes.POINTER(dust.DustParams), ctypes.c_void_p] + [ctypes.c_void_p] * 7
                   + [ctypes.c_char_p, ctypes.c_int])
    return fn


@pytest.mark.parametrize("bad", ["H", "W", "targets", "G", "loss", "rewards", "g"])
def test_noalloc_rejects_misaligned_pointers_before_any_cuda_call(lib, bad):
    """The allocation-free entry point checks alignment on the host: the call
    returns DUST_ERR_ARG without touching a device (none exists here), so the
    fake addresses below are never dereferenced."""
    prm = _p(S=10)
    ptrs = {"H": 0x10000, "W": 0x20000, "targets": 0x30000, "G": 0x40000, "loss": 0x50000,
            "rewards": 0x60000, "g": 0x70000}
    ptrs[bad] += 2 if bad in ("H", "W", "targets") else 1
    if bad in ("H", "W"):
        ptrs[bad] = ptrs[bad] - 2 + 8          # 8-byte but not 16-byte aligned
    msg = ctypes.create_string_buffer(256)
    st = _noalloc(lib)(ctypes.byref(prm), None, *[ctypes.c_void_p(ptrs[k]) for k in
                       ("H", "W", "targets", "G", "loss", "rewards", "g")], msg, 256)
    assert st == 1 and b"aligned" in msg.value


def test_noalloc_rejects_bad_parameters_on_the_host(lib):
    msg = ctypes.create_string_buffer(256)
    p = ctypes.c_void_p(0x10000)
    st = _noalloc(lib)(ctypes.byref(_p(K=0)), None, p, p, p, p, p, p, p, msg, 256)
    assert st == 1 and b"K must" in msg.value
    st = _noalloc(lib)(ctypes.byref(_p()), None, None, p, p, p, p, p, p, msg, 256)
    assert st == 1 and b"non-NULL" in msg.value
