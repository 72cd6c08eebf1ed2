"""The Python binding's shape checks (no GPU): the C-ABI reads every size from
its parameters, so the binding must refuse tensors whose shapes disagree
with those sizes before any pointer reaches a kernel."""
import pytest
import torch

import zeroth_order_transformer_dust_b200 as dust

bf16, f32 = torch.bfloat16, torch.float32


def _t(*shape, dtype=f32):
    return torch.zeros(*shape, dtype=dtype)


def test_head_shapes():
    assert dust._head_shapes(_t(5, 8), _t(30, 8), _t(5, dtype=torch.int32)) == (5, 8, 30)
    with pytest.raises(ValueError, match="W must be V x 8"):
        dust._head_shapes(_t(5, 8), _t(30, 9), _t(5, dtype=torch.int32))
    with pytest.raises(ValueError, match="targets"):
        dust._head_shapes(_t(5, 8), _t(30, 8), _t(4, dtype=torch.int32))
    with pytest.raises(ValueError, match="H must be 2-D"):
        dust._head_shapes(_t(40), _t(30, 8), _t(5, dtype=torch.int32))


def test_mlp_shapes():
    T, d, dff, V = 6, 8, 16, 40
    y = _t(T, dtype=torch.int32)
    ok = dict(X=_t(T, d, dtype=bf16), W_up=_t(dff, d, dtype=bf16),
              W_down=_t(d, dff, dtype=bf16), W_head=_t(V, d, dtype=bf16), targets=y)
    assert dust._mlp_shapes(**ok) == (T, d, dff, V)
    assert dust._mlp_shapes(**ok, O=_t(T, 12, dtype=bf16)) == (T, d, dff, V)
    with pytest.raises(ValueError, match="W_down"):
        dust._mlp_shapes(**{**ok, "W_down": _t(dff, d, dtype=bf16)})
    with pytest.raises(ValueError, match="W_head"):
        dust._mlp_shapes(**{**ok, "W_head": _t(V, d + 1, dtype=bf16)})
    with pytest.raises(ValueError, match="targets"):
        dust._mlp_shapes(**{**ok, "targets": _t(T + 1, dtype=torch.int32)})
    with pytest.raises(ValueError, match="O must have 6 rows"):
        dust._mlp_shapes(**ok, O=_t(T - 1, 12, dtype=bf16))
    with pytest.raises(TypeError, match="W_up must be bfloat16"):
        dust._mlp_shapes(**{**ok, "W_up": _t(dff, d)})
    with pytest.raises(TypeError, match="targets must be int32"):
        dust._mlp_shapes(**{**ok, "targets": _t(T, dtype=torch.int64)})


def test_attn_shapes():
    T, d, D = 8, 5, 12
    qkve = [_t(T, D) for _ in range(4)]
    assert dust._attn_shapes(_t(T, d, dtype=bf16), *qkve, 3) == (T, d, D)
    with pytest.raises(ValueError, match="Q must have shape"):
        dust._attn_shapes(_t(T + 1, d), *qkve, 3)
    with pytest.raises(ValueError, match="E must have shape"):
        dust._attn_shapes(_t(T, d), *qkve[:3], _t(T, D + 1), 3)
    with pytest.raises(TypeError, match="K_cache must be fp32"):
        dust._attn_shapes(_t(T, d), qkve[0], _t(T, D, dtype=torch.float64), *qkve[2:], 3)
    with pytest.raises(ValueError, match="multiple of n_heads"):
        dust._attn_shapes(_t(T, d), *qkve, 5)


def test_caller_outputs():
    shapes = {"G": (4, 3), "loss": (7,)}
    dust._check_outputs({"G": _t(4, 3), "loss": _t(7)}, shapes, None)
    dust._check_outputs({"extra": _t(1)}, shapes, None)       # other keys pass through
    with pytest.raises(ValueError, match="output G must have shape"):
        dust._check_outputs({"G": _t(3, 4)}, shapes, None)
    with pytest.raises(ValueError, match="fp32"):
        dust._check_outputs({"loss": _t(7, dtype=bf16)}, shapes, None)
    with pytest.raises(ValueError, match="fp32"):
        dust._check_outputs({"G": _t(3, 4).t()}, shapes, None)  # not contiguous
    with pytest.raises(ValueError, match="wrong device"):
        dust._check_outputs({"G": _t(4, 3)}, shapes, 0)         # host tensor for cuda:0


class _FakeLib:
    """Records the C-ABI calls a Context makes and returns DUST_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("dust_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


def _fake_context():
    import ctypes
    import types
    c = dust.Context.__new__(dust.Context)
    c._L = _FakeLib()
    c.device = 0
    c._h = ctypes.c_void_p(1)
    c._stream = types.SimpleNamespace(cuda_stream=0)
    c._dev = lambda t, name: t          # host tensors stand in for device ones here
    return c


def _estimator_calls(c):
    return [(n, a) for n, a in c._L.calls if n.endswith("_grad")]


def test_head_call_marshals_sizes():
    c = _fake_context()
    out = c.head_grad(_t(5, 8), _t(30, 8), _t(5, dtype=torch.int32), K=4, sigma=0.1, S=7,
                      want_rewards=True, want_g=True, token_offset=3)
    (name, args), = _estimator_calls(c)
    prm = args[1]._obj
    assert name == "dust_head_grad"
    assert (prm.T, prm.d, prm.V, prm.K, prm.S, prm.token_offset) == (5, 8, 30, 4, 7, 3)
    assert {k: tuple(v.shape) for k, v in out.items()} == {
        "G": (30, 8), "loss": (5,), "rewards": (5, 4), "g": (5, 30)}
    with pytest.raises(ValueError):
        c.head_grad(_t(5, 8), _t(30, 8), _t(6, dtype=torch.int32), K=4, sigma=0.1)
    with pytest.raises(ValueError):
        c.head_grad(_t(5, 8), _t(30, 8), _t(5, dtype=torch.int32), K=4, sigma=0.1,
                    out={"G": _t(8, 30)})
    assert len(_estimator_calls(c)) == 1        # refused before reaching the library


@pytest.mark.parametrize("layer,fn,gshape,gwidth", [
    ("up", "dust_mlp_grad", (16, 8), 16), ("down", "dust_mlp_down_grad", (8, 16), 8),
    ("attn_out", "dust_attn_out_grad", (8, 24), 8)])
def test_mlp_call_marshals_sizes(layer, fn, gshape, gwidth):
    c = _fake_context()
    T, d, dff, V = 6, 8, 16, 40
    O = _t(T, 24, dtype=bf16) if layer == "attn_out" else None
    out = c.mlp_grad(_t(T, d, dtype=bf16), _t(dff, d, dtype=bf16), _t(d, dff, dtype=bf16),
                     _t(V, d, dtype=bf16), _t(T, dtype=torch.int32), K=3, sigma=0.1,
                     layer=layer, O=O, want_g=True)
    (name, args), = _estimator_calls(c)
    prm = args[1]._obj
    assert name == fn and (prm.T, prm.d, prm.V, prm.d_ff, prm.K) == (T, d, V, dff, 3)
    assert tuple(out["G"].shape) == gshape and tuple(out["g"].shape) == (T, gwidth)
    if layer == "attn_out":
        assert args[4] == 24                    # d_o, O's width
    with pytest.raises(ValueError):
        c.mlp_grad(_t(T, d, dtype=bf16), _t(dff, d, dtype=bf16), _t(dff, d, dtype=bf16),
                   _t(V, d, dtype=bf16), _t(T, dtype=torch.int32), K=3, sigma=0.1,
                   layer=layer, O=O)
    assert len(_estimator_calls(c)) == 1


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_attention_call_marshals_sizes(which):
    c = _fake_context()
    T, d, H, dh = 8, 5, 2, 64
    qkve = [_t(T, H * dh) for _ in range(4)]
    out = c.attn_grad(_t(T, d, dtype=bf16), *qkve, seq_len=4, n_heads=H, which=which, K=6,
                      sigma=0.1, want_rewards=True, want_g=True)
    (name, args), = _estimator_calls(c)
    prm, shape = args[1]._obj, args[2]._obj
    assert name == "dust_attn_grad" and (prm.T, prm.d, prm.K) == (T, d, 6)
    assert (shape.seq_len, shape.n_heads, shape.head_dim, shape.which) == (
        4, H, dh, dust.ATTN_WHICH[which])
    assert {k: tuple(v.shape) for k, v in out.items()} == {
        "G": (H * dh, d), "rewards": (T, 6), "g": (T, H * dh)}
    with pytest.raises(ValueError):
        c.attn_grad(_t(T - 1, d, dtype=bf16), *qkve, seq_len=4, n_heads=H, which=which, K=6,
                    sigma=0.1)
    assert len(_estimator_calls(c)) == 1


def test_debug_exports_check_layouts():
    c = _fake_context()
    C = c.debug_gemm(_t(3, 16, dtype=bf16), _t(5, 16, dtype=bf16))
    assert tuple(C.shape) == (3, 5)
    with pytest.raises(ValueError, match="B must have shape"):
        c.debug_gemm(_t(3, 16, dtype=bf16), _t(5, 8, dtype=bf16))
    assert tuple(c.debug_philox(1, _t(7, 4, dtype=torch.int32)).shape) == (7, 4)
    for bad in (_t(7, 3, dtype=torch.int32), _t(28, dtype=torch.int32), _t(7, 4)):
        with pytest.raises(ValueError, match="n x 4 int32"):
            c.debug_philox(1, bad)
    assert [n for n, _ in c._L.calls if n.startswith("dust_debug")] == [
        "dust_debug_gemm_bf16", "dust_debug_philox"]


def test_training_loop_draw_offsets_and_reduction():
    # step s of a run resumed at first_step draws at [(first_step + s) K, ...),
    # the all-reduce hook sees every step's G before its update, and the
    # update receives the bf16 copy to refresh
    from zeroth_order_transformer_dust_b200.train import train_head
    c = _fake_context()
    c.device = None                     # outputs live in host memory here
    reduced = []
    W_lp = _t(30, 8, dtype=bf16)
    train_head(c, _t(5, 8, dtype=bf16), _t(30, 8), _t(5, dtype=torch.int32), steps=3, lr=0.1,
               mu=0.9, K=16, sigma=0.01, S=4, seed=2, token_offset=40, W_lp=W_lp, first_step=5,
               allreduce=lambda G: reduced.append(G.data_ptr()))
    heads = [a[1]._obj for n, a in c._L.calls if n == "dust_head_grad"]
    assert [p.draw_offset for p in heads] == [80, 96, 112]
    assert all((p.token_offset, p.K, p.S, p.seed) == (40, 16, 4, 2) for p in heads)
    updates = [a for n, a in c._L.calls if n == "dust_sgd_momentum"]
    assert len(updates) == 3 and len(reduced) == 3
    assert all(u[7].value == W_lp.data_ptr() for u in updates)
    assert [n for n, _ in c._L.calls].count("dust_check") == 1
