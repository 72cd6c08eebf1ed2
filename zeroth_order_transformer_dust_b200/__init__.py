"""Dust per-token activation-space gradient estimator on B200 (sm_100a).

Thin ctypes binding over the C ABI declared in ``include/dust.h``
(``libdust.so``, built in-tree by ``python -m zeroth_order_transformer_dust_b200.build``).
This module only marshals arguments: torch provides device memory and the
CUDA stream, and every step of the estimator runs in the library's kernels.
There is no CPU fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdust.so")

DUST_OK = 0
STATUS_NAMES = {0: "DUST_OK", 1: "DUST_ERR_ARG", 2: "DUST_ERR_CUDA", 3: "DUST_ERR_OOM",
                4: "DUST_ERR_BOUNDS", 5: "DUST_ERR_TIMEOUT", 6: "DUST_ERR_UNSUPPORTED"}
DUST_F32, DUST_BF16 = 0, 1
FLAG_LITERAL_TARGET_SCALE = 1 << 0
FLAG_ASYNC = 1 << 1
VARIANT_HEAD, VARIANT_MLP, VARIANT_ATTN = 0, 1, 2
TAG_HEAD, TAG_SUBSET_OFFSET, TAG_MLP_UP = 0, 1, 2

# Every extern "C" symbol include/dust.h declares.
EXPORTS = ("dust_create", "dust_set_stream", "dust_destroy", "dust_last_error",
           "dust_status_string", "dust_validate", "dust_subset_stride", "dust_check",
           "dust_head_grad", "dust_head_grad_host", "dust_mlp_grad", "dust_debug_philox",
           "dust_debug_gauss", "dust_set_stage_timing", "dust_stage_times",
           "dust_kernel_launches", "dust_debug_gemm_bf16", "dust_debug_gemm_bf16_mn",
           "dust_debug_gauss_tab",
           "dust_debug_gauss_tab_scalar",
           "dust_head_grad_noalloc", "dust_debug_bm_radius", "dust_debug_bm_angle",
           "dust_attn_grad",
           "dust_sgd_momentum", "dust_mlp_down_grad", "dust_attn_out_grad")


class DustParams(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("V", ctypes.c_int64),
                ("d_ff", ctypes.c_int64), ("K", ctypes.c_int32), ("S", ctypes.c_int32),
                ("sigma", ctypes.c_float), ("dtype", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("token_offset", ctypes.c_int64), ("draw_offset", ctypes.c_int64),
                ("subset_a", ctypes.c_int64), ("stream_id", ctypes.c_uint32),
                ("flags", ctypes.c_uint32)]


class DustAttnShape(ctypes.Structure):
    """dust_attn_shape: the geometry of the attention-internals variant."""
    _fields_ = [("seq_len", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("which", ctypes.c_int32)]


ATTN_WHICH = {"q": 0, "k": 1, "v": 2}


class DustError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None
_lib_lock = threading.Lock()


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdust.so (raises FileNotFoundError when it has not been built)."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise FileNotFoundError(
                f"{path} is missing: build it with `python -m zeroth_order_transformer_dust_b200.build`")
        L = ctypes.CDLL(path)
        P, I64, I32, U32, U64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                 ctypes.c_uint32, ctypes.c_uint64)
        PP = ctypes.POINTER(DustParams)
        sig = {
            "dust_create": (I32, [ctypes.POINTER(P), ctypes.c_int, P]),
            "dust_set_stream": (I32, [P, P]),
            "dust_destroy": (None, [P]),
            "dust_last_error": (ctypes.c_char_p, [P]),
            "dust_status_string": (ctypes.c_char_p, [I32]),
            "dust_validate": (I32, [PP, ctypes.c_int, ctypes.c_char_p, ctypes.c_int]),
            "dust_subset_stride": (I64, [PP]),
            "dust_check": (I32, [P]),
            "dust_head_grad": (I32, [P, PP, P, P, P, P, P, P, P]),
            "dust_head_grad_host": (I32, [P, PP, P, P, P, P, P, P, P]),
            "dust_mlp_grad": (I32, [P, PP, P, P, P, P, P, P, P, P, P]),
            "dust_mlp_down_grad": (I32, [P, PP, P, P, P, P, P, P, P, P, P]),
            "dust_attn_out_grad": (I32, [P, PP, P, P, I64, P, P, P, P, P, P, P, P]),
            "dust_attn_grad": (I32, [P, PP, ctypes.POINTER(DustAttnShape), P, P, P, P, P, P, P,
                                     P]),
            "dust_debug_philox": (I32, [P, U64, P, I64, P]),
            "dust_debug_gauss": (I32, [P, PP, I32, I64, I64, I64, P]),
            "dust_set_stage_timing": (I32, [P, ctypes.c_int]),
            "dust_stage_times": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_char_p),
                                                ctypes.POINTER(ctypes.c_float), ctypes.c_int]),
            "dust_kernel_launches": (I64, [P]),
            "dust_debug_gemm_bf16": (I32, [P, I64, I64, I64, P, P, P, ctypes.c_int]),
            "dust_debug_gemm_bf16_mn": (I32, [P, I64, I64, I64, P, P, P, ctypes.c_int]),
            "dust_debug_gauss_tab": (I32, [P, PP, I32, I64, I64, I64, P]),
            "dust_debug_gauss_tab_scalar": (I32, [P, PP, I32, I64, I64, I64, P]),
            "dust_head_grad_noalloc": (I32, [PP, P, P, P, P, P, P, P, P, ctypes.c_char_p,
                                             ctypes.c_int]),
            "dust_debug_bm_radius": (I32, [P, I32, ctypes.c_float, P]),
            "dust_debug_bm_angle": (I32, [P, I32, P]),
            "dust_sgd_momentum": (I32, [P, I64, ctypes.c_float, ctypes.c_float, P, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
        return L


def make_params(T, d, V, K, sigma, *, S=0, d_ff=0, dtype=DUST_BF16, seed=0, token_offset=0,
                draw_offset=0, subset_a=0, stream_id=0, flags=0) -> DustParams:
    return DustParams(T=T, d=d, V=V, d_ff=d_ff, K=K, S=S, sigma=float(sigma), dtype=dtype,
                      seed=seed & 0xFFFFFFFFFFFFFFFF, token_offset=token_offset,
                      draw_offset=draw_offset, subset_a=subset_a, stream_id=stream_id,
                      flags=flags)


def validate(params: DustParams, variant: int = VARIANT_HEAD):
    """Host-only parameter check; returns (status, message)."""
    L = load_library()
    buf = ctypes.create_string_buffer(256)
    st = L.dust_validate(ctypes.byref(params), variant, buf, 256)
    return st, buf.value.decode()


def subset_stride(params: DustParams) -> int:
    return int(load_library().dust_subset_stride(ctypes.byref(params)))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DUST_BF16
    if t.dtype == torch.float32:
        return DUST_F32
    raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")


# The C-ABI takes plain pointers and reads every size from its parameters, so
# the binding checks that each tensor's shape agrees with those sizes: a
# mismatch would otherwise read or write beyond the tensor.
def _matrix(t: torch.Tensor, name: str):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _shape(t: torch.Tensor, shape, name: str):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_outputs(out: dict, shapes: dict, device: Optional[int]):
    """Caller-supplied outputs: fp32, contiguous, the expected shape, and on
    cuda:device (device None: host memory)."""
    for key, shape in shapes.items():
        t = out.get(key)
        if t is None:
            continue
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"output {key} must be a contiguous fp32 tensor")
        on_dev = t.is_cuda and t.device.index == device
        if (device is None and t.is_cuda) or (device is not None and not on_dev):
            raise ValueError(f"output {key} is on the wrong device")
        _shape(t, shape, f"output {key}")


def _head_shapes(H, W, targets):
    """(T, d, V) of the LM-head call; raises on inconsistent shapes."""
    T, d = _matrix(H, "H")
    V, dw = _matrix(W, "W")
    if dw != d:
        raise ValueError(f"W must be V x {d} (H is T x {d}), got {tuple(W.shape)}")
    _shape(targets, (T,), "targets")
    return T, d, V


def _mlp_shapes(X, W_up, W_down, W_head, targets, O=None):
    """(T, d, d_ff, V) of the MLP-block call; raises on inconsistent shapes
    or dtypes (every operand bf16)."""
    T, d = _matrix(X, "X")
    d_ff = _matrix(W_up, "W_up")[0]
    _shape(W_up, (d_ff, d), "W_up")
    _shape(W_down, (d, d_ff), "W_down")
    V = _matrix(W_head, "W_head")[0]
    _shape(W_head, (V, d), "W_head")
    _shape(targets, (T,), "targets")
    ops = [(X, "X"), (W_up, "W_up"), (W_down, "W_down"), (W_head, "W_head")]
    if O is not None:
        if _matrix(O, "O")[0] != T:
            raise ValueError(f"O must have {T} rows, got {tuple(O.shape)}")
        ops.append((O, "O"))
    for t, n in ops:
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{n} must be bfloat16")
    if targets.dtype != torch.int32:
        raise TypeError("targets must be int32")
    return T, d, d_ff, V


def _attn_shapes(X, Q, K_cache, V_cache, E, n_heads):
    """(T, d, D) of the attention-internals call; raises on inconsistent
    shapes or dtypes."""
    T, d = _matrix(X, "X")
    D = _matrix(Q, "Q")[1]
    for t, n in ((Q, "Q"), (K_cache, "K_cache"), (V_cache, "V_cache"), (E, "E")):
        if t.dtype != torch.float32:
            raise TypeError(f"{n} must be fp32")
        _shape(t, (T, D), n)
    if n_heads < 1 or D % n_heads:
        raise ValueError("the width of Q must be a positive multiple of n_heads")
    return T, d, D


class Context:
    """A library context bound to one CUDA device and (by default) torch's current stream."""

    def __init__(self, device: Optional[int] = None, stream: Optional[torch.cuda.Stream] = None):
        self._L = load_library()
        if device is None:
            device = torch.cuda.current_device()
        self.device = int(device)
        h = ctypes.c_void_p()
        st = self._L.dust_create(ctypes.byref(h), self.device, None)
        if st != DUST_OK:
            raise DustError(st, f"dust_create(device={self.device}) failed")
        self._h = h
        self._stream = stream

    def close(self):
        if getattr(self, "_h", None):
            self._L.dust_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- helpers ---------------------------------------------------------------
    def _bind_stream(self):
        s = self._stream if self._stream is not None else torch.cuda.current_stream(self.device)
        self._L.dust_set_stream(self._h, ctypes.c_void_p(s.cuda_stream))

    def _check(self, st: int):
        if st != DUST_OK:
            msg = self._L.dust_last_error(self._h).decode()
            raise DustError(st, msg)

    def check(self):
        self._check(self._L.dust_check(self._h))

    def _dev(self, t: torch.Tensor, name: str):
        if not t.is_cuda or t.device.index != self.device:
            raise ValueError(f"{name} must be on cuda:{self.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return t

    # -- estimator ---------------------------------------------------------------
    def head_grad(self, H, W, targets, *, K, sigma, S=0, seed=0, token_offset=0, draw_offset=0,
                  subset_a=0, stream_id=0, literal_target_scale=False, want_G=True,
                  want_loss=True, want_rewards=False, want_g=False, asynchronous=False,
                  out=None) -> dict:
        """LM-head estimator. H (T x d), W (V x d) on this device, fp32 or bf16;
        targets (T,) int32. Returns a dict of the requested fp32 outputs."""
        self._dev(H, "H"), self._dev(W, "W"), self._dev(targets, "targets")
        if H.dtype != W.dtype:
            raise TypeError("H and W must share a dtype")
        if targets.dtype != torch.int32:
            raise TypeError("targets must be int32")
        T, d, V = _head_shapes(H, W, targets)
        flags = (FLAG_LITERAL_TARGET_SCALE if literal_target_scale else 0) | (
            FLAG_ASYNC if asynchronous else 0)
        prm = make_params(T, d, V, K, sigma, S=S, dtype=_dtype_code(H), seed=seed,
                          token_offset=token_offset, draw_offset=draw_offset, subset_a=subset_a,
                          stream_id=stream_id, flags=flags)
        out = dict(out or {})
        _check_outputs(out, {"G": (V, d), "loss": (T,), "rewards": (T, K), "g": (T, V)},
                       self.device)
        dev = H.device
        f32 = dict(dtype=torch.float32, device=dev)
        if want_G and "G" not in out:
            out["G"] = torch.empty(V, d, **f32)
        if want_loss and "loss" not in out:
            out["loss"] = torch.empty(T, **f32)
        if want_rewards and "rewards" not in out:
            out["rewards"] = torch.empty(T, K, **f32)
        if want_g and "g" not in out:
            out["g"] = torch.empty(T, V, **f32)
        self._bind_stream()
        st = self._L.dust_head_grad(self._h, ctypes.byref(prm), _ptr(H), _ptr(W), _ptr(targets),
                                    _ptr(out.get("G")), _ptr(out.get("loss")),
                                    _ptr(out.get("rewards")), _ptr(out.get("g")))
        self._check(st)
        return out

    def head_grad_host(self, H, W, targets, *, K, sigma, S=0, seed=0, token_offset=0,
                       draw_offset=0, subset_a=0, stream_id=0, out=None, want_G=True,
                       want_loss=True, want_rewards=False, want_g=False) -> dict:
        """Same estimator with every tensor in host memory (pin it for fast copies);
        the call copies the inputs to the device and the outputs back."""
        for t, n in ((H, "H"), (W, "W"), (targets, "targets")):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous host tensor")
        if H.dtype != W.dtype:
            raise TypeError("H and W must share a dtype")
        if targets.dtype != torch.int32:
            raise TypeError("targets must be int32")
        T, d, V = _head_shapes(H, W, targets)
        prm = make_params(T, d, V, K, sigma, S=S, dtype=_dtype_code(H), seed=seed,
                          token_offset=token_offset, draw_offset=draw_offset, subset_a=subset_a,
                          stream_id=stream_id)
        out = dict(out or {})
        _check_outputs(out, {"G": (V, d), "loss": (T,), "rewards": (T, K), "g": (T, V)}, None)
        for name, want, shape in (("G", want_G, (V, d)), ("loss", want_loss, (T,)),
                                  ("rewards", want_rewards, (T, K)), ("g", want_g, (T, V))):
            if want and name not in out:
                out[name] = torch.empty(*shape, dtype=torch.float32, pin_memory=True)
        self._bind_stream()
        st = self._L.dust_head_grad_host(self._h, ctypes.byref(prm), _ptr(H), _ptr(W),
                                         _ptr(targets), _ptr(out.get("G")), _ptr(out.get("loss")),
                                         _ptr(out.get("rewards")), _ptr(out.get("g")))
        self._check(st)
        return out

    def mlp_grad(self, X, W_up, W_down, W_head, targets, *, K, sigma, seed=0, token_offset=0,
                 draw_offset=0, stream_id=0, want_G=True, want_loss=True, want_rewards=False,
                 want_g=False, out=None, layer="up", O=None) -> dict:
        """MLP-block estimator (bf16 inputs) for the up-projection (layer="up":
        G is d_ff x d, g is T x d_ff), the down-projection (layer="down": G is
        d x d_ff, g is T x d) or the attention output projection whose output
        enters the block (layer="attn_out", O its T x d_o input: G is d x d_o,
        g is T x d). Returns the requested fp32 outputs."""
        if layer not in ("up", "down", "attn_out"):
            raise ValueError("layer must be 'up', 'down' or 'attn_out'")
        if (layer == "attn_out") != (O is not None):
            raise ValueError("O is given exactly for layer='attn_out'")
        if O is not None:
            self._dev(O, "O")
        for t, n in ((X, "X"), (W_up, "W_up"), (W_down, "W_down"), (W_head, "W_head"),
                     (targets, "targets")):
            self._dev(t, n)
        T, d, d_ff, V = _mlp_shapes(X, W_up, W_down, W_head, targets, O)
        prm = make_params(T, d, V, K, sigma, d_ff=d_ff, dtype=_dtype_code(X), seed=seed,
                          token_offset=token_offset, draw_offset=draw_offset, stream_id=stream_id)
        out = dict(out or {})
        f32 = dict(dtype=torch.float32, device=X.device)
        width = d_ff if layer == "up" else d
        gshape = {"up": (d_ff, d), "down": (d, d_ff)}.get(layer) or (d, O.shape[1])
        _check_outputs(out, {"G": gshape, "loss": (T,), "rewards": (T, K), "g": (T, width)},
                       self.device)
        if want_G and "G" not in out:
            out["G"] = torch.empty(*gshape, **f32)
        if want_loss and "loss" not in out:
            out["loss"] = torch.empty(T, **f32)
        if want_rewards and "rewards" not in out:
            out["rewards"] = torch.empty(T, K, **f32)
        if want_g and "g" not in out:
            out["g"] = torch.empty(T, width, **f32)
        self._bind_stream()
        tail = (_ptr(targets), _ptr(out.get("G")), _ptr(out.get("loss")),
                _ptr(out.get("rewards")), _ptr(out.get("g")))
        if layer == "attn_out":
            st = self._L.dust_attn_out_grad(self._h, ctypes.byref(prm), _ptr(X), _ptr(O),
                                            O.shape[1], _ptr(W_up), _ptr(W_down), _ptr(W_head),
                                            *tail)
        else:
            fn = self._L.dust_mlp_grad if layer == "up" else self._L.dust_mlp_down_grad
            st = fn(self._h, ctypes.byref(prm), _ptr(X), _ptr(W_up), _ptr(W_down), _ptr(W_head),
                    *tail)
        self._check(st)
        return out

    def attn_grad(self, X, Q, K_cache, V_cache, E, *, seq_len, n_heads, which, K, sigma, seed=0,
                  token_offset=0, draw_offset=0, stream_id=0, want_G=True, want_rewards=False,
                  want_g=False, out=None) -> dict:
        """Attention-internals estimator: noise on the output of the query
        (which="q"), key ("k") or value ("v") projection. X (T x d, fp32 or
        bf16) is the projection's input; Q, K_cache, V_cache (T x D fp32) the
        cached projections; E (T x D fp32) the error signal at the attention
        output; D = n_heads head_dim. G is D x d, g is T x D, rewards T x K."""
        if which not in ATTN_WHICH:
            raise ValueError("which must be 'q', 'k' or 'v'")
        for t, n in ((X, "X"), (Q, "Q"), (K_cache, "K_cache"), (V_cache, "V_cache"), (E, "E")):
            self._dev(t, n)
        T, d, D = _attn_shapes(X, Q, K_cache, V_cache, E, n_heads)
        shape = DustAttnShape(seq_len=seq_len, n_heads=n_heads, head_dim=D // n_heads,
                              which=ATTN_WHICH[which])
        prm = make_params(T, d, 1, K, sigma, dtype=_dtype_code(X), seed=seed,
                          token_offset=token_offset, draw_offset=draw_offset, stream_id=stream_id)
        out = dict(out or {})
        _check_outputs(out, {"G": (D, d), "rewards": (T, K), "g": (T, D)}, self.device)
        f32 = dict(dtype=torch.float32, device=X.device)
        if want_G and "G" not in out:
            out["G"] = torch.empty(D, d, **f32)
        if want_rewards and "rewards" not in out:
            out["rewards"] = torch.empty(T, K, **f32)
        if want_g and "g" not in out:
            out["g"] = torch.empty(T, D, **f32)
        self._bind_stream()
        self._check(self._L.dust_attn_grad(self._h, ctypes.byref(prm), ctypes.byref(shape),
                                           _ptr(X), _ptr(Q), _ptr(K_cache), _ptr(V_cache),
                                           _ptr(E), _ptr(out.get("G")), _ptr(out.get("rewards")),
                                           _ptr(out.get("g"))))
        return out

    # -- instrumentation -------------------------------------------------------------
    def set_stage_timing(self, enable: bool = True):
        self._check(self._L.dust_set_stage_timing(self._h, 1 if enable else 0))

    def stage_times(self) -> dict:
        """Per-stage device milliseconds of the last call (stage timing must be on)."""
        names = (ctypes.c_char_p * 16)()
        ms = (ctypes.c_float * 16)()
        n = self._L.dust_stage_times(self._h, names, ms, 16)
        return {names[i].decode(): float(ms[i]) for i in range(min(n, 16))}

    @property
    def kernel_launches(self) -> int:
        return int(self._L.dust_kernel_launches(self._h))

    def sgd_momentum(self, G, v, W, *, lr: float, mu: float, W_bf16=None) -> None:
        """Heavy-ball step in place: v <- mu v + G, W <- W - lr v (fp32 device
        tensors of one size); W_bf16, if given, receives W rounded to bf16."""
        for t, name in ((G, "G"), (v, "v"), (W, "W")):
            self._dev(t, name)
            if t.dtype != torch.float32 or t.numel() != G.numel():
                raise TypeError(f"{name} must be fp32 with G's size")
        if W_bf16 is not None:
            self._dev(W_bf16, "W_bf16")
            if W_bf16.dtype != torch.bfloat16 or W_bf16.numel() != G.numel():
                raise TypeError("W_bf16 must be bf16 with G's size")
        self._bind_stream()
        self._check(self._L.dust_sgd_momentum(self._h, G.numel(), float(lr), float(mu), _ptr(G),
                                              _ptr(v), _ptr(W), _ptr(W_bf16)))

    # -- debug exports -------------------------------------------------------------
    def debug_gemm(self, A: torch.Tensor, B: torch.Tensor, path: int = 0) -> torch.Tensor:
        """C = A B^T (bf16 operands, fp32 out); path 0 auto, 1 CUDA cores, 2 tensor cores
        (one CTA per tile), 3 tensor cores with CTA pairs, 4 path 2 with an injected
        timeout of its pipeline waits (raises DustError with DUST_ERR_TIMEOUT)."""
        self._dev(A, "A"), self._dev(B, "B")
        if A.dtype != torch.bfloat16 or B.dtype != torch.bfloat16:
            raise TypeError("A and B must be bfloat16")
        M, K = _matrix(A, "A")
        N = _matrix(B, "B")[0]
        _shape(B, (N, K), "B")
        C = torch.empty(M, N, dtype=torch.float32, device=A.device)
        self._bind_stream()
        self._check(self._L.dust_debug_gemm_bf16(self._h, M, N, K, _ptr(A), _ptr(B), _ptr(C), path))
        return C

    def debug_gemm_mn(self, At: torch.Tensor, Bt: torch.Tensor, path: int = 0) -> torch.Tensor:
        """C = At^T Bt for MN-major operands At (K x M) and Bt (K x N), bf16, fp32 out;
        paths as debug_gemm."""
        self._dev(At, "At"), self._dev(Bt, "Bt")
        if At.dtype != torch.bfloat16 or Bt.dtype != torch.bfloat16:
            raise TypeError("At and Bt must be bfloat16")
        K, M = _matrix(At, "At")
        N = _matrix(Bt, "Bt")[1]
        _shape(Bt, (K, N), "Bt")
        C = torch.empty(M, N, dtype=torch.float32, device=At.device)
        self._bind_stream()
        self._check(self._L.dust_debug_gemm_bf16_mn(self._h, M, N, K, _ptr(At), _ptr(Bt), _ptr(C),
                                                    path))
        return C

    def debug_philox(self, seed: int, ctr: torch.Tensor) -> torch.Tensor:
        """Raw Philox4x32-10 words for counters ctr (n x 4, int32 storage of uint32)."""
        self._dev(ctr, "ctr")
        if ctr.dtype != torch.int32 or ctr.dim() != 2 or ctr.shape[1] != 4:
            raise ValueError("ctr must be an n x 4 int32 tensor")
        out = torch.empty_like(ctr)
        self._bind_stream()
        self._check(self._L.dust_debug_philox(self._h, seed & 0xFFFFFFFFFFFFFFFF, _ptr(ctr),
                                              ctr.shape[0], _ptr(out)))
        return out

    def debug_gauss(self, nt, ni, nslots, *, tag=TAG_HEAD, seed=0, token_offset=0, draw_offset=0,
                    stream_id=0, table=False, scalar=False) -> torch.Tensor:
        """eps[t, i, k]; table=True uses the LM-head kernels' table-driven angle
        step in their packed form, with scalar=True in scalar form."""
        prm = make_params(1, 1, 1, 1, 0.0, seed=seed, token_offset=token_offset,
                          draw_offset=draw_offset, stream_id=stream_id)
        out = torch.empty(nt, ni, nslots, dtype=torch.float32, device=f"cuda:{self.device}")
        self._bind_stream()
        fn = ((self._L.dust_debug_gauss_tab_scalar if scalar else self._L.dust_debug_gauss_tab)
              if table else self._L.dust_debug_gauss)
        self._check(fn(self._h, ctypes.byref(prm), tag, nt, ni, nslots, _ptr(out)))
        return out

    def debug_bm_radius(self, sigma: float = 1.0, table: bool = False) -> torch.Tensor:
        """For every u1 = (j + 1) 2^-24, j < 2^24: the radius sigma sqrt(-2 ln u1)
        of the polynomial angle step, or (table=True) rho = sqrt(-log2 u1), the
        factor of the table step."""
        out = torch.empty(1 << 24, dtype=torch.float32, device=f"cuda:{self.device}")
        self._bind_stream()
        self._check(self._L.dust_debug_bm_radius(self._h, 1 if table else 0, float(sigma),
                                                 _ptr(out)))
        return out

    def debug_bm_angle(self, table: bool) -> torch.Tensor:
        """(cos, sin) of 2 pi m 2^-24 for every m < 2^24 (2^24 x 2); the table
        step returns them times sqrt(2 ln 2)."""
        out = torch.empty(1 << 24, 2, dtype=torch.float32, device=f"cuda:{self.device}")
        self._bind_stream()
        self._check(self._L.dust_debug_bm_angle(self._h, 1 if table else 0, _ptr(out)))
        return out


_contexts: dict = {}


def context(device: Optional[int] = None) -> Context:
    """Per-device default context."""
    if device is None:
        device = torch.cuda.current_device()
    ctx = _contexts.get(device)
    if ctx is None:
        ctx = _contexts[device] = Context(device)
    return ctx


def head_grad(H, W, targets, **kw) -> dict:
    return context(H.device.index).head_grad(H, W, targets, **kw)


def mlp_grad(X, W_up, W_down, W_head, targets, **kw) -> dict:
    return context(X.device.index).mlp_grad(X, W_up, W_down, W_head, targets, **kw)


def attn_grad(X, Q, K_cache, V_cache, E, **kw) -> dict:
    return context(X.device.index).attn_grad(X, Q, K_cache, V_cache, E, **kw)
