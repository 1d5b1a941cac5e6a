"""Thin ctypes binding of ``liblmoe.so`` (include/lmoe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  The functions keep the C names; torch tensors (device memory)
are passed as raw pointers, streams as ``torch.cuda.Stream`` or raw handles.
If the shared library is missing or fails to load, importing this module
raises -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

from .configs import LayerConfig

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblmoe.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} not built; run `python -m latent_mixture_experts_top_b200.build`")
_lib = C.CDLL(_LIB_PATH)

LMOE_EFF, LMOE_ACC = 0, 1
LMOE_F32, LMOE_BF16 = 0, 1
LMOE_SWIGLU, LMOE_RELU2 = 0, 1
LMOE_WEIGHTS_BF16, LMOE_WEIGHTS_FP8, LMOE_WEIGHTS_NVFP4 = 0, 1, 2
STATUS = {0: "LMOE_OK", -1: "LMOE_ERR_INVALID_CONFIG", -2: "LMOE_ERR_NULL_ARG",
          -3: "LMOE_ERR_NOT_LOADED", -4: "LMOE_ERR_TOO_MANY_TOKENS", -5: "LMOE_ERR_CUDA",
          -6: "LMOE_ERR_DEVICE_TIMEOUT", -7: "LMOE_ERR_UNSUPPORTED",
          -8: "LMOE_ERR_OUT_OF_MEMORY", -9: "LMOE_ERR_MISALIGNED"}
EXPORTED = ("lmoe_create", "lmoe_load_weights", "lmoe_route", "lmoe_forward",
            "lmoe_forward_host", "lmoe_forward_host_batches", "lmoe_get_dims",
            "lmoe_device_status", "lmoe_debug_buffer", "lmoe_profile", "lmoe_stage_times", "lmoe_dispatch_noalloc",
            "lmoe_selftest_wait_timeout", "lmoe_backward", "lmoe_ep_dispatch", "lmoe_ep_experts",
            "lmoe_ep_combine", "lmoe_strerror", "lmoe_destroy")
LMOE_NUM_STAGES = 8
STAGE_NAMES = ("x_gemm_router_down", "topk", "dispatch", "permute_z",
               "expert_gate_up_gemm", "expert_down_gemm", "combine", "out_gemm")


class lmoe_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "d", "m", "n_experts", "top_k", "alpha", "n_shared", "m_shared", "variant", "dtype",
        "n_routed_override", "top_k_override", "has_router_bias", "max_tokens", "activation",
        "training", "weight_format", "ep_rank", "ep_world")]


class lmoe_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "w_router", "b_router", "w_down", "w_up", "w_gate", "w_upx", "w_out", "s_gate",
        "s_up", "s_out")]


GRAD_NAMES = ("w_router", "b_router", "w_down", "w_up", "w_gate", "w_upx", "w_out", "s_gate",
              "s_up", "s_out")


class lmoe_grads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in GRAD_NAMES]


P, I32 = C.c_void_p, C.c_int32
_lib.lmoe_create.argtypes = [C.POINTER(lmoe_config), C.POINTER(C.c_void_p)]
_lib.lmoe_load_weights.argtypes = [P, C.POINTER(lmoe_weights), P]
_lib.lmoe_route.argtypes = [P, P, I32, P, P, P, P, P]
_lib.lmoe_forward.argtypes = [P, P, P, I32, P]
_lib.lmoe_forward_host.argtypes = [P, P, P, I32, P]
_lib.lmoe_forward_host_batches.argtypes = [P, I32, C.POINTER(C.c_void_p),
                                            C.POINTER(C.c_void_p), I32, P]
_lib.lmoe_get_dims.argtypes = [P, C.POINTER(I32), C.POINTER(I32), C.POINTER(I32)]
_lib.lmoe_device_status.argtypes = [P, P]
_lib.lmoe_debug_buffer.argtypes = [P, I32, C.POINTER(C.c_void_p), C.POINTER(C.c_int64)]
_lib.lmoe_profile.argtypes = [P, I32]
_lib.lmoe_stage_times.argtypes = [P, C.POINTER(C.c_float), I32, C.POINTER(I32),
                                  C.POINTER(C.c_int64)]
_lib.lmoe_dispatch_noalloc.argtypes = [P, I32, I32, I32, P, P, P]
_lib.lmoe_selftest_wait_timeout.argtypes = [P, C.c_int64, P]
_lib.lmoe_backward.argtypes = [P, P, P, P, C.POINTER(lmoe_grads), I32, P]
_lib.lmoe_ep_dispatch.argtypes = [P, P, I32, P, P, P]
_lib.lmoe_ep_experts.argtypes = [P, P, P, I32, P, P]
_lib.lmoe_ep_combine.argtypes = [P, P, P, I32, P]
_lib.lmoe_strerror.argtypes = [C.c_int]
_lib.lmoe_strerror.restype = C.c_char_p
_lib.lmoe_destroy.argtypes = [P]
for _n in EXPORTED:
    if _n != "lmoe_strerror":
        getattr(_lib, _n).restype = C.c_int


class LmoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({lmoe_strerror(code)})")


def _check(rc: int, what: str):
    if rc != 0:
        raise LmoeError(rc, what)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t)


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def library_path() -> str:
    return _LIB_PATH


def lmoe_strerror(code: int) -> str:
    return _lib.lmoe_strerror(code).decode()


def config_from(cfg: LayerConfig, max_tokens: int | None = None,
                training: bool = False, ep_rank: int = 0, ep_world: int = 0) -> lmoe_config:
    return lmoe_config(
        d=cfg.d, m=cfg.m, n_experts=cfg.n_experts, top_k=cfg.top_k, alpha=cfg.alpha,
        n_shared=cfg.n_shared, m_shared=cfg.m_shared,
        variant=LMOE_ACC if cfg.variant == "acc" else LMOE_EFF,
        dtype=LMOE_BF16 if cfg.dtype == "bf16" else LMOE_F32,
        n_routed_override=cfg.n_routed_override, top_k_override=cfg.top_k_override,
        has_router_bias=int(cfg.has_router_bias),
        max_tokens=cfg.T if max_tokens is None else max_tokens,
        activation=LMOE_RELU2 if cfg.activation == "relu2" else LMOE_SWIGLU,
        training=int(training),
        weight_format={"fp8": LMOE_WEIGHTS_FP8, "nvfp4": LMOE_WEIGHTS_NVFP4}.get(
            cfg.weights, LMOE_WEIGHTS_BF16),
        ep_rank=ep_rank, ep_world=ep_world)


def lmoe_create(config: lmoe_config) -> int:
    h = C.c_void_p()
    _check(_lib.lmoe_create(C.byref(config), C.byref(h)), "lmoe_create")
    return h.value


def lmoe_load_weights(handle: int, weights: dict, stream=None) -> None:
    w = lmoe_weights(**{k: _ptr(weights.get(k)) for k, _ in lmoe_weights._fields_})
    _check(_lib.lmoe_load_weights(handle, C.byref(w), _stream(stream)), "lmoe_load_weights")


def lmoe_route(handle: int, x, T: int, ids=None, gates=None, offsets=None, perm=None,
               stream=None) -> None:
    _check(_lib.lmoe_route(handle, _ptr(x), T, _ptr(ids), _ptr(gates), _ptr(offsets),
                           _ptr(perm), _stream(stream)), "lmoe_route")


def lmoe_forward(handle: int, x, y, T: int, stream=None) -> None:
    _check(_lib.lmoe_forward(handle, _ptr(x), _ptr(y), T, _stream(stream)), "lmoe_forward")


def lmoe_forward_host(handle: int, x_host, y_host, T: int, stream=None) -> None:
    _check(_lib.lmoe_forward_host(handle, _ptr(x_host), _ptr(y_host), T, _stream(stream)),
           "lmoe_forward_host")


def lmoe_forward_host_batches(handle: int, x_hosts, y_hosts, T: int, stream=None) -> None:
    """x_hosts, y_hosts: equal-length sequences of host tensors ([T][d] each)."""
    if len(x_hosts) != len(y_hosts):
        raise ValueError("x_hosts and y_hosts differ in length")
    n = len(x_hosts)
    xs = (C.c_void_p * max(n, 1))(*[_ptr(t) for t in x_hosts])
    ys = (C.c_void_p * max(n, 1))(*[_ptr(t) for t in y_hosts])
    _check(_lib.lmoe_forward_host_batches(handle, n, xs, ys, T, _stream(stream)),
           "lmoe_forward_host_batches")


def lmoe_get_dims(handle: int):
    l, n, k = I32(), I32(), I32()
    _check(_lib.lmoe_get_dims(handle, C.byref(l), C.byref(n), C.byref(k)), "lmoe_get_dims")
    return l.value, n.value, k.value


def lmoe_device_status(handle: int, stream=None) -> int:
    return _lib.lmoe_device_status(handle, _stream(stream))


def lmoe_debug_buffer(handle: int, which: int):
    p, n = C.c_void_p(), C.c_int64()
    _check(_lib.lmoe_debug_buffer(handle, which, C.byref(p), C.byref(n)), "lmoe_debug_buffer")
    return p.value, n.value


def lmoe_profile(handle: int, slots: int) -> None:
    _check(_lib.lmoe_profile(handle, int(slots)), "lmoe_profile")


def lmoe_stage_times(handle: int):
    """(per-stage ms summed over the profiled forwards, their count, launches)."""
    ms = (C.c_float * LMOE_NUM_STAGES)()
    nf = I32()
    n = C.c_int64()
    _check(_lib.lmoe_stage_times(handle, ms, LMOE_NUM_STAGES, C.byref(nf), C.byref(n)),
           "lmoe_stage_times")
    return list(ms), nf.value, n.value


def lmoe_launches(handle: int) -> int:
    n = C.c_int64()
    _check(_lib.lmoe_stage_times(handle, None, 0, None, C.byref(n)), "lmoe_stage_times")
    return n.value


def lmoe_dispatch_noalloc(ids, T: int, k_active: int, n_routed: int, offsets, perm,
                          stream=None) -> None:
    """Dispatch with no allocation (see include/lmoe.h); for callers that may
    not allocate device memory where they run it."""
    _check(_lib.lmoe_dispatch_noalloc(_ptr(ids), T, k_active, n_routed, _ptr(offsets),
                                      _ptr(perm), _stream(stream)), "lmoe_dispatch_noalloc")


def lmoe_selftest_wait_timeout(handle: int, limit_ns: int, stream=None) -> None:
    _check(_lib.lmoe_selftest_wait_timeout(handle, int(limit_ns), _stream(stream)),
           "lmoe_selftest_wait_timeout")


def lmoe_backward(handle: int, x, dy, dx, grads: dict, T: int, stream=None) -> None:
    """dx and the weight gradients (dict of float32 device tensors named as
    GRAD_NAMES; absent names pass NULL) for the cotangent dy of layer(x)."""
    g = lmoe_grads(**{k: _ptr(grads.get(k)) for k in GRAD_NAMES})
    _check(_lib.lmoe_backward(handle, _ptr(x), _ptr(dy), _ptr(dx), C.byref(g), T,
                              _stream(stream)), "lmoe_backward")


def lmoe_ep_dispatch(handle: int, x, T: int, send_rows, expert_counts, stream=None) -> None:
    _check(_lib.lmoe_ep_dispatch(handle, _ptr(x), T, _ptr(send_rows), _ptr(expert_counts),
                                 _stream(stream)), "lmoe_ep_dispatch")


def lmoe_ep_experts(handle: int, recv_rows, recv_counts, R: int, out_rows, stream=None) -> None:
    _check(_lib.lmoe_ep_experts(handle, _ptr(recv_rows), _ptr(recv_counts), R, _ptr(out_rows),
                                _stream(stream)), "lmoe_ep_experts")


def lmoe_ep_combine(handle: int, back_rows, y, T: int, stream=None) -> None:
    _check(_lib.lmoe_ep_combine(handle, _ptr(back_rows), _ptr(y), T, _stream(stream)),
           "lmoe_ep_combine")


def lmoe_destroy(handle: int) -> None:
    _check(_lib.lmoe_destroy(handle), "lmoe_destroy")


class LatentMoELayer:
    """Convenience owner of one handle: create, load weights, forward.

    Keeps the handle alive and destroys it with the object; every call goes
    straight through the C ABI above.
    """

    def __init__(self, cfg: LayerConfig, weights: dict, max_tokens: int | None = None,
                 stream=None, training: bool = False, ep_rank: int = 0, ep_world: int = 0):
        """ep_world > 1: an expert-parallel rank (see lmoe_ep_dispatch) holding
        experts [ep_rank * N'/ep_world, (ep_rank + 1) * N'/ep_world) of the full
        expert weights in ``weights``."""
        self.cfg = cfg
        self.ep_rank, self.ep_world = ep_rank, ep_world
        self.handle = lmoe_create(config_from(cfg, max_tokens, training, ep_rank, ep_world))
        if ep_world > 1:
            nl = cfg.n_routed // ep_world
            weights = dict(weights)
            for k in ("w_gate", "w_upx", "w_out"):
                if weights.get(k) is not None:
                    weights[k] = weights[k][ep_rank * nl:(ep_rank + 1) * nl]
        try:
            lmoe_load_weights(self.handle, weights, stream)
        except Exception:
            lmoe_destroy(self.handle)
            self.handle = None
            raise
        self.l, self.n_routed, self.k_active = lmoe_get_dims(self.handle)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None):
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        lmoe_forward(self.handle, x, y, T, stream)
        return y

    def grad_shapes(self) -> dict:
        c = self.cfg
        N, d, l, m, ns, ms = self.n_routed, c.d, self.l, c.m, c.n_shared, c.m_shared
        shapes = {"w_router": (N, d), "w_down": (l, d), "w_up": (d, l), "w_upx": (N, m, l),
                  "w_out": (N, l, m)}
        if c.activation != "relu2":
            shapes["w_gate"] = (N, m, l)
        if c.has_router_bias:
            shapes["b_router"] = (N,)
        if ns > 0:
            shapes.update(s_up=(ns, ms, d), s_out=(ns, d, ms))
            if c.activation != "relu2":
                shapes["s_gate"] = (ns, ms, d)
        return shapes

    def backward(self, x: torch.Tensor, dy: torch.Tensor, stream=None):
        """(dx, dict of float32 weight gradients) for the cotangent dy."""
        T = x.shape[0]
        dx = torch.empty_like(x)
        grads = {k: torch.empty(v, dtype=torch.float32, device=x.device)
                 for k, v in self.grad_shapes().items()}
        lmoe_backward(self.handle, x, dy, dx, grads, T, stream)
        return dx, grads

    def route(self, x: torch.Tensor, stream=None):
        T = x.shape[0]
        dev = x.device
        ids = torch.empty((T, self.k_active), dtype=torch.int32, device=dev)
        gates = torch.empty((T, self.k_active), dtype=torch.float32, device=dev)
        offsets = torch.empty((self.n_routed + 1,), dtype=torch.int32, device=dev)
        perm = torch.empty((T * self.k_active,), dtype=torch.int32, device=dev)
        lmoe_route(self.handle, x, T, ids, gates, offsets, perm, stream)
        return ids, gates, offsets, perm

    def debug_tensor(self, which: int, dtype: torch.dtype, shape) -> torch.Tensor:
        """A copy of one internal buffer (test hook; see lmoe_debug_buffer)."""
        ptr, numel = lmoe_debug_buffer(self.handle, which)
        return device_view(ptr, numel, dtype, shape).clone()

    def close(self):
        if getattr(self, "handle", None):
            lmoe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_TYPESTR = {torch.float32: "<f4", torch.bfloat16: "<u2", torch.int32: "<i4", torch.uint8: "|u1"}


def device_view(ptr: int, numel: int, dtype: torch.dtype, shape) -> torch.Tensor:
    """Zero-copy torch view of `numel` elements at a device address."""
    n = 1
    for s in shape:
        n *= s
    if n > numel:
        raise ValueError("view larger than the buffer")
    holder = type("_DevBuf", (), {})()
    holder.__cuda_array_interface__ = {"shape": (n,), "typestr": _TYPESTR[dtype],
                                       "data": (ptr, False), "version": 3}
    t = torch.as_tensor(holder, device="cuda")
    if dtype == torch.bfloat16:
        t = t.view(torch.bfloat16)
    return t.view(*shape)
