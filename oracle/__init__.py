"""ctypes binding of the fp64 CPU oracle (``oracle/lmoe_oracle.c``): the
LatentMoE layer forward and its backward.

TEST INFRASTRUCTURE ONLY.  The oracle is what the CUDA library is checked
against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package; the product path never
does, and the oracle never imports the product package.

Every array is numpy.  x and all weights share one element type: float32,
float64, or bf16 given as its raw uint16 bit pattern (a bf16 value is the top
half of an IEEE float32, so widening is exact).  The router bias is float64.

Functions whose parity is "unpinned" (no printed value or closed form checks
them by themselves): none -- every step is pinned by tests/test_oracle_pins.py
through brute force, closed forms, hand-derived golden cases and invariants;
full-size outputs are pinned only through those properties, since the pages
print no worked numeric example of the layer.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lmoe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblmoe_oracle.so")
_lock = threading.Lock()
_lib = None

ODT_F32, ODT_BF16, ODT_F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (ISO C11: no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
               "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


class _Layer(C.Structure):
    _fields_ = [
        ("d", C.c_int32), ("l", C.c_int32), ("m", C.c_int32),
        ("n_routed", C.c_int32), ("k_active", C.c_int32),
        ("n_shared", C.c_int32), ("m_shared", C.c_int32), ("dtype", C.c_int32),
        ("activation", C.c_int32),
        ("w_router", C.c_void_p), ("b_router", C.c_void_p),
        ("w_down", C.c_void_p), ("w_up", C.c_void_p),
        ("w_gate", C.c_void_p), ("w_upx", C.c_void_p), ("w_out", C.c_void_p),
        ("s_gate", C.c_void_p), ("s_up", C.c_void_p), ("s_out", C.c_void_p),
        ("act_quant", C.c_int32),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P, I64, I32 = C.c_void_p, C.c_int64, C.c_int
            lib.oracle_router_logits.argtypes = [P, P, I64, P]
            lib.oracle_router_logits.restype = None
            lib.oracle_select.argtypes = [P, I64, I32, I32, P, P]
            lib.oracle_select.restype = C.c_int
            lib.oracle_gates.argtypes = [P, I64, I32, I32, P, P]
            lib.oracle_gates.restype = C.c_int
            lib.oracle_forward.argtypes = [P, P, I64, P, I64, P, P, P, P]
            lib.oracle_forward.restype = C.c_int
            lib.oracle_dispatch.argtypes = [P, I64, I32, I32, P, P, P]
            lib.oracle_dispatch.restype = C.c_int
            lib.oracle_down.argtypes = [P, P, I64, P]
            lib.oracle_down.restype = None
            lib.oracle_expert.argtypes = [P, I32, P, P]
            lib.oracle_expert.restype = None
            lib.oracle_up.argtypes = [P, P, P]
            lib.oracle_up.restype = None
            lib.oracle_shared.argtypes = [P, P, I64, P]
            lib.oracle_shared.restype = None
            lib.oracle_backward.argtypes = [P, P, I64, P, I64, P, P, P]
            lib.oracle_backward.restype = C.c_int
            lib.oracle_fp8_rows.argtypes = [P, I32, I64, I32, P, P]
            lib.oracle_fp8_rows.restype = None
            lib.oracle_nvfp4_rows.argtypes = [P, I32, I64, I32, P, P, P]
            lib.oracle_nvfp4_rows.restype = I32
            lib.oracle_threads.argtypes = []
            lib.oracle_threads.restype = C.c_int
            _lib = lib
    return _lib


def _swap_library(path: str | None):
    """Point the wrapper at another build of the oracle (used by the mutation
    test, which compiles deliberately broken copies); returns the previous
    library handle.  ``None`` restores lazy loading of the real oracle."""
    global _lib
    with _lock:
        old = _lib
        _lib = None
    if path is not None:
        saved = globals()["build"]
        globals()["build"] = lambda force=False: path
        try:
            _load()
        finally:
            globals()["build"] = saved
    return old


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return ODT_F32
    if a.dtype == np.uint16:
        return ODT_BF16
    if a.dtype == np.float64:
        return ODT_F64
    raise TypeError(f"oracle takes float32, float64 or bf16-as-uint16, got {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data


class Layer:
    """A LatentMoE layer's weights, in nn.Linear [out][in] layout.

    w_router [N'][d], b_router [N'] (float64) or None, w_down [l][d],
    w_up [d][l], w_gate / w_upx [N'][m][l], w_out [N'][l][m],
    s_gate / s_up [n_s][m_s][d], s_out [n_s][d][m_s].
    activation "swiglu" (three matrices) or "relu2" (squared ReLU, two
    matrices: w_upx / s_up are the up-projections; w_gate / s_gate unused).
    act_fp8: the routed experts multiply E4M3 activations -- each token's z
    and each expert's hidden vector quantised with the weight rows' rule (a
    power-of-two scale, the smallest that brings the largest magnitude
    within 448); the backward is then not defined.
    act_fp4: the same with NVFP4 activations (nvfp4_rows' rule: E2M1 codes,
    an E4M3 scale per 16 elements, a power-of-two row scale); l and m must
    be multiples of 16.
    act_bf16: the quantised rows are rounded to bf16 first, as a bf16 layer
    always does (for a float64 layer standing for a bf16 one).
    """

    def __init__(self, *, w_router, b_router, w_down, w_up, w_gate, w_upx,
                 w_out, s_gate, s_up, s_out, k_active, activation="swiglu",
                 act_fp8=False, act_fp4=False, act_bf16=False):
        if act_fp8 and act_fp4:
            raise ValueError("act_fp8 and act_fp4 are exclusive")
        if activation not in ("swiglu", "relu2"):
            raise ValueError("activation must be 'swiglu' or 'relu2'")
        self.activation = activation
        if activation == "relu2":   # two matrices: the gate weights are unused
            w_gate = w_upx if w_gate is None else w_gate
            s_gate = s_up if s_gate is None else s_gate
        arrs = dict(w_router=w_router, w_down=w_down, w_up=w_up, w_gate=w_gate,
                    w_upx=w_upx, w_out=w_out, s_gate=s_gate, s_up=s_up, s_out=s_out)
        self._keep = {k: np.ascontiguousarray(v) for k, v in arrs.items()}
        codes = {_dtype_code(v) for v in self._keep.values()}
        if len(codes) != 1:
            raise TypeError("all weights must share one element type")
        self.dtype = codes.pop()
        self.b_router = None if b_router is None else np.ascontiguousarray(
            b_router, dtype=np.float64)
        N, d = self._keep["w_router"].shape
        l = self._keep["w_down"].shape[0]
        m = self._keep["w_gate"].shape[1]
        ns, ms = self._keep["s_gate"].shape[0], self._keep["s_gate"].shape[1]
        self.d, self.l, self.m, self.N, self.K, self.n_s, self.m_s = d, l, m, N, k_active, ns, ms
        assert self._keep["w_down"].shape == (l, d)
        assert self._keep["w_up"].shape == (d, l)
        assert self._keep["w_gate"].shape == (N, m, l)
        assert self._keep["w_upx"].shape == (N, m, l)
        assert self._keep["w_out"].shape == (N, l, m)
        assert self._keep["s_up"].shape == (ns, ms, d)
        assert self._keep["s_out"].shape == (ns, d, ms)
        k = self._keep
        self._c = _Layer(d, l, m, N, k_active, ns, ms, self.dtype,
                         1 if activation == "relu2" else 0,
                         _ptr(k["w_router"]), _ptr(self.b_router), _ptr(k["w_down"]),
                         _ptr(k["w_up"]), _ptr(k["w_gate"]), _ptr(k["w_upx"]),
                         _ptr(k["w_out"]), _ptr(k["s_gate"]), _ptr(k["s_up"]),
                         _ptr(k["s_out"]),
                         (1 if act_fp8 else (2 if act_fp4 else 0)) | (16 if act_bf16 else 0))
        self.act_fp8 = bool(act_fp8)
        self.act_fp4 = bool(act_fp4)

    @property
    def cref(self):
        return C.byref(self._c)

    def _x(self, x):
        x = np.ascontiguousarray(x)
        if _dtype_code(x) != self.dtype:
            raise TypeError("x must have the weights' element type")
        assert x.ndim == 2 and x.shape[1] == self.d
        return x


def router_logits(layer: Layer, x) -> np.ndarray:
    """s[t][e] = x_t . W_r[e] (+ b_e), fp64."""
    x = layer._x(x)
    s = np.empty((x.shape[0], layer.N), dtype=np.float64)
    _load().oracle_router_logits(layer.cref, _ptr(x), x.shape[0], _ptr(s))
    return s


def select(logits: np.ndarray, k: int):
    """Top-k of each row by (logit desc, index asc); gates = softmax renormalised."""
    s = np.ascontiguousarray(logits, dtype=np.float64)
    T, N = s.shape
    ids = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float64)
    if _load().oracle_select(_ptr(s), T, N, k, _ptr(ids), _ptr(g)) != 0:
        raise ValueError("k must be in [1, N']")
    return ids, g


def gates_for_ids(logits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Gates of given selections: softmax at ``ids`` renormalised over them (fp64)."""
    s = np.ascontiguousarray(logits, dtype=np.float64)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, N = s.shape
    assert ids.shape[0] == T
    k = ids.shape[1]
    g = np.empty((T, k), dtype=np.float64)
    rc = _load().oracle_gates(_ptr(s), T, N, k, _ptr(ids), _ptr(g))
    if rc != 0:
        raise ValueError("k must be in [1, N'] and every id in [0, N')")
    return g


def forward(layer: Layer, x, tokens=None, ids=None):
    """y for the listed tokens (all if None); ids given -> forward_given_ids.

    Returns (y [n][d] f64, ids [n][K'] int32, gates [n][K'] f64).
    """
    x = layer._x(x)
    T = x.shape[0]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = T if tok is None else tok.shape[0]
    ids_in = None
    if ids is not None:
        ids_in = np.ascontiguousarray(ids, dtype=np.int32)
        assert ids_in.shape == (T, layer.K)
    y = np.empty((n, layer.d), dtype=np.float64)
    ids_out = np.empty((n, layer.K), dtype=np.int32)
    g_out = np.empty((n, layer.K), dtype=np.float64)
    rc = _load().oracle_forward(layer.cref, _ptr(x), T, _ptr(tok), n, _ptr(ids_in),
                                _ptr(y), _ptr(ids_out), _ptr(g_out))
    if rc != 0:
        raise ValueError(f"oracle_forward failed ({rc})")
    return y, ids_out, g_out


def dispatch(ids: np.ndarray, n_routed: int):
    """(offsets [N'+1], perm [T*K'], pos [T*K']) -- grouping by expert, token order."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, K = ids.shape
    offsets = np.empty(n_routed + 1, dtype=np.int32)
    perm = np.empty(T * K, dtype=np.int32)
    pos = np.empty(T * K, dtype=np.int32)
    if _load().oracle_dispatch(_ptr(ids), T, K, n_routed, _ptr(offsets), _ptr(perm),
                               _ptr(pos)) != 0:
        raise ValueError("ids outside [0, N')")
    return offsets, perm, pos


def down(layer: Layer, x, t: int) -> np.ndarray:
    x = layer._x(x)
    z = np.empty(layer.l, dtype=np.float64)
    _load().oracle_down(layer.cref, _ptr(x), t, _ptr(z))
    return z


def expert(layer: Layer, e: int, z) -> np.ndarray:
    z = np.ascontiguousarray(z, dtype=np.float64)
    out = np.empty(layer.l, dtype=np.float64)
    _load().oracle_expert(layer.cref, e, _ptr(z), _ptr(out))
    return out


def up(layer: Layer, u) -> np.ndarray:
    u = np.ascontiguousarray(u, dtype=np.float64)
    out = np.empty(layer.d, dtype=np.float64)
    _load().oracle_up(layer.cref, _ptr(u), _ptr(out))
    return out


def shared(layer: Layer, x, t: int) -> np.ndarray:
    x = layer._x(x)
    out = np.empty(layer.d, dtype=np.float64)
    _load().oracle_shared(layer.cref, _ptr(x), t, _ptr(out))
    return out


class _Grads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "dx", "w_router", "b_router", "w_down", "w_up", "w_gate", "w_upx", "w_out",
        "s_gate", "s_up", "s_out")]


GRAD_NAMES = ("w_router", "b_router", "w_down", "w_up", "w_gate", "w_upx", "w_out",
              "s_gate", "s_up", "s_out")


def backward(layer: Layer, x, dy, tokens=None, ids=None, want=GRAD_NAMES):
    """Gradients of the layer output for the cotangent dy (fp64).

    dy [n][d] holds the cotangent of the listed tokens' outputs (all tokens if
    tokens is None).  Weight gradients sum the listed tokens' contributions.
    ids as in forward().  Returns a dict: "dx" [n][d] and each name in want
    (weight-gradient arrays in the weights' shapes).
    """
    x = layer._x(x)
    T = x.shape[0]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n = T if tok is None else tok.shape[0]
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    assert dy.shape == (n, layer.d)
    ids_in = None
    if ids is not None:
        ids_in = np.ascontiguousarray(ids, dtype=np.int32)
        assert ids_in.shape == (T, layer.K)
    shapes = {"w_router": (layer.N, layer.d), "b_router": (layer.N,),
              "w_down": (layer.l, layer.d), "w_up": (layer.d, layer.l),
              "w_gate": (layer.N, layer.m, layer.l), "w_upx": (layer.N, layer.m, layer.l),
              "w_out": (layer.N, layer.l, layer.m),
              "s_gate": (layer.n_s, layer.m_s, layer.d), "s_up": (layer.n_s, layer.m_s, layer.d),
              "s_out": (layer.n_s, layer.d, layer.m_s)}
    out = {"dx": np.empty((n, layer.d), dtype=np.float64)}
    for k in want:
        out[k] = np.zeros(shapes[k], dtype=np.float64)
    g = _Grads(*[_ptr(out.get(k)) for k in ("dx",) + GRAD_NAMES])
    rc = _load().oracle_backward(layer.cref, _ptr(x), T, _ptr(tok), n, _ptr(ids_in),
                                 _ptr(dy), C.byref(g))
    if rc != 0:
        raise ValueError(f"oracle_backward failed ({rc})")
    return out


def fp8_rows(w):
    """Row-wise E4M3 quantisation with power-of-two scales (see the C source):
    returns (W' dequantised, float64, same shape; scales [rows])."""
    w = np.ascontiguousarray(w)
    code = _dtype_code(w)
    cols = w.shape[-1]
    rows = w.size // cols
    wq = np.empty(w.shape, dtype=np.float64)
    sc = np.empty(rows, dtype=np.float64)
    _load().oracle_fp8_rows(_ptr(w), code, rows, cols, _ptr(wq), _ptr(sc))
    return wq, sc


def nvfp4_rows(w):
    """Row-wise NVFP4 quantisation (E2M1 codes, an E4M3 scale per 16
    elements, a power-of-two row scale; see the C source): returns (W'
    dequantised, float64, same shape; row scales [rows]; block scales, the
    shape of W with cols/16 in place of cols)."""
    w = np.ascontiguousarray(w)
    code = _dtype_code(w)
    cols = w.shape[-1]
    if cols % 16:
        raise ValueError("NVFP4 rows need a multiple of 16 columns")
    rows = w.size // cols
    wq = np.empty(w.shape, dtype=np.float64)
    sc = np.empty(rows, dtype=np.float64)
    bs = np.empty(w.shape[:-1] + (cols // 16,), dtype=np.float64)
    rc = _load().oracle_nvfp4_rows(_ptr(w), code, rows, cols, _ptr(wq), _ptr(sc), _ptr(bs))
    if rc != 0:
        raise ValueError(f"oracle_nvfp4_rows failed ({rc})")
    return wq, sc, bs


def threads() -> int:
    return int(_load().oracle_threads())
