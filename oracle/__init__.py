"""fp64 CPU oracle for the fused SwiGLU gate/up projection and dSwiGLU.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product library never imports it, and this package imports nothing from the
product: the two share only the seeded input generators, which hold none of
the method's arithmetic.

The arithmetic lives in ``swiglu_oracle.c`` (plain C, IEEE double, no
fast-math, no FMA contraction); this module compiles it with gcc and wraps it
with numpy arrays through ctypes.  See the C file's header for what is
computed and which page passage each part follows.

``Oracle(path)`` wraps any build of that source; the module-level functions
use the default build ``liboracle.so`` next to this file.  Tests use a second
instance to load copies of the source with a mistake planted in them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "swiglu_oracle.c")
LIB_PATH = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-std=c11"]

_lock = threading.Lock()
_default = None


def compile_source(src: str, out: str) -> str:
    """gcc-compile one oracle C source file into a shared library."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, src, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``swiglu_oracle.c`` into ``liboracle.so`` if it is missing or
    older than the source.  Returns the library path."""
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SOURCE)):
        return LIB_PATH
    return compile_source(SOURCE, LIB_PATH)


_D = ctypes.c_double
_I64 = ctypes.c_int64
_P = ctypes.c_void_p


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_bits(a) -> np.ndarray:
    """bf16 operand as a contiguous uint16 array of its bit patterns.  Accepts
    a numpy uint16 array or a CPU torch.bfloat16 tensor."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16, a.dtype
        return np.ascontiguousarray(a)
    import torch  # only for tensor inputs
    assert a.dtype == torch.bfloat16 and a.device.type == "cpu"
    return a.contiguous().view(torch.int16).numpy().view(np.uint16)


def _as_f32(a) -> np.ndarray:
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a, dtype=np.float32)
    import torch
    assert a.dtype == torch.float32 and a.device.type == "cpu"
    return a.contiguous().numpy()


class Oracle:
    """ctypes wrapper of one build of the oracle's C source."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        for name in ("oracle_sigmoid", "oracle_silu", "oracle_dsilu", "oracle_gelu_tanh",
                     "oracle_dgelu_tanh"):
            f = getattr(lib, name)
            f.restype = _D
            f.argtypes = [_D]
        for name in ("oracle_act", "oracle_dact"):
            f = getattr(lib, name)
            f.restype = _D
            f.argtypes = [_D, ctypes.c_int]
        lib.oracle_swiglu_fwd_act_f64.restype = None
        lib.oracle_swiglu_fwd_act_f64.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _D,
                                                  _P, _P, _P, _P, _P]
        lib.oracle_swiglu_fwd_points_act.restype = ctypes.c_int
        lib.oracle_swiglu_fwd_points_act.argtypes = [ctypes.c_int, _P, _P, _P, _I64, _P, _P, _I64,
                                                     ctypes.c_int, _D, _P, _P, _P, _P, _P]
        lib.oracle_dswiglu_act_f64.restype = None
        lib.oracle_dswiglu_act_f64.argtypes = [_P, _P, _P, _I64, ctypes.c_int, _D, _P, _P]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_int]
        lib.oracle_e4m3_encode.restype = ctypes.c_int
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        lib.oracle_ue8m0_exponent.restype = ctypes.c_int
        lib.oracle_ue8m0_exponent.argtypes = [ctypes.c_double]
        lib.oracle_quant_e4m3.restype = None
        lib.oracle_quant_e4m3.argtypes = [_P, _I64, _I64, _P, _P]
        lib.oracle_bwd_dx_f64.restype = None
        lib.oracle_bwd_dx_f64.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _P]
        lib.oracle_bwd_dw_f64.restype = None
        lib.oracle_bwd_dw_f64.argtypes = [_P, _P, _P, _I64, _I64, _I64, _P, _P]
        for name in ("oracle_bf16_to_f64", "oracle_f32_to_f64"):
            f = getattr(lib, name)
            f.restype = None
            f.argtypes = [_P, _P, _I64]
        lib.oracle_swiglu_fwd_f64.restype = None
        lib.oracle_swiglu_fwd_f64.argtypes = [_P, _P, _P, _I64, _I64, _I64,
                                              _P, _P, _P, _P, _P]
        lib.oracle_swiglu_fwd_points_f64.restype = None
        for name in ("oracle_swiglu_fwd_points_f64",
                     "oracle_swiglu_fwd_points_bf16",
                     "oracle_swiglu_fwd_points_f32"):
            getattr(lib, name).argtypes = [_P, _P, _P, _I64, _P, _P, _I64,
                                           _P, _P, _P, _P, _P]
        lib.oracle_swiglu_fwd_points_bf16.restype = ctypes.c_int
        lib.oracle_swiglu_fwd_points_f32.restype = ctypes.c_int
        for name in ("oracle_dswiglu_f64", "oracle_dswiglu_bf16",
                     "oracle_dswiglu_f32"):
            f = getattr(lib, name)
            f.restype = None
            f.argtypes = [_P, _P, _P, _I64, _P, _P]
        self.lib = lib
        self.path = lib_path

    # ---- scalar definitions ---------------------------------------------------
    def sigmoid(self, x: float) -> float:
        return self.lib.oracle_sigmoid(float(x))

    def silu(self, x: float) -> float:
        return self.lib.oracle_silu(float(x))

    def dsilu(self, x: float) -> float:
        return self.lib.oracle_dsilu(float(x))

    def gelu_tanh(self, x: float) -> float:
        return self.lib.oracle_gelu_tanh(float(x))

    def dgelu_tanh(self, x: float) -> float:
        return self.lib.oracle_dgelu_tanh(float(x))

    def act(self, x: float, act: int) -> float:
        """Activation code 0 = SiLU, 1 = GELU(tanh)."""
        return self.lib.oracle_act(float(x), int(act))

    def dact(self, x: float, act: int) -> float:
        return self.lib.oracle_dact(float(x), int(act))

    # ---- decoding ------------------------------------------------------------
    def decode_bf16(self, a) -> np.ndarray:
        """Exact float64 values of bf16 bit patterns (the oracle's decoder)."""
        bits = _as_bits(a)
        out = np.empty(bits.shape, dtype=np.float64)
        self.lib.oracle_bf16_to_f64(_ptr(bits), _ptr(out), bits.size)
        return out

    def decode(self, a, dtype: str) -> np.ndarray:
        if dtype == "bf16":
            return self.decode_bf16(a)
        if dtype != "f32":
            raise ValueError(dtype)
        f = _as_f32(a)
        out = np.empty(f.shape, dtype=np.float64)
        self.lib.oracle_f32_to_f64(_ptr(f), _ptr(out), f.size)
        return out

    # ---- forward ---------------------------------------------------------------
    def swiglu_fwd_f64(self, X, Wg, Wu, want_magnitudes: bool = False, act: int = 0,
                       alpha: float = 1.0):
        """Full forward on float64 operands X [M,K], Wg/Wu [N,K]:
        H = act(alpha * G) * U (act 0 = SiLU, 1 = GELU(tanh)).

        Returns a dict with G, U, H (float64 [M,N]) and, if asked,
        AG = sum_k |x wg| and AU = sum_k |x wu| (error-bound magnitudes)."""
        X = np.ascontiguousarray(X, dtype=np.float64)
        Wg = np.ascontiguousarray(Wg, dtype=np.float64)
        Wu = np.ascontiguousarray(Wu, dtype=np.float64)
        M, K = X.shape
        N = Wg.shape[0]
        assert Wg.shape == (N, K) and Wu.shape == (N, K)
        out = {k: np.empty((M, N), dtype=np.float64) for k in ("G", "U", "H")}
        if want_magnitudes:
            out["AG"] = np.empty((M, N), dtype=np.float64)
            out["AU"] = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_swiglu_fwd_act_f64(
            _ptr(X), _ptr(Wg), _ptr(Wu), M, K, N, int(act), float(alpha), _ptr(out["G"]),
            _ptr(out["U"]), _ptr(out["H"]),
            _ptr(out["AG"]) if want_magnitudes else None,
            _ptr(out["AU"]) if want_magnitudes else None)
        return out

    def swiglu_fwd(self, X, Wg, Wu, dtype: str = "bf16",
                   want_magnitudes: bool = False, act: int = 0, alpha: float = 1.0):
        """Full forward from bf16 (uint16 bits / torch.bfloat16) or fp32."""
        return self.swiglu_fwd_f64(self.decode(X, dtype), self.decode(Wg, dtype),
                                   self.decode(Wu, dtype), want_magnitudes, act, alpha)

    def swiglu_fwd_points(self, X, Wg, Wu, idx_m, idx_n, dtype: str = "bf16",
                          act: int = 0, alpha: float = 1.0):
        """Forward at the sampled outputs (idx_m[i], idx_n[i]) only, straight
        from the stored operands.  Returns float64 vectors G, U, H, AG, AU."""
        idx_m = np.ascontiguousarray(idx_m, dtype=np.int64)
        idx_n = np.ascontiguousarray(idx_n, dtype=np.int64)
        count = idx_m.size
        assert idx_n.size == count
        if dtype == "bf16":
            Xa, Wga, Wua = _as_bits(X), _as_bits(Wg), _as_bits(Wu)
            fn = self.lib.oracle_swiglu_fwd_points_bf16
        elif dtype == "f32":
            Xa, Wga, Wua = _as_f32(X), _as_f32(Wg), _as_f32(Wu)
            fn = self.lib.oracle_swiglu_fwd_points_f32
        else:
            raise ValueError(dtype)
        M, K = Xa.shape
        N = Wga.shape[0]
        assert Wga.shape == (N, K) and Wua.shape == (N, K)
        assert count == 0 or (0 <= idx_m.min() and idx_m.max() < M
                              and 0 <= idx_n.min() and idx_n.max() < N)
        out = {k: np.empty(count, dtype=np.float64)
               for k in ("G", "U", "H", "AG", "AU")}
        if act == 0 and alpha == 1.0:
            rc = fn(_ptr(Xa), _ptr(Wga), _ptr(Wua), K, _ptr(idx_m), _ptr(idx_n),
                    count, _ptr(out["G"]), _ptr(out["U"]), _ptr(out["H"]),
                    _ptr(out["AG"]), _ptr(out["AU"]))
        else:
            rc = self.lib.oracle_swiglu_fwd_points_act(
                0 if dtype == "bf16" else 1, _ptr(Xa), _ptr(Wga), _ptr(Wua), K, _ptr(idx_m),
                _ptr(idx_n), count, int(act), float(alpha), _ptr(out["G"]), _ptr(out["U"]),
                _ptr(out["H"]), _ptr(out["AG"]), _ptr(out["AU"]))
        if rc != 0:
            raise MemoryError("oracle: row buffer allocation failed")
        return out

    def set_num_threads(self, n: int) -> None:
        """OpenMP threads of the row loops (timing only; results unchanged)."""
        self.lib.oracle_set_num_threads(int(n))

    # ---- quantised output ------------------------------------------------------
    def e4m3_decode(self, code: int) -> float:
        return self.lib.oracle_e4m3_decode(int(code))

    def e4m3_encode(self, v: float) -> int:
        return self.lib.oracle_e4m3_encode(float(v))

    def ue8m0_exponent(self, amax: float) -> int:
        return self.lib.oracle_ue8m0_exponent(float(amax))

    def quant_e4m3(self, H):
        """(q uint8 [M,N] e4m3 codes, s uint8 [M, ceil(N/32)] UE8M0 codes)
        of a float64 [M,N] array, per (1,32) block."""
        H = np.ascontiguousarray(H, dtype=np.float64)
        if H.ndim == 1:
            H = H[None, :]
        M, N = H.shape
        q = np.empty((M, N), dtype=np.uint8)
        s = np.empty((M, (N + 31) // 32), dtype=np.uint8)
        self.lib.oracle_quant_e4m3(_ptr(H), M, N, q.ctypes.data_as(ctypes.c_void_p),
                                   s.ctypes.data_as(ctypes.c_void_p))
        return q, s

    # ---- backward GEMMs -------------------------------------------------------
    def bwd_dx_f64(self, dG, dU, Wg, Wu):
        """dX [M,K] = dG Wg + dU Wu for dG, dU [M,N] and Wg, Wu [N,K]."""
        dG, dU, Wg, Wu = (np.ascontiguousarray(a, dtype=np.float64) for a in (dG, dU, Wg, Wu))
        M, N = dG.shape
        K = Wg.shape[1]
        assert dU.shape == (M, N) and Wg.shape == (N, K) and Wu.shape == (N, K)
        dX = np.empty((M, K), dtype=np.float64)
        self.lib.oracle_bwd_dx_f64(_ptr(dG), _ptr(dU), _ptr(Wg), _ptr(Wu), M, K, N, _ptr(dX))
        return dX

    def bwd_dw_f64(self, dG, dU, X):
        """(dWg, dWu) [N,K] = (dG^T X, dU^T X) for dG, dU [M,N] and X [M,K]."""
        dG, dU, X = (np.ascontiguousarray(a, dtype=np.float64) for a in (dG, dU, X))
        M, N = dG.shape
        K = X.shape[1]
        assert dU.shape == (M, N) and X.shape == (M, K)
        dWg = np.empty((N, K), dtype=np.float64)
        dWu = np.empty((N, K), dtype=np.float64)
        self.lib.oracle_bwd_dw_f64(_ptr(dG), _ptr(dU), _ptr(X), M, K, N, _ptr(dWg), _ptr(dWu))
        return dWg, dWu

    # ---- backward --------------------------------------------------------------
    def dswiglu_f64(self, dH, G, U, act: int = 0, alpha: float = 1.0):
        """Elementwise backward of h = act(alpha g) u on float64 arrays of
        equal shape -> (dG, dU); act 0 = SiLU (dSwiGLU), 1 = GELU(tanh)."""
        dH = np.ascontiguousarray(dH, dtype=np.float64)
        G = np.ascontiguousarray(G, dtype=np.float64)
        U = np.ascontiguousarray(U, dtype=np.float64)
        assert dH.shape == G.shape == U.shape
        dG = np.empty(G.shape, dtype=np.float64)
        dU = np.empty(G.shape, dtype=np.float64)
        self.lib.oracle_dswiglu_act_f64(_ptr(dH), _ptr(G), _ptr(U), G.size, int(act),
                                        float(alpha), _ptr(dG), _ptr(dU))
        return dG, dU

    def dswiglu(self, dH, G, U, dtype: str = "bf16", act: int = 0, alpha: float = 1.0):
        """dSwiGLU straight from bf16 (bits / torch.bfloat16) or fp32."""
        if act != 0 or alpha != 1.0:
            return self.dswiglu_f64(self.decode(dH, dtype), self.decode(G, dtype),
                                    self.decode(U, dtype), act, alpha)
        if dtype == "bf16":
            a, b, c = _as_bits(dH), _as_bits(G), _as_bits(U)
            fn = self.lib.oracle_dswiglu_bf16
        elif dtype == "f32":
            a, b, c = _as_f32(dH), _as_f32(G), _as_f32(U)
            fn = self.lib.oracle_dswiglu_f32
        else:
            raise ValueError(dtype)
        assert a.shape == b.shape == c.shape
        dG = np.empty(a.shape, dtype=np.float64)
        dU = np.empty(a.shape, dtype=np.float64)
        fn(_ptr(a), _ptr(b), _ptr(c), a.size, _ptr(dG), _ptr(dU))
        return dG, dU


def default() -> Oracle:
    """The oracle built from the committed source (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def __getattr__(name):
    # Module-level convenience: oracle.swiglu_fwd(...) etc. use default().
    if name in {"sigmoid", "silu", "dsilu", "gelu_tanh", "dgelu_tanh", "act", "dact",
                "decode_bf16", "decode",
                "swiglu_fwd_f64", "swiglu_fwd", "swiglu_fwd_points",
                "dswiglu_f64", "dswiglu", "bwd_dx_f64", "bwd_dw_f64",
                "e4m3_decode", "e4m3_encode", "ue8m0_exponent", "quant_e4m3",
                "set_num_threads"}:
        return getattr(default(), name)
    raise AttributeError(name)
