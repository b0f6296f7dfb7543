"""ctypes wrapper around the fp64 C oracle for ReLU linear attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. It shares no code with the
CUDA library. What the oracle computes, with the passages it follows, is written
at the top of ``linattn_oracle.c``.

Inputs are numpy arrays of shape (B, N, H, d); they are converted to float64
(lossless for the bf16 and fp32 values the workloads use). Outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "linattn_oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")

_c_long = ctypes.c_long
_c_double = ctypes.c_double
_ptr = ctypes.c_void_p


def compile_library(source: str = SOURCE, out: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) into ``out``."""
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           *extra_flags, source, "-o", out]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _stale(lib: str, src: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(src)


class Oracle:
    """Loaded oracle library. ``path`` may point at another build of the same
    source (the mutation tests load deliberately broken copies this way)."""

    def __init__(self, path: str | None = None):
        if path is None:
            path = LIBRARY
            if _stale(path, SOURCE):
                compile_library()
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_state.argtypes = [_ptr, _ptr, _c_long, _c_long, _c_long, _c_long, _ptr]
        lib.oracle_state.restype = None
        lib.oracle_apply.argtypes = [_ptr, _ptr, _c_long, _c_long, _c_long, _c_long,
                                     _c_double, _ptr, _ptr]
        lib.oracle_apply.restype = None
        lib.oracle_block_causal_state.argtypes = [_ptr, _ptr, _c_long, _c_long, _c_long, _c_long,
                                                  _c_long, _ptr]
        lib.oracle_block_causal_state.restype = None
        lib.oracle_block_causal_apply.argtypes = [_ptr, _ptr, _c_long, _c_long, _c_long, _c_long,
                                                  _c_long, _c_double, _ptr]
        lib.oracle_block_causal_apply.restype = None
        lib.oracle_state_fm.argtypes = [_ptr, _ptr, _c_long, _c_long, _c_long, _c_long, ctypes.c_int, _ptr]
        lib.oracle_state_fm.restype = None
        lib.oracle_apply_fm.argtypes = [_ptr, _ptr, _c_long, _c_long, _c_long, _c_long, ctypes.c_int,
                                        _c_double, _ptr, _ptr]
        lib.oracle_apply_fm.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        self._lib = lib

    @staticmethod
    def _f64(x) -> np.ndarray:
        a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
        if a.ndim != 4:
            raise ValueError(f"expected a (B, N, H, d) array, got shape {a.shape}")
        return a

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def state(self, K, V) -> np.ndarray:
        """S = phi(K)^T [V | 1] per (b, h): shape (B, H, d, d+1), float64."""
        K = self._f64(K)
        V = self._f64(V)
        if K.shape != V.shape:
            raise ValueError("K and V must have the same shape")
        B, N, H, d = K.shape
        S = np.empty((B, H, d, d + 1), dtype=np.float64)
        self._lib.oracle_state(K.ctypes.data, V.ctypes.data, B, N, H, d, S.ctypes.data)
        return S

    def apply(self, Q, S, eps: float, return_den: bool = False):
        """O = (phi(Q) S[:, :d]) / (phi(Q) S[:, d] + eps): shape (B, N, H, d)."""
        Q = self._f64(Q)
        S = np.ascontiguousarray(np.asarray(S, dtype=np.float64))
        B, N, H, d = Q.shape
        if S.shape != (B, H, d, d + 1):
            raise ValueError(f"state shape {S.shape} does not match Q {Q.shape}")
        O = np.empty((B, N, H, d), dtype=np.float64)
        den = np.empty((B, N, H), dtype=np.float64) if return_den else None
        self._lib.oracle_apply(Q.ctypes.data, S.ctypes.data, B, N, H, d, float(eps),
                               O.ctypes.data, den.ctypes.data if return_den else None)
        return (O, den) if return_den else O

    def forward(self, Q, K, V, eps: float, return_den: bool = False):
        S = self.state(K, V)
        return self.apply(Q, S, eps, return_den=return_den)


    FEATURE_MAPS = {"relu": 0, "elu1": 1, "cos": 2}

    def state_fm(self, K, V, feature: str) -> np.ndarray:
        """S = phi(K)^T [V | 1] with phi = relu | elu1 (ELU + 1) | cos."""
        K = self._f64(K)
        V = self._f64(V)
        if K.shape != V.shape:
            raise ValueError("K and V must have the same shape")
        B, N, H, d = K.shape
        S = np.empty((B, H, d, d + 1), dtype=np.float64)
        self._lib.oracle_state_fm(K.ctypes.data, V.ctypes.data, B, N, H, d,
                                  self.FEATURE_MAPS[feature], S.ctypes.data)
        return S

    def apply_fm(self, Q, S, feature: str, eps: float, return_den: bool = False):
        Q = self._f64(Q)
        S = np.ascontiguousarray(np.asarray(S, dtype=np.float64))
        B, N, H, d = Q.shape
        if S.shape != (B, H, d, d + 1):
            raise ValueError(f"state shape {S.shape} does not match Q {Q.shape}")
        O = np.empty((B, N, H, d), dtype=np.float64)
        den = np.empty((B, N, H), dtype=np.float64) if return_den else None
        self._lib.oracle_apply_fm(Q.ctypes.data, S.ctypes.data, B, N, H, d, self.FEATURE_MAPS[feature],
                                  float(eps), O.ctypes.data, den.ctypes.data if return_den else None)
        return (O, den) if return_den else O

    def forward_fm(self, Q, K, V, feature: str, eps: float, return_den: bool = False):
        return self.apply_fm(Q, self.state_fm(K, V, feature), feature, eps, return_den=return_den)

    # ---------------------------------------------- projection-fused state --
    # "SANA: Efficient High-Resolution Image Synthesis with Linear Diffusion
    # Transformers" (phd-frog.tistory.com/40), section 4 "On-Device Deployment":
    # the ReLU(K)^T V product is fused into the QKV projection, and the key-value
    # projection stays in full precision. Reading: K = X Wk^T and V = X Wv^T
    # (no bias), each rounded to bf16 as the projection would store it, then the
    # state phi(K)^T [V | 1] as above; the fused kernel never writes K or V.

    @staticmethod
    def round_bf16(x) -> np.ndarray:
        """Round to the nearest bfloat16 value (8 significant bits, ties to even), as float64."""
        x = np.asarray(x, dtype=np.float64)
        m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
        return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)   # np.round: half to even

    def project_kv(self, X, Wk, Wv, H: int):
        """K, V (B, N, H, d) = bf16(X Wk^T), bf16(X Wv^T) for X (B, N, C) and W (H*d, C)."""
        X = np.asarray(X, dtype=np.float64)
        Wk = np.asarray(Wk, dtype=np.float64)
        Wv = np.asarray(Wv, dtype=np.float64)
        B, N, C = X.shape
        HD = Wk.shape[0]
        if Wk.shape != (HD, C) or Wv.shape != (HD, C) or HD % H:
            raise ValueError("weights must be (H*d, C) with C matching X")
        K = self.round_bf16(X @ Wk.T).reshape(B, N, H, HD // H)
        V = self.round_bf16(X @ Wv.T).reshape(B, N, H, HD // H)
        return K, V

    def projected_state(self, X, Wk, Wv, H: int) -> np.ndarray:
        """phi(K)^T [V | 1] with K, V from the key-value projection of X."""
        K, V = self.project_kv(X, Wk, Wv, H)
        return self.state(K, V)

    # ------------------------------------------------------------- Mix-FFN --
    # "SANA: Efficient High-Resolution Image Synthesis with Linear Diffusion
    # Transformers" (phd-frog.tistory.com/40), section 2.2 "선형 어텐션 블럭":
    # Mix-FFN = an inverted residual block (1x1 expand, 3x3 depthwise conv over
    # the 2-D token grid, 1x1 project) with a GLU; section 4: the GLU is fused
    # into the Mix-FFN kernel. Readings: tokens n = y * W + x on an (Hg, W)
    # grid; expand X -> U = X W1^T with 2*Ch channels; depthwise 3x3 with zero
    # padding; GLU with the original sigmoid gate on the channel halves,
    # Z = D[:, :Ch] * sigmoid(D[:, Ch:]); project Y = Z W2^T. No biases, no
    # other activation, no residual inside the block. U and Z are rounded to
    # bf16 as the stored intermediates of a kernel pipeline would be.

    @staticmethod
    def depthwise3x3(U, Kdw, hw) -> np.ndarray:
        """D[b, y, x, c] = sum_{dy, dx in 0..2} U[b, y+dy-1, x+dx-1, c] Kdw[c, dy, dx]
        (zero outside the grid); U (B, Hg*W, Cc) -> D (B, Hg*W, Cc)."""
        U = np.asarray(U, dtype=np.float64)
        Kdw = np.asarray(Kdw, dtype=np.float64)
        Hg, W = hw
        B, N, Cc = U.shape
        if N != Hg * W or Kdw.shape != (Cc, 3, 3):
            raise ValueError("grid or kernel shape mismatch")
        G = np.zeros((B, Hg + 2, W + 2, Cc))
        G[:, 1:-1, 1:-1, :] = U.reshape(B, Hg, W, Cc)
        D = np.zeros((B, Hg, W, Cc))
        for dy in range(3):
            for dx in range(3):
                D += G[:, dy:dy + Hg, dx:dx + W, :] * Kdw[:, dy, dx]
        return D.reshape(B, N, Cc)

    def expand(self, X, W1) -> np.ndarray:
        """The 1x1 expand, stored as bf16: U = bf16(X W1^T), (B, N, 2 Ch)."""
        X = np.asarray(X, dtype=np.float64)
        W1 = np.asarray(W1, dtype=np.float64)
        if W1.shape[1] != X.shape[-1]:
            raise ValueError("W1 must be (2 Ch, C) with C matching X")
        return self.round_bf16(X @ W1.T)

    def depthwise_glu(self, U, Kdw, hw) -> np.ndarray:
        """The 3x3 depthwise conv of U followed by the GLU with the sigmoid gate
        on the channel halves, stored as bf16:
        Z = bf16(D[..., :Ch] * sigmoid(D[..., Ch:])), D = depthwise3x3(U)."""
        D = self.depthwise3x3(U, Kdw, hw)
        Ch2 = D.shape[-1]
        if Ch2 % 2:
            raise ValueError("U must have an even channel count (2 Ch)")
        Ch = Ch2 // 2
        return self.round_bf16(D[..., :Ch] / (1.0 + np.exp(-D[..., Ch:])))

    def mix_ffn(self, X, W1, Kdw, W2, hw) -> np.ndarray:
        """Y (B, N, C) for X (B, N, C), W1 (2 Ch, C), Kdw (2 Ch, 3, 3), W2 (C, Ch):
        expand, depthwise conv + GLU, then the 1x1 project Y = Z W2^T."""
        X = np.asarray(X, dtype=np.float64)
        W1 = np.asarray(W1, dtype=np.float64)
        W2 = np.asarray(W2, dtype=np.float64)
        Ch2 = W1.shape[0]
        if Ch2 % 2 or W2.shape[1] * 2 != Ch2 or W1.shape[1] != X.shape[2]:
            raise ValueError("weight shapes do not match")
        Z = self.depthwise_glu(self.expand(X, W1), Kdw, hw)
        return Z @ W2.T

    def block_causal_state(self, K, V, L: int) -> np.ndarray:
        """Inclusive prefix states of blocks of L tokens: (B, H, nblk, d, d+1)."""
        K = self._f64(K)
        V = self._f64(V)
        if K.shape != V.shape:
            raise ValueError("K and V must have the same shape")
        if L < 1:
            raise ValueError("block length must be >= 1")
        B, N, H, d = K.shape
        nblk = -(-N // L)
        P = np.empty((B, H, nblk, d, d + 1), dtype=np.float64)
        self._lib.oracle_block_causal_state(K.ctypes.data, V.ctypes.data, B, N, H, d, int(L),
                                            P.ctypes.data)
        return P

    def block_causal_apply(self, Q, P, L: int, eps: float) -> np.ndarray:
        """O for block-causal attention from the prefix states P."""
        Q = self._f64(Q)
        P = np.ascontiguousarray(np.asarray(P, dtype=np.float64))
        B, N, H, d = Q.shape
        if L < 1 or P.shape != (B, H, -(-N // L), d, d + 1):
            raise ValueError(f"prefix states {P.shape} do not match Q {Q.shape} and L={L}")
        O = np.empty((B, N, H, d), dtype=np.float64)
        self._lib.oracle_block_causal_apply(Q.ctypes.data, P.ctypes.data, B, N, H, d, int(L),
                                            float(eps), O.ctypes.data)
        return O

    def block_causal_forward(self, Q, K, V, L: int, eps: float) -> np.ndarray:
        return self.block_causal_apply(Q, self.block_causal_state(K, V, L), L, eps)


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``linattn_oracle.c`` (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
