"""fp64 CPU oracle for fused alpha-entmax attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never does, and the two
share no code: this module compiles ``entmax_oracle.c`` with gcc and wraps it
with ctypes/numpy.

Every function cites the definition it follows ("AdaSplash-2: Faster
Differentiable Sparse Attention", §2.2 scores, §2.3 Eq. 3, §2.4 Eq. 4 and the
sorting-based solvers, §3.3 block mask and backward support, Appendix C.4 mask
packing; the "gpt2-adasplash-attention" model card for the window-with-sink
mask). Inputs are converted to float64 exactly (bf16 and fp32 widen without
rounding).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "entmax_oracle.c")
_LIB = os.path.join(_HERE, "liborcl.so")
_lib = None

METHOD_SORT = 0
METHOD_BISECT = 1
METHOD_AUTO = 2     # the sorting solver for alpha in {1.5, 2}, bisection otherwise


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -O2, OpenMP). Returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        lp = ctypes.POINTER(ctypes.c_long)
        up = ctypes.POINTER(ctypes.c_uint32)
        i, d_ = ctypes.c_int, ctypes.c_double
        lib.orc_f.argtypes = [dp, i, d_, d_]
        lib.orc_f.restype = d_
        lib.orc_tau_sort.argtypes = [dp, i, d_]
        lib.orc_tau_sort.restype = d_
        lib.orc_tau_bisect.argtypes = [dp, i, d_, i]
        lib.orc_tau_bisect.restype = d_
        lib.orc_tau_hist.argtypes = [dp, i, d_, i]
        lib.orc_tau_hist.restype = d_
        lib.orc_entmax_rows.argtypes = [dp, ctypes.c_long, i, ctypes.c_long, d_, i, dp, dp]
        lib.orc_entmax_rows.restype = None
        shape = [i, i, i, i, d_, d_, i, i, ip, dp]   # ..., kv_len, alibi slopes
        lib.orc_attn_rows.argtypes = shape + [dp, dp, dp, dp, lp, ctypes.c_long, dp, dp, dp, dp, dp, dp]
        lib.orc_attn_rows.restype = i
        lib.orc_attn_cols.argtypes = shape + [dp, dp, dp, dp, dp, dp, lp, ctypes.c_long, dp, dp]
        lib.orc_attn_cols.restype = i
        lib.orc_block_mask.argtypes = shape + [dp, dp, dp, i, i, d_, up, up, up]
        lib.orc_block_mask.restype = i
        lib.orc_max_threads.restype = i
        lib.orc_set_threads.argtypes = [i]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening to contiguous float64 (torch tensors of any float dtype or numpy)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray, ct=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ct)) if a is not None else None


def max_threads() -> int:
    return int(_load().orc_max_threads())


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


# ----------------------------------------------------------------------------- rows
def f_root(z, alpha: float, tau: float) -> float:
    """Eq. 4, f(tau) = -1 + sum_j [z_j - tau]_+^{1/(alpha-1)} on z = (alpha-1) s."""
    z = _f64(z).ravel()
    return float(_load().orc_f(_p(z), z.size, float(alpha), float(tau)))


def tau_sort(z, alpha: float) -> float:
    """Exact tau* (Eq. 3 units) from the sorting-based solver of §2.4, alpha in {1.5, 2}."""
    z = _f64(z).ravel().copy()
    return float(_load().orc_tau_sort(_p(z), z.size, float(alpha)))


def tau_bisect(z, alpha: float, iters: int = 200) -> float:
    """Bisection on Eq. 4 over the §2.4 bracket (any alpha > 1)."""
    z = _f64(z).ravel()
    return float(_load().orc_tau_bisect(_p(z), z.size, float(alpha), int(iters)))


def tau_hist(z, alpha: float, bins: int) -> float:
    """Histogram initialisation of tau (AdaSplash-2 §3.1, Appendix C.3) on z = (alpha-1) s:
    the root of Eq. 4 with every score replaced by the left edge of its bin (B bins over the
    shifted range [0, 1]); Proposition 3.1 bounds it by tau* - 1/B < tau_h <= tau*."""
    z = _f64(z).ravel()
    return float(_load().orc_tau_hist(_p(z), z.size, float(alpha), int(bins)))


def entmax_rows(S, alpha: float, method: int = METHOD_AUTO):
    """alpha-entmax of each row of raw scores S [rows, n] (-inf = inactive).

    Returns (P [rows, n], tau [rows]) with P = [(alpha-1) S - tau]_+^{1/(alpha-1)} (Eq. 3).
    """
    S = _f64(S)
    rows, n = S.shape
    P = np.zeros_like(S)
    tau = np.zeros(rows)
    _load().orc_entmax_rows(_p(S), rows, n, n, float(alpha), int(method), _p(P), _p(tau))
    return P, tau


# ------------------------------------------------------------------------ attention
class Problem:
    """One attention problem held in float64: Q, K, V, dO [B, H, L, d] and its options."""

    def __init__(self, Q, K, V, dO=None, *, alpha: float, scale: float, causal: bool = False,
                 window: int = -1, kv_len=None, alibi=None):
        self.Q, self.K, self.V = _f64(Q), _f64(K), _f64(V)
        self.dO = _f64(dO) if dO is not None else None
        self.B, self.H, self.L, self.d = self.Q.shape
        self.alpha, self.scale = float(alpha), float(scale)
        self.causal, self.window = int(bool(causal) or window >= 0), int(window)
        if kv_len is None:
            self.kv_len = None
        else:
            self.kv_len = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32).reshape(self.B))
        # ALiBi slopes m_h per head (score units per position), or None.
        self.alibi = None if alibi is None else np.ascontiguousarray(np.asarray(alibi, dtype=np.float64).reshape(self.H))

    def _shape(self):
        kv = self.kv_len.ctypes.data_as(ctypes.POINTER(ctypes.c_int)) if self.kv_len is not None else None
        ab = self.alibi.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if self.alibi is not None else None
        return [self.B, self.H, self.L, self.d, self.alpha, self.scale, self.causal, self.window, kv, ab]

    def all_rows(self) -> np.ndarray:
        return np.arange(self.B * self.H * self.L, dtype=np.int64)

    def head_rows(self, b: int, h: int) -> np.ndarray:
        base = (b * self.H + h) * self.L
        return np.arange(base, base + self.L, dtype=np.int64)

    def rows(self, rows=None, *, backward: bool = False) -> dict:
        """Row pass for flattened rows (b*H + h)*L + i: O, tau, sum g, O~ and, if
        backward, delta and dQ. O = sum_j p_ij V_j, O~ = sum_j g_ij V_j with
        g = p^{2-alpha}; delta_i = sum_j g_ij (dO_i.V_j) / sum_j g_ij;
        dQ_i = scale sum_j g_ij (dO_i.V_j - delta_i) K_j."""
        rows = self.all_rows() if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n, d = rows.size, self.d
        out = {"O": np.zeros((n, d)), "tau": np.zeros(n), "sumg": np.zeros(n), "Ot": np.zeros((n, d))}
        if backward:
            if self.dO is None:
                raise ValueError("backward needs dO")
            out["delta"] = np.zeros(n)
            out["dQ"] = np.zeros((n, d))
        rc = _load().orc_attn_rows(*self._shape(), _p(self.Q), _p(self.K), _p(self.V),
                                   _p(self.dO) if backward else None, _p(rows, ctypes.c_long), n,
                                   _p(out["O"]), _p(out["tau"]), _p(out["sumg"]), _p(out["Ot"]),
                                   _p(out.get("delta")), _p(out.get("dQ")))
        if rc != 0:
            raise ValueError("oracle attention needs alpha > 1")
        return out

    def cols(self, tau_all: np.ndarray, delta_all: np.ndarray, cols=None) -> dict:
        """Column pass: dK_j = scale sum_i dS_ij Q_i and dV_j = sum_i p_ij dO_i for the
        flattened key positions cols; tau_all and delta_all cover every row."""
        cols = self.all_rows() if cols is None else np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
        n, d = cols.size, self.d
        dK, dV = np.zeros((n, d)), np.zeros((n, d))
        tau_all = np.ascontiguousarray(tau_all, dtype=np.float64)
        delta_all = np.ascontiguousarray(delta_all, dtype=np.float64)
        rc = _load().orc_attn_cols(*self._shape(), _p(self.Q), _p(self.K), _p(self.V), _p(self.dO),
                                   _p(tau_all), _p(delta_all), _p(cols, ctypes.c_long), n, _p(dK), _p(dV))
        if rc != 0:
            raise ValueError("oracle attention needs alpha > 1")
        return {"dK": dK, "dV": dV}

    def forward(self) -> dict:
        """Full forward: O [B,H,L,d], tau [B,H,L], sumg [B,H,L], Ot [B,H,L,d]."""
        r = self.rows()
        B, H, L, d = self.B, self.H, self.L, self.d
        return {"O": r["O"].reshape(B, H, L, d), "tau": r["tau"].reshape(B, H, L),
                "sumg": r["sumg"].reshape(B, H, L), "Ot": r["Ot"].reshape(B, H, L, d)}

    def backward(self) -> dict:
        """Full forward + backward: adds dQ, dK, dV [B,H,L,d] and delta [B,H,L]."""
        r = self.rows(backward=True)
        c = self.cols(r["tau"], r["delta"])
        B, H, L, d = self.B, self.H, self.L, self.d
        return {"O": r["O"].reshape(B, H, L, d), "tau": r["tau"].reshape(B, H, L),
                "sumg": r["sumg"].reshape(B, H, L), "Ot": r["Ot"].reshape(B, H, L, d),
                "delta": r["delta"].reshape(B, H, L), "dQ": r["dQ"].reshape(B, H, L, d),
                "dK": c["dK"].reshape(B, H, L, d), "dV": c["dV"].reshape(B, H, L, d)}

    def block_mask(self, tau: np.ndarray, Br: int = 128, Bc: int = 128, margin: float = 0.0):
        """Packed block masks (Appendix C.4) from fp64 z and tau [B,H,L]: returns
        (M, M_lo, M_hi) uint32 [B, H, Tr, ceil(Tc/32)]; M_lo/M_hi use tau +/- margin."""
        Tr, Tc = -(-self.L // Br), -(-self.L // Bc)
        Wc = -(-Tc // 32)
        shape = (self.B, self.H, Tr, Wc)
        M, Mlo, Mhi = (np.zeros(shape, dtype=np.uint32) for _ in range(3))
        tau = np.ascontiguousarray(np.asarray(tau, dtype=np.float64).reshape(-1))
        _load().orc_block_mask(*self._shape(), _p(self.Q), _p(self.K), _p(tau), int(Br), int(Bc),
                               float(margin), _p(M, ctypes.c_uint32), _p(Mlo, ctypes.c_uint32),
                               _p(Mhi, ctypes.c_uint32))
        return M, Mlo, Mhi
