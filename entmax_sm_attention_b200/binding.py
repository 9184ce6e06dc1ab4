"""ctypes binding of libentmax_attn.so (declared in include/entmax_attn.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels. PyTorch supplies device memory and the current stream. If the
shared object is missing the first call raises, with no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libentmax_attn.so")

(ENTMAX_OK, ENTMAX_EINVAL, ENTMAX_EUNSUPPORTED, ENTMAX_ECUDA, ENTMAX_ENOCONVERGE, ENTMAX_ETIMEOUT,
 ENTMAX_ERANGE) = range(7)
STATUS_NAMES = {0: "ENTMAX_OK", 1: "ENTMAX_EINVAL", 2: "ENTMAX_EUNSUPPORTED", 3: "ENTMAX_ECUDA",
                4: "ENTMAX_ENOCONVERGE", 5: "ENTMAX_ETIMEOUT", 6: "ENTMAX_ERANGE"}
ENTMAX_BF16, ENTMAX_FP32 = 0, 1
ENTMAX_MAX_L = 16384
ENTMAX_TILE = 128
EXPORTS = ("entmax_attn_workspace_bytes", "entmax_attn_fwd", "entmax_attn_bwd", "entmax_rows",
           "entmax_last_device_status", "entmax_attn_block_mask", "entmax_attn_block_mask64",
           "entmax_attn_fwd_noalloc")
ENTMAX_NOALLOC_SCRATCH_BYTES = 16 << 20
ENTMAX_SELFTEST_STALL = 1
FWD_STATS = 8     # int32 counters per query tile (forward)
BWD_STATS = 8     # int32 counters per key tile (backward)


class EntmaxError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


class AttnDesc(ctypes.Structure):
    """Mirror of entmax_attn_desc."""
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("d", ctypes.c_int),
        ("alpha", ctypes.c_float), ("scale", ctypes.c_float),
        ("causal", ctypes.c_int), ("window", ctypes.c_int),
        ("kv_len", ctypes.c_void_p), ("dtype", ctypes.c_int), ("max_sweeps", ctypes.c_int),
        ("wait_limit_us", ctypes.c_int), ("alibi_slopes", ctypes.c_void_p), ("selftest", ctypes.c_int),
        ("mask64", ctypes.c_int),
    ]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library; raises if it has not been built (no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m entmax_sm_attention_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    dp = ctypes.POINTER(AttnDesc)
    lib.entmax_attn_workspace_bytes.argtypes = [dp]
    lib.entmax_attn_workspace_bytes.restype = sz
    lib.entmax_attn_fwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp]
    lib.entmax_attn_fwd.restype = i
    lib.entmax_attn_bwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.entmax_attn_bwd.restype = i
    lib.entmax_rows.argtypes = [vp, i, i, i, f, vp, vp, vp, vp]
    lib.entmax_rows.restype = i
    lib.entmax_last_device_status.argtypes = [dp, vp, ctypes.POINTER(i), vp]
    lib.entmax_last_device_status.restype = i
    lib.entmax_attn_block_mask.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.entmax_attn_block_mask.restype = i
    lib.entmax_attn_block_mask64.argtypes = [dp, vp, vp, vp]
    lib.entmax_attn_block_mask64.restype = i
    lib.entmax_attn_fwd_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp]
    lib.entmax_attn_fwd_noalloc.restype = i
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, code: int, ok=(ENTMAX_OK,)):
    if code not in ok:
        raise EntmaxError(fn, code)
    return code


@dataclass
class Options:
    alpha: float = 1.5
    scale: float | None = None
    causal: bool = False
    window: int = -1
    max_sweeps: int = 0


def make_desc(B: int, H: int, L: int, d: int = 64, *, alpha: float = 1.5, scale: float | None = None,
              causal: bool = False, window: int = -1, kv_len: torch.Tensor | None = None,
              dtype: int = ENTMAX_BF16, max_sweeps: int = 0, wait_limit_us: int = 0,
              alibi: torch.Tensor | None = None, selftest: int = 0, mask64: bool = False) -> AttnDesc:
    """Fill an entmax_attn_desc. kv_len, if given, is a device int32 tensor [B]; alibi, if
    given, a device float32 tensor [H] of ALiBi slopes."""
    if kv_len is not None and (kv_len.dtype != torch.int32 or not kv_len.is_cuda):
        raise ValueError("kv_len must be a CUDA int32 tensor")
    if alibi is not None and (alibi.dtype != torch.float32 or not alibi.is_cuda or alibi.numel() != H):
        raise ValueError("alibi must be a CUDA float32 tensor of H slopes")
    return AttnDesc(B, H, L, d, float(alpha), float(scale if scale is not None else d ** -0.5),
                    int(bool(causal) or window >= 0), int(window), _ptr(kv_len), int(dtype), int(max_sweeps),
                    int(wait_limit_us), _ptr(alibi), int(selftest), int(bool(mask64)))


def entmax_attn_workspace_bytes(desc: AttnDesc) -> int:
    return int(load_library().entmax_attn_workspace_bytes(ctypes.byref(desc)))


def entmax_attn_fwd(desc: AttnDesc, Q, K, V, O, tau, workspace, stream=None) -> int:
    return _check("entmax_attn_fwd", load_library().entmax_attn_fwd(
        ctypes.byref(desc), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(tau), _ptr(workspace), _stream(stream)))


def entmax_attn_bwd(desc: AttnDesc, Q, K, V, dO, tau, workspace, dQ, dK, dV, stream=None) -> int:
    return _check("entmax_attn_bwd", load_library().entmax_attn_bwd(
        ctypes.byref(desc), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(tau), _ptr(workspace),
        _ptr(dQ), _ptr(dK), _ptr(dV), _stream(stream)))


def entmax_rows(S, rows: int, n: int, ld: int, alpha: float, P, tau, status=None, stream=None) -> int:
    return _check("entmax_rows", load_library().entmax_rows(
        _ptr(S), int(rows), int(n), int(ld), float(alpha), _ptr(P), _ptr(tau), _ptr(status), _stream(stream)))


def entmax_last_device_status(desc: AttnDesc, workspace, stream=None) -> tuple[int, int]:
    """Returns (status code, raw status word); synchronises the stream. workspace=None reads
    the no-allocation forward's scratch on the current device."""
    word = ctypes.c_int(0)
    code = load_library().entmax_last_device_status(ctypes.byref(desc), _ptr(workspace), ctypes.byref(word),
                                                     _stream(stream))
    _check("entmax_last_device_status", code, ok=(ENTMAX_OK, ENTMAX_ENOCONVERGE, ENTMAX_ETIMEOUT, ENTMAX_ERANGE))
    return code, word.value


def entmax_attn_block_mask(desc: AttnDesc, workspace, M=None, stats=None, bwd_stats=None, stream=None) -> int:
    return _check("entmax_attn_block_mask", load_library().entmax_attn_block_mask(
        ctypes.byref(desc), _ptr(workspace), _ptr(M), _ptr(stats), _ptr(bwd_stats), _stream(stream)))


def entmax_attn_block_mask64(desc: AttnDesc, workspace, M64, stream=None) -> int:
    return _check("entmax_attn_block_mask64", load_library().entmax_attn_block_mask64(
        ctypes.byref(desc), _ptr(workspace), _ptr(M64), _stream(stream)))


def entmax_attn_fwd_noalloc(desc: AttnDesc, Q, K, V, O, tau, stream=None) -> int:
    """Forward for callers that cannot allocate: the library's fixed per-GPU scratch
    replaces the workspace (see include/entmax_attn.h for the size limit and the rule
    that overlapping calls race)."""
    return _check("entmax_attn_fwd_noalloc", load_library().entmax_attn_fwd_noalloc(
        ctypes.byref(desc), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(tau), _stream(stream)))


# ---------------------------------------------------------------- tensor conveniences
def alloc_workspace(desc: AttnDesc, device="cuda") -> torch.Tensor:
    n = entmax_attn_workspace_bytes(desc)
    if n == 0:
        raise EntmaxError("entmax_attn_workspace_bytes", ENTMAX_EINVAL)
    return torch.empty(n, dtype=torch.uint8, device=device)


def mask_shape(desc: AttnDesc) -> tuple:
    T = -(-desc.L // ENTMAX_TILE)
    return (desc.B, desc.H, T, -(-T // 32))


def mask64_shape(desc: AttnDesc) -> tuple:
    T = -(-desc.L // ENTMAX_TILE)
    return (desc.B, desc.H, 2 * T, -(-2 * T // 32))


def forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, *, alpha: float = 1.5, scale=None,
            causal: bool = False, window: int = -1, kv_len=None, max_sweeps: int = 0, wait_limit_us: int = 0,
            alibi=None, selftest: int = 0, mask64: bool = False):
    """O, tau and the (desc, workspace) context of one forward call on [B, H, L, 64] tensors."""
    B, H, L, d = Q.shape
    dtype = ENTMAX_BF16 if Q.dtype == torch.bfloat16 else ENTMAX_FP32
    desc = make_desc(B, H, L, d, alpha=alpha, scale=scale, causal=causal, window=window, kv_len=kv_len,
                     dtype=dtype, max_sweeps=max_sweeps, wait_limit_us=wait_limit_us, alibi=alibi,
                     selftest=selftest, mask64=mask64)
    ws = alloc_workspace(desc, Q.device)
    O = torch.empty((B, H, L, d), dtype=torch.float32, device=Q.device)
    tau = torch.empty((B, H, L), dtype=torch.float32, device=Q.device)
    entmax_attn_fwd(desc, Q, K, V, O, tau, ws)
    return O, tau, (desc, ws)


def backward(ctx, Q, K, V, dO, tau):
    """dQ, dK, dV for the forward that produced ctx and tau."""
    desc, ws = ctx
    dQ, dK, dV = (torch.empty(Q.shape, dtype=torch.float32, device=Q.device) for _ in range(3))
    entmax_attn_bwd(desc, Q, K, V, dO, tau, ws, dQ, dK, dV)
    return dQ, dK, dV


def block_mask(ctx):
    """(M as int32 bit patterns [B, H, Tr, ceil(Tc/32)], stats int32 [B, H, Tr, 8]) of a
    forward; stats = (refinement passes, S tiles computed, flagged tiles, active tiles,
    then cycles of the max pass, of refinement + mask decision, of the output pass, total)."""
    desc, ws = ctx
    Mv = torch.empty(mask_shape(desc), dtype=torch.int32, device=ws.device)
    st = torch.empty(mask_shape(desc)[:3] + (FWD_STATS,), dtype=torch.int32, device=ws.device)
    entmax_attn_block_mask(desc, ws, Mv, st)
    return Mv, st


def block_mask64(ctx):
    """The forward's mask at 64 x 64 blocks as int32 bit patterns [B, H, 2 Tr, ceil(2 Tc/32)]."""
    desc, ws = ctx
    M64 = torch.empty(mask64_shape(desc), dtype=torch.int32, device=ws.device)
    entmax_attn_block_mask64(desc, ws, M64)
    return M64


def bwd_counters(ctx):
    """int32 [B, H, Tc, 8] counters of the last backward per key tile: flagged query tiles
    visited, total cycles, and the first row-owner warp's cycles waiting for S/dA, waiting
    for the previous tile's MMAs, forming A/dS, staging dQ, and the part of forming spent
    loading S and dA from tensor memory (then a zero)."""
    desc, ws = ctx
    st = torch.empty(mask_shape(desc)[:3] + (BWD_STATS,), dtype=torch.int32, device=ws.device)
    entmax_attn_block_mask(desc, ws, None, None, st)
    return st


def rows(S: torch.Tensor, alpha: float = 1.5, return_status: bool = False):
    """P, tau = alpha-entmax of the rows of a CUDA fp32 matrix S [rows, n] (n % 4 == 0 or padded).
    With return_status, also the device status word (1 = a row reached the iteration cap)."""
    r, n = S.shape
    P = torch.empty_like(S)
    tau = torch.empty(r, dtype=torch.float32, device=S.device)
    status = torch.zeros(1, dtype=torch.int32, device=S.device)
    entmax_rows(S, r, n, S.stride(0), alpha, P, tau, status)
    if return_status:
        return P, tau, int(status.item())
    return P, tau
