"""Seeded synthetic workloads for fused alpha-entmax attention.

This module draws inputs and nothing else: it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it.

The workload shapes follow the experiments on the pages. "AdaSplash-2: Faster
Differentiable Sparse Attention", §4.2 "Sparsity-speed tradeoff", uses random
Gaussian Q, K, V with d=64 in bf16, and sets block sparsity through the query
variance. The GPT-2-small shape (12 heads, 1k context) comes from the same
paper's GPT-2 runs. The window-with-sink mask (W=32, sink at key 0) comes from
the "gpt2-adasplash-attention" model card.

Recipe: one CPU ``torch.Generator`` seeded with ``seed`` draws fp32
``randn`` tensors in the order Q, K, V, dO. Q is multiplied by ``sigma_q``, and
every tensor is then rounded to the config's dtype. The same rounded values go
to the GPU and, widened exactly to fp64, to the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int = 64
    dtype: str = "bf16"          # dtype of Q, K, V, dO
    causal: bool = False
    window: int = -1             # >= 0: active = {0} U [max(1, i-window), i]
    kv_len: int | None = None    # valid keys per sequence (same for every batch entry)
    alphas: tuple = (1.5,)
    sigma_q: float = 1.0
    backward: bool = True
    alibi: tuple | None = None   # ALiBi slopes per head (score units per position), or None
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "fp32": torch.float32}[self.dtype]

    def kv_len_list(self):
        return None if self.kv_len is None else [self.kv_len] * self.B

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "single_head_L128_fp32": Workload(
        "single_head_L128_fp32", B=1, H=1, L=128, dtype="fp32", causal=False, alphas=(1.5,),
        backward=False, note="forward only, plus entmax_rows on the 128x128 score matrix"),
    "gpt2_causal_L1024": Workload(
        "gpt2_causal_L1024", B=8, H=12, L=1024, causal=True, alphas=(1.5,)),
    "long_causal_L8192": Workload(
        "long_causal_L8192", B=1, H=12, L=8192, causal=True, alphas=(1.5, 2.0), sigma_q=3.0,
        note="Q ~ N(0, 3^2): peaked rows (query variance sets sparsity)"),
    "encoder_padded_L4096": Workload(
        "encoder_padded_L4096", B=4, H=12, L=4096, causal=False, kv_len=3072, alphas=(1.5, 2.0),
        note="bidirectional, trailing 25% of keys padded"),
    "window_sink_L2048": Workload(
        "window_sink_L2048", B=16, H=12, L=2048, causal=True, window=32, alphas=(1.5,)),
}

# The headline throughput workload (fwd+bwd at L=8192).
HEADLINE = "long_causal_L8192"


def make_inputs(w: Workload, seed: int = 0, device: str = "cpu") -> dict:
    """Q, K, V, dO [B, H, L, d] in the workload dtype (drawn on the CPU, then moved)."""
    g = torch.Generator().manual_seed(seed)
    shape = (w.B, w.H, w.L, w.d)
    Q = torch.randn(shape, generator=g, dtype=torch.float32) * w.sigma_q
    K = torch.randn(shape, generator=g, dtype=torch.float32)
    V = torch.randn(shape, generator=g, dtype=torch.float32)
    dO = torch.randn(shape, generator=g, dtype=torch.float32)
    out = {k: v.to(w.torch_dtype).contiguous() for k, v in (("Q", Q), ("K", K), ("V", V), ("dO", dO))}
    if device != "cpu":
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_kv_len(w: Workload, device: str = "cpu"):
    if w.kv_len is None:
        return None
    return torch.full((w.B,), w.kv_len, dtype=torch.int32, device=device)


def make_score_rows(rows: int, n: int, seed: int = 0, sigma: float = 1.0) -> torch.Tensor:
    """fp32 score rows ~ N(0, sigma^2) for the row-wise solver (the Gaussian score
    vectors of AdaSplash-2 §4.1)."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((rows, n), generator=g, dtype=torch.float32) * sigma).contiguous()


def small_case(name: str, *, B=1, H=2, L=300, d=64, dtype="bf16", causal=False, window=-1,
               kv_len=None, sigma_q=1.0, alphas=(1.5, 2.0), alibi=None) -> Workload:
    """A reduced workload the oracle finishes in seconds: several tiles plus a ragged tail."""
    return Workload(name, B=B, H=H, L=L, d=d, dtype=dtype, causal=causal, window=window,
                    kv_len=kv_len, sigma_q=sigma_q, alphas=alphas, alibi=None if alibi is None else tuple(alibi))


def make_planted_inputs(w: Workload, rho: float, seed: int = 0, gamma: float = 3.0) -> dict:
    """Block-structured inputs whose support lies in a chosen fraction rho of the key tiles.

    This family is not on the pages. It stands in for the trained models whose block
    sparsity AdaSplash-2 §4.2 and Fig. 7 report, which iid Gaussian inputs do not reach at
    128 x 128 tiles. Every key tile t of every (b, h) gets a centre c_t ~ N(0, I), and its
    keys are K_j = c_t + 0.3 N(0, I). Each query tile picks max(1, round(rho * n)) of the
    n key tiles it may attend to (causal: tiles 0..it). Each query row aims at one of the
    picked tiles t*: Q_i = gamma * c_{t*} + 0.5 N(0, I). With gamma = 3 and d = 64 a key of
    the chosen tile scores about gamma |c|^2 / sqrt(d) = 24 and any other key about
    N(0, gamma^2) = N(0, 9), so the support, and with it the flagged blocks, stays in the
    picked tiles (block sparsity about 1 - rho). V and dO ~ N(0, 1).
    """
    g = torch.Generator().manual_seed(seed)
    B, H, L, d, T = w.B, w.H, w.L, w.d, 128
    nT = -(-L // T)
    centres = torch.randn((B, H, nT, d), generator=g)
    tile_of = torch.arange(L) // T
    K = centres[:, :, tile_of, :] + 0.3 * torch.randn((B, H, L, d), generator=g)
    Q = 0.5 * torch.randn((B, H, L, d), generator=g)
    for it in range(nT):
        n_allowed = it + 1 if w.causal else nT
        n_pick = max(1, int(round(rho * n_allowed)))
        rows = slice(it * T, min(L, (it + 1) * T))
        nrows = rows.stop - rows.start
        for b in range(B):
            for h in range(H):
                picked = torch.randperm(n_allowed, generator=g)[:n_pick]
                choice = picked[torch.randint(0, n_pick, (nrows,), generator=g)]
                Q[b, h, rows] += gamma * centres[b, h, choice]
    V = torch.randn((B, H, L, d), generator=g)
    dO = torch.randn((B, H, L, d), generator=g)
    dt = w.torch_dtype
    return {"Q": Q.to(dt).contiguous(), "K": K.to(dt).contiguous(), "V": V.to(dt).contiguous(),
            "dO": dO.to(dt).contiguous()}
