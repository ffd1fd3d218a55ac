"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This module holds no attention arithmetic: it draws i.i.d. N(0, 1) tensors
from a seeded torch generator (one generator per (seed, tensor id), so each
tensor is reproducible on its own), rounds them once to bf16 (round to
nearest even) where the workload is bf16, and builds the structured inputs
the workloads need (global-token index sets, ring positions).  Both the CUDA
path and the CPU oracle consume exactly the tensors returned here.

Workload shapes follow the pages' models: Mistral-7B's causal window of 4096
with GQA 32/8 heads, Longformer-style global tokens, 64-token blocks for the
block-sparse dilation remark, and a 4096-slot ring cache for decode.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(tensor_id) * 7919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal(shape, seed: int, tensor_id: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0,1) fp32 draw, then a single rounding to ``dtype``."""
    x = torch.randn(*shape, generator=_gen(seed, tensor_id, device), device=device,
                    dtype=torch.float32)
    return x if dtype == torch.float32 else x.to(dtype)


def uniform_int(n: int, lo: int, hi: int, seed: int, tensor_id: int) -> torch.Tensor:
    """n integers uniform in [lo, hi] (inclusive), int64, on the CPU."""
    return torch.randint(lo, hi + 1, (n,), generator=_gen(seed, tensor_id, "cpu"),
                         dtype=torch.int64)


def every_nth(N: int, step: int) -> torch.Tensor:
    """Global-token set {0} plus every step-th position: {p : p % step == 0}."""
    return torch.arange(0, N, step, dtype=torch.int32)


@dataclass
class FwdConfig:
    name: str
    B: int
    N: int
    H: int
    Hkv: int
    D: int
    win_left: int
    win_right: int
    dilation: int = 1
    dilation_block: int = 0
    global_step: int = 0  # 0: no global tokens
    dtype: torch.dtype = torch.bfloat16
    scale: float = 0.0  # <= 0: 1/sqrt(D)
    seed: int = 1

    @property
    def global_idx(self) -> torch.Tensor:
        if self.global_step <= 0:
            return torch.zeros(0, dtype=torch.int32)
        return every_nth(self.N, self.global_step)


@dataclass
class DecodeConfig:
    name: str
    B: int
    H: int
    Hkv: int
    D: int
    W: int
    pos_lo: int
    pos_hi: int
    seed: int = 5
    extra: dict = field(default_factory=dict)


# The five workloads of the method's pages, plus shrunken variants used as
# parity cases (ragged tails, N < window, pos < W - 1, N mod d != 0).
CONFIGS = {
    "tiny_bidir_fp32": FwdConfig("tiny_bidir_fp32", B=1, N=256, H=2, Hkv=2, D=64,
                                 win_left=16, win_right=16, dtype=torch.float32,
                                 scale=1.0 / 8.0, seed=1001),
    "mistral_causal_prefill": FwdConfig("mistral_causal_prefill", B=1, N=8192, H=32, Hkv=8,
                                        D=128, win_left=4095, win_right=0, seed=1002),
    "longformer_global": FwdConfig("longformer_global", B=4, N=4096, H=12, Hkv=12, D=64,
                                   win_left=256, win_right=256, global_step=512, seed=1003),
    "dilated_token": FwdConfig("dilated_token", B=2, N=16384, H=16, Hkv=16, D=64,
                               win_left=128, win_right=128, dilation=4, seed=1004),
    "dilated_block": FwdConfig("dilated_block", B=2, N=16384, H=16, Hkv=16, D=64,
                               win_left=128, win_right=128, dilation=4, dilation_block=64,
                               seed=1004),
    # shrunken parity cases
    "small_causal": FwdConfig("small_causal", B=1, N=1000, H=8, Hkv=2, D=128,
                              win_left=300, win_right=0, seed=2002),
    "small_global": FwdConfig("small_global", B=2, N=700, H=3, Hkv=3, D=64,
                              win_left=40, win_right=40, global_step=128, seed=2003),
    "small_dilated": FwdConfig("small_dilated", B=1, N=1003, H=2, Hkv=2, D=64,
                               win_left=50, win_right=50, dilation=3, seed=2004),
    "small_block": FwdConfig("small_block", B=1, N=1024 + 320, H=2, Hkv=1, D=64,
                             win_left=128, win_right=128, dilation=4, dilation_block=64,
                             seed=2005),
}

DECODE_CONFIGS = {
    "ring_decode": DecodeConfig("ring_decode", B=64, H=32, Hkv=8, D=128, W=4096,
                                pos_lo=4096, pos_hi=131072, seed=1005),
    "small_ring_partial": DecodeConfig("small_ring_partial", B=5, H=8, Hkv=2, D=128, W=512,
                                       pos_lo=0, pos_hi=700, seed=2006),
}


def forward_inputs(cfg: FwdConfig, device="cpu"):
    """(q, k, v, global_idx) for a forward workload; q [B,N,H,D], k/v [B,N,Hkv,D]."""
    q = normal((cfg.B, cfg.N, cfg.H, cfg.D), cfg.seed, 0, cfg.dtype, device)
    k = normal((cfg.B, cfg.N, cfg.Hkv, cfg.D), cfg.seed, 1, cfg.dtype, device)
    v = normal((cfg.B, cfg.N, cfg.Hkv, cfg.D), cfg.seed, 2, cfg.dtype, device)
    return q, k, v, cfg.global_idx


def decode_inputs(cfg: DecodeConfig, device="cpu"):
    """(q [B,H,D], k_ring [B,W,Hkv,D], v_ring [B,W,Hkv,D], pos [B] int64)."""
    q = normal((cfg.B, cfg.H, cfg.D), cfg.seed, 0, torch.bfloat16, device)
    kr = normal((cfg.B, cfg.W, cfg.Hkv, cfg.D), cfg.seed, 1, torch.bfloat16, device)
    vr = normal((cfg.B, cfg.W, cfg.Hkv, cfg.D), cfg.seed, 2, torch.bfloat16, device)
    pos = uniform_int(cfg.B, cfg.pos_lo, cfg.pos_hi, cfg.seed, 3)
    return q, kr, vr, pos


@dataclass
class PagedConfig:
    """Decode over a paged cache: page_size-row pages of a shared pool, each
    sequence's live window scattered over randomly chosen physical pages;
    logical pages that left the window are marked -1 (evicted)."""
    name: str
    B: int
    H: int
    Hkv: int
    D: int
    W: int
    page_size: int
    pos_lo: int
    pos_hi: int
    seed: int = 7


@dataclass
class AppendConfig:
    """A chunk of C new tokens per sequence entering a W-slot ring cache."""
    name: str
    B: int
    C: int
    H: int
    Hkv: int
    D: int
    W: int
    pos_lo: int
    pos_hi: int
    seed: int = 8


PAGED_CONFIGS = {
    # the ring_decode workload's shapes with the cache in 256-row pages
    "paged_decode": PagedConfig("paged_decode", B=64, H=32, Hkv=8, D=128, W=4096, page_size=256,
                                pos_lo=4096, pos_hi=131072, seed=1007),
    "small_paged": PagedConfig("small_paged", B=5, H=8, Hkv=2, D=128, W=300, page_size=64,
                               pos_lo=0, pos_hi=1000, seed=2008),
}

APPEND_CONFIGS = {
    # chunked prefill / streaming: 64-token chunks into a Mistral-sized ring
    "ring_append": AppendConfig("ring_append", B=8, C=64, H=32, Hkv=8, D=128, W=4096,
                                pos_lo=4096, pos_hi=131072, seed=1009),
    "small_append": AppendConfig("small_append", B=4, C=37, H=8, Hkv=2, D=128, W=256,
                                 pos_lo=0, pos_hi=600, seed=2010),
}


def paged_inputs(cfg: PagedConfig, device="cpu"):
    """(q [B,H,D], k_pages, v_pages [P*page_size,Hkv,D], block_table [B,max_pages]
    int32, pos [B] int64).  The pool holds exactly the pages of the live
    windows, assigned to sequences in a seeded random order."""
    pos = uniform_int(cfg.B, cfg.pos_lo, cfg.pos_hi, cfg.seed, 3)
    ps = cfg.page_size
    first = [max(0, int(p) - cfg.W + 1) // ps for p in pos]
    last = [int(p) // ps for p in pos]
    n_live = [l - f + 1 for f, l in zip(first, last)]
    P = sum(n_live)
    perm = torch.randperm(P, generator=_gen(cfg.seed, 4, "cpu"))
    max_pages = max(last) + 1
    table = torch.full((cfg.B, max_pages), -1, dtype=torch.int32)
    k = 0
    for b in range(cfg.B):
        for lp in range(first[b], last[b] + 1):
            table[b, lp] = int(perm[k])
            k += 1
    q = normal((cfg.B, cfg.H, cfg.D), cfg.seed, 0, torch.bfloat16, device)
    kp = normal((P * ps, cfg.Hkv, cfg.D), cfg.seed, 1, torch.bfloat16, device)
    vp = normal((P * ps, cfg.Hkv, cfg.D), cfg.seed, 2, torch.bfloat16, device)
    return q, kp, vp, table, pos


def append_inputs(cfg: AppendConfig, device="cpu"):
    """(q [B,C,H,D], k_new, v_new [B,C,Hkv,D], k_ring, v_ring [B,W,Hkv,D], pos0 [B])."""
    q = normal((cfg.B, cfg.C, cfg.H, cfg.D), cfg.seed, 0, torch.bfloat16, device)
    kn = normal((cfg.B, cfg.C, cfg.Hkv, cfg.D), cfg.seed, 1, torch.bfloat16, device)
    vn = normal((cfg.B, cfg.C, cfg.Hkv, cfg.D), cfg.seed, 2, torch.bfloat16, device)
    kr = normal((cfg.B, cfg.W, cfg.Hkv, cfg.D), cfg.seed, 3, torch.bfloat16, device)
    vr = normal((cfg.B, cfg.W, cfg.Hkv, cfg.D), cfg.seed, 4, torch.bfloat16, device)
    pos0 = uniform_int(cfg.B, cfg.pos_lo, cfg.pos_hi, cfg.seed, 5)
    return q, kn, vn, kr, vr, pos0
