"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module only draws random numbers and holds the workload shapes; it holds
none of the attention arithmetic, so both the CUDA path and the fp64 oracle
can be fed from it without sharing any of the method's code.

Recipe (the same on every machine, CPU generator, so the GPU and the oracle
see identical values):

* ``torch.Generator('cpu').manual_seed(seed)``;
* ``torch.randn(shape, dtype=float32)`` for q, k, v and, when asked, dO, in
  that order, each [B, H, N, d];
* FP8 workload only: after the randn draws, for q, k, v in turn, a mask
  ``torch.rand(shape) < 1e-3`` from the same generator marks the outliers,
  which are multiplied by 20;
* finally ``.to(torch.bfloat16)`` (round to nearest even).

The Hadamard sign vector is drawn here too (``signs``), so the rotation's
randomness is an input to both sides rather than something either recomputes.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: Tuple[bool, ...]
    seed: int
    backward: bool = False
    fp8: bool = False
    note: str = ""


# The workloads of the pages' kind of kernel micro-benchmark ("sequences >= 1K",
# short contexts, d in {64, 128}); synthetic stand-ins, no public suite.
TINY = Workload("attn_fwd_B1_H1_N128_d64", 1, 1, 128, 64, (False,), seed=0,
                note="single tile, launch-latency bound")
SMALL = Workload("attn_fwd_B2_H8_N1024_d64", 2, 8, 1024, 64, (True, False), seed=1,
                 note="128 query tiles, fewer than the 148 SMs")
LONG = Workload("attn_fwdbwd_B4_H16_N4096_d128_causal", 4, 16, 4096, 128, (True,), seed=2,
                backward=True, note="tensor-core bound forward and backward")
FP8 = Workload("attn_fp8_B2_H16_N8192_d128", 2, 16, 8192, 128, (False,), seed=3,
               fp8=True, note="E4M3 with 0.1% x20 outliers, rotation on/off")
SIGN_SEED = 4


def sweep() -> Tuple[Workload, ...]:
    """B*N = 16384 tokens, hidden 2048 split as (H=32, d=64) and (H=16, d=128)."""
    out = []
    idx = 0
    for hd in ((32, 64), (16, 128)):
        for n in (512, 1024, 2048, 4096, 8192, 16384):
            out.append(Workload(f"sweep_N{n}_H{hd[0]}_d{hd[1]}", 16384 // n, hd[0], n, hd[1],
                                (True, False), seed=10 + idx, backward=True))
            idx += 1
    return tuple(out)


def make_qkv(B: int, H: int, N: int, d: int, seed: int, with_do: bool = False,
             outliers: bool = False):
    """CPU bf16 tensors (q, k, v[, do]) of shape [B, H, N, d] from ``seed``."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shape = (B, H, N, d)
    names = ["q", "k", "v"] + (["do"] if with_do else [])
    t = {n: torch.randn(shape, dtype=torch.float32, generator=g) for n in names}
    if outliers:
        for n in ("q", "k", "v"):
            mask = torch.rand(shape, generator=g) < 1e-3
            t[n] = torch.where(mask, t[n] * 20.0, t[n])
    out = tuple(t[n].to(torch.bfloat16) for n in names)
    return out


def make_gqa(B: int, H: int, H_kv: int, N: int, d: int, seed: int, with_do: bool = False,
             outliers: bool = False):
    """CPU bf16 (q, k, v[, do]) with grouped K/V heads: q, do [B, H, N, d];
    k, v [B, H_kv, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shapes = {"q": (B, H, N, d), "k": (B, H_kv, N, d), "v": (B, H_kv, N, d), "do": (B, H, N, d)}
    names = ["q", "k", "v"] + (["do"] if with_do else [])
    t = {n: torch.randn(shapes[n], dtype=torch.float32, generator=g) for n in names}
    if outliers:
        for n in ("q", "k", "v"):
            mask = torch.rand(shapes[n], generator=g) < 1e-3
            t[n] = torch.where(mask, t[n] * 20.0, t[n])
    return tuple(t[n].to(torch.bfloat16) for n in names)


def make_workload(w: Workload):
    return make_qkv(w.B, w.H, w.N, w.d, w.seed, with_do=w.backward, outliers=w.fp8)


def signs(d: int, seed: int = SIGN_SEED) -> torch.Tensor:
    """Random +-1 vector of length d (float32, CPU) for the Hadamard rotation."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    bits = torch.randint(0, 2, (d,), generator=g)
    return (bits * 2 - 1).to(torch.float32)
