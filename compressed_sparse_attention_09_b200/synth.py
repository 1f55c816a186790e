"""Seeded synthetic inputs shaped like the CSA workloads.

This module only draws random numbers (torch's seeded CPU generator, normal
draws in fp32, rounded to bf16 where the workload is bf16); it holds none of
the method's arithmetic.  Both the CUDA path and the CPU oracle are fed from
it.

Distributions: H ~ N(0, 1); every projection weight ~ N(0, 1/fan_in) with
fan_in its number of rows (d for the H-side weights, d_c for the two
up-projections); the position biases ~ N(0, 0.1) (variance 0.1); decode
caches and ring rows ~ N(0, 1); ragged lengths ~ U[lo, hi] integers.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

from .capi import CSA_BF16, CSA_F32, Dims

WEIGHT_NAMES = ("W_aKV", "W_bKV", "W_aZ", "W_bZ", "B_a", "B_b", "W_aKV_I", "W_bKV_I", "W_aZ_I",
                "W_bZ_I", "B_a_I", "B_b_I", "W_DQ", "W_IUQ", "W_UQ", "W_w")


@dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    seqlens: tuple        # prefill: packed sequence lengths; decode: ()
    decode_batch: int = 0
    decode_pos: int = 0   # index t of the new token (decode)
    cache_cap: int = 0
    seed: int = 1000


def workloads():
    """The five workloads: tiny fp32, prefill n=8192, decode, long prefill, ragged prefill."""
    big = dict(d=4096, c=512, m=4, cI=128, nhI=64, dc=1536)
    ragged = tuple(int(x) for x in torch.randint(1024, 32769, (16,), generator=torch.Generator().manual_seed(1005)))
    return {
        "tiny": Workload("tiny", Dims(d=256, c=64, m=4, cI=32, nhI=4, nh=8, dc=128, topk=16, dtype=CSA_F32),
                         (256,), seed=1001),
        "prefill": Workload("prefill", Dims(nh=64, topk=512, dtype=CSA_BF16, **big), (8192,), seed=1002),
        "decode": Workload("decode", Dims(nh=128, topk=2048, dtype=CSA_BF16, **big), (), decode_batch=64,
                           decode_pos=65536, cache_cap=16384 + 64, seed=1003),
        "long": Workload("long", Dims(nh=64, topk=2048, dtype=CSA_BF16, **big), (131072,), seed=1004),
        "ragged": Workload("ragged", Dims(nh=64, topk=1024, dtype=CSA_BF16, **big), ragged, seed=1005),
    }


def torch_dtype(dims: Dims):
    return torch.bfloat16 if dims.dtype == CSA_BF16 else torch.float32


def _normal(shape, std, gen, dtype):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def make_weights(dims: Dims, seed: int):
    """Dict of CPU tensors, each [in, out] as on the page, in the workload's dtype."""
    g = torch.Generator().manual_seed(seed)
    dt = torch_dtype(dims)
    d, c, m, cI, nhI, nh, dc = dims.d, dims.c, dims.m, dims.cI, dims.nhI, dims.nh, dims.dc
    shapes = {
        "W_aKV": ((d, c), d), "W_bKV": ((d, c), d), "W_aZ": ((d, c), d), "W_bZ": ((d, c), d),
        "B_a": ((m, c), None), "B_b": ((m, c), None),
        "W_aKV_I": ((d, cI), d), "W_bKV_I": ((d, cI), d), "W_aZ_I": ((d, cI), d), "W_bZ_I": ((d, cI), d),
        "B_a_I": ((m, cI), None), "B_b_I": ((m, cI), None),
        "W_DQ": ((d, dc), d), "W_IUQ": ((dc, nhI * cI), dc), "W_UQ": ((dc, nh * c), dc), "W_w": ((d, nhI), d),
    }
    out = {}
    for name in WEIGHT_NAMES:
        shape, fan_in = shapes[name]
        std = math.sqrt(0.1) if fan_in is None else 1.0 / math.sqrt(fan_in)
        out[name] = _normal(shape, std, g, dt)
    return out


def make_hidden(T: int, dims: Dims, seed: int):
    g = torch.Generator().manual_seed(seed + 7919)
    return _normal((T, dims.d), 1.0, g, torch_dtype(dims))


def make_normal(shape, dims: Dims, seed: int, std: float = 1.0):
    """Generic seeded N(0, std^2) tensor in the workload's dtype (stage inputs, caches, rings)."""
    g = torch.Generator().manual_seed(seed)
    return _normal(shape, std, g, torch_dtype(dims))


def scaled(w: Workload, **dims_over) -> Workload:
    """The same workload with some dimensions replaced (smaller parity cases)."""
    return replace(w, dims=replace(w.dims, **dims_over))
