"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same seeded inputs.

Comparison protocol (tolerances of the bf16 and fp32 configurations):
* top-k sets: where the oracle's k-th / (k+1)-th score gap exceeds 1e-3
  relative, the GPU set must equal the oracle's exactly; below that gap the
  set must be valid (k_eff distinct visible blocks, each with an oracle score
  within the bar of the k-th score).  Relative here means relative to
  max(|I_(k)|, 1e-2 * max_s |I_s|), so that a k-th score that happens to sit
  near zero does not demand more than fp32 can resolve.  Stage tests feed
  both sides bit-identical inputs and use exactly this bar.  End-to-end bf16
  tests widen it by the score perturbation that bf16 storage rounding itself
  causes in the oracle (rounding_sensitivity): there both sides round their
  own projections to bf16 and a few stored elements legitimately land on
  neighbouring bf16 values.
* outputs: the GPU output o_t is compared with eq. (11) evaluated by the
  oracle on the GPU's own index set (this isolates the attention error from
  the selection): bf16 max-abs <= 2e-2 and relative L2 <= 1e-2; fp32
  max-abs <= 1e-5 and relative L2 <= 1e-5.
* compressed entries: bf16 max-abs <= 2e-2 and relative L2 <= 1e-2; fp32
  max-abs <= 1e-5.
"""
from __future__ import annotations

import numpy as np
import torch

import compressed_sparse_attention_09_b200 as csa
from oracle import csa_oracle as orc

GAP_REL = 1e-3
TOL = {csa.CSA_BF16: dict(max_abs=2e-2, rel_l2=1e-2), csa.CSA_F32: dict(max_abs=1e-5, rel_l2=1e-5)}


def store_mode(dims):
    return "bf16" if dims.dtype == csa.CSA_BF16 else "f32"


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def weights_f64(W):
    return {k: f64(v) for k, v in W.items()}


def gpu_pack(dims, W_cpu, dev="cuda"):
    Wd = {k: v.to(dev) for k, v in W_cpu.items()}
    packed = torch.empty(csa.csa_packed_weights_bytes(dims), dtype=torch.uint8, device=dev)
    csa.csa_pack_weights(dims, Wd, packed)
    return packed


def gpu_forward(dims, W_cpu, H_cpu, seqlens, dev="cuda", packed=None):
    """Runs csa_forward; returns CPU tensors O [T, nh, c], C_comp, K_icomp, idx."""
    T = H_cpu.shape[0]
    cu, cb = csa.cu_from_lengths(seqlens, dims.m)
    NB = int(cb[-1])
    dt = H_cpu.dtype
    if packed is None:
        packed = gpu_pack(dims, W_cpu, dev)
    H = H_cpu.to(dev)
    O = torch.empty(T, dims.nh * dims.c, dtype=dt, device=dev)
    Cc = torch.empty(max(NB, 1), dims.c, dtype=dt, device=dev)
    KI = torch.empty(max(NB, 1), dims.cI, dtype=dt, device=dev)
    idx = torch.empty(T, dims.topk, dtype=torch.int32, device=dev)
    ws = torch.empty(csa.csa_forward_workspace_bytes(dims, T, len(seqlens)), dtype=torch.uint8, device=dev)
    csa.csa_forward(dims, packed, H, cu.to(dev), cb.to(dev), len(seqlens), T, NB, max(seqlens), O,
                    Cc, KI, idx, ws)
    st = csa.csa_get_device_status()
    assert st == 0, csa.status_string(st)
    return {"O": O.cpu().view(T, dims.nh, dims.c), "C_comp": Cc.cpu()[:NB], "K_icomp": KI.cpu()[:NB],
            "idx": idx.cpu()}


def compare_dense(got, want, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    tol = TOL[dtype]
    err = np.abs(got - want)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(want)) or 1.0
    rel = float(np.linalg.norm(got - want)) / denom
    assert max_abs <= tol["max_abs"] and rel <= tol["rel_l2"], \
        f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e} (tol {tol})"
    return max_abs, rel


def check_topk_row(gpu_row, scores, k, extra_tol=0.0):
    """Check one GPU top-k row against the oracle's fp64 scores; returns 'exact'/'valid'.

    extra_tol (absolute) widens the gap bar where the two sides do not see
    bit-identical inputs (end-to-end runs, where both round their own fp32 /
    fp64 projections to bf16 and so may store neighbouring bf16 values)."""
    gpu_row = np.asarray(gpu_row, dtype=np.int64)
    avail = len(scores)
    keff = min(k, avail)
    assert np.all(gpu_row[keff:] == -1), "padding must be -1"
    sel = gpu_row[:keff]
    assert np.all(np.diff(sel) > 0), "indices must be distinct and ascending"
    assert keff == 0 or (sel[0] >= 0 and sel[-1] < avail), "indices must be visible blocks"
    if keff == avail:
        assert np.array_equal(sel, np.arange(avail))
        return "exact"
    want = orc.topk_select(scores, k)[:keff]
    srt = np.sort(scores)[::-1]
    Ik, Ik1 = srt[keff - 1], srt[keff]
    denom = max(abs(Ik), 1e-2 * float(np.abs(scores).max()), 1e-300)
    bar = max(GAP_REL * denom, extra_tol)
    if Ik - Ik1 > bar:
        assert np.array_equal(sel, want), f"set differs with gap {(Ik - Ik1) / denom:.2e} (bar {bar / denom:.2e})"
        return "exact"
    assert np.all(scores[sel] >= Ik - bar), "a chosen block scores below the k-th"
    return "valid"


def rounding_sensitivity(scores_bf16, scores_exact):
    """Score perturbation caused by bf16 storage rounding alone, from the oracle:
    max_s |I_bf16(t, s) - I_exact(t, s)| over one row (0 for an empty row)."""
    if len(scores_bf16) == 0:
        return 0.0
    return float(np.abs(np.asarray(scores_bf16) - np.asarray(scores_exact)).max())
