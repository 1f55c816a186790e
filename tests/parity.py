"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same seeded inputs.

Comparison protocol (tolerances of the bf16 and fp32 configurations):
* top-k sets (eq. 9 of "Compressed Sparse Attention", cnblogs; the exactness
  bar is a gap of 1e-3 relative to the k-th score, ties to the lower block).
  Every candidate score I_s the oracle computes carries an admissible
  perturbation delta_s >= 0: the worst-case error of evaluating eq. (8) in
  fp32 from the same inputs (fp32_score_bound), plus, end to end in bf16,
  that candidate's own bf16-storage sensitivity |I_bf16(s) - I_exact(s)|
  (both sides round their own projections to bf16, and a stored element may
  land on the neighbouring bf16 value).  Let top be the oracle's set and
      lo = min_{s in top} (I_s - delta_s),  hi = max_{u not in top} (I_u + delta_u).
  If lo - hi > 1e-3 |I_(k)| the set is stable under every admissible
  perturbation and the GPU set must equal it exactly ("required").  With all
  delta_s = 0 this is exactly "I_(k) - I_(k+1) > 1e-3 |I_(k)|".  Otherwise the
  GPU set must be a correct top-k of some admissible perturbation of the
  scores, i.e. min_{s in gpu} (I_s + delta_s) >= max_{u not in gpu}
  (I_u - delta_u) - 1e-3 |I_(k)|, with k_eff distinct visible blocks in
  ascending order and -1 padding.
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


# Rounding unit of one fp32 operation in the bound below: 2^-23, twice the
# round-to-nearest unit, so that accumulation that truncates (as a tensor
# core's adder may) is covered as well.
U32 = 2.0 ** -23


def fp32_score_bound(qI_t, wI_t, KI_avail):
    """Worst-case |I_fp32(t, s) - I_exact(t, s)| of eq. (8) evaluated in fp32
    arithmetic (any summation order) from the same inputs, per visible block.

    qI_t [n_h^I, c^I], wI_t [n_h^I], KI_avail [avail, c^I].  Each term
    w_h * ReLU(q_h . K_s) is a c^I-term dot product (products of bf16 values
    are exact in fp32; one more rounding each for fp32 inputs), a ReLU
    (exact), a product with w_h and a sum over n_h^I heads, so the standard
    summation bound gives gamma_n * sum_h |w_h| sum_j |q_hj K_sj| with
    n = c^I + n_h^I + 2 and gamma_n = n u / (1 - n u)."""
    KI_avail = np.asarray(KI_avail, dtype=np.float64)
    if KI_avail.shape[0] == 0:
        return np.zeros(0)
    q, w = np.abs(np.asarray(qI_t, dtype=np.float64)), np.abs(np.asarray(wI_t, dtype=np.float64))
    n = q.shape[1] + q.shape[0] + 2
    gamma = n * U32 / (1.0 - n * U32)
    return gamma * (w @ (q @ np.abs(KI_avail).T))


def score_delta(scores_store, scores_exact, qI_t, wI_t, KI_avail):
    """Admissible perturbation of each candidate score of one row: the fp32
    evaluation bound plus, where given, the candidate's own bf16-storage
    sensitivity |I_bf16(s) - I_exact(s)| from the oracle."""
    d = fp32_score_bound(qI_t, wI_t, KI_avail)
    if scores_exact is not None:
        d = d + np.abs(np.asarray(scores_store, dtype=np.float64) - np.asarray(scores_exact, dtype=np.float64))
    return d


def check_topk_row(gpu_row, scores, k, delta=None, gap_rel=GAP_REL):
    """Check one GPU top-k row against the oracle's fp64 scores under the
    protocol of this module.  delta: per-candidate admissible perturbation
    (None = 0).  gap_rel: the relative margin (1e-3 of the k-th score; stage
    tests, whose two sides see bit-identical inputs, pass 0 and so demand
    exactness wherever the set is stable under the fp32 evaluation bound
    alone, which is stricter).  Returns "all" (k_eff = avail: every block),
    "required" (stable set, matched exactly), "equal" (not required but
    equal) or "valid" (a correct top-k of an admissible perturbation)."""
    gpu_row = np.asarray(gpu_row, dtype=np.int64)
    scores = np.asarray(scores, dtype=np.float64)
    avail = len(scores)
    keff = min(k, avail)
    assert np.all(gpu_row[keff:] == -1), "padding must be -1"
    sel = gpu_row[:keff]
    assert np.all(np.diff(sel) > 0), "indices must be distinct and ascending"
    assert keff == 0 or (sel[0] >= 0 and sel[-1] < avail), "indices must be visible blocks"
    if keff == avail:
        assert np.array_equal(sel, np.arange(avail))
        return "all"
    delta = np.zeros(avail) if delta is None else np.asarray(delta, dtype=np.float64)
    want = orc.topk_select(scores, k)[:keff]
    Ik = np.sort(scores)[::-1][keff - 1]
    bar = gap_rel * abs(Ik)
    top = np.zeros(avail, dtype=bool)
    top[want] = True
    lo = float((scores - delta)[top].min())
    hi = float((scores + delta)[~top].max())
    if lo - hi > bar:
        assert np.array_equal(sel, want), \
            f"stable set differs: net gap {(lo - hi) / max(abs(Ik), 1e-300):.2e} of |I_(k)|"
        return "required"
    if np.array_equal(sel, want):
        return "equal"
    mine = np.zeros(avail, dtype=bool)
    mine[sel] = True
    lo_g = float((scores + delta)[mine].min())
    hi_g = float((scores - delta)[~mine].max())
    assert lo_g >= hi_g - bar, \
        f"not a top-k of any admissible perturbation: {lo_g:.6g} < {hi_g:.6g} - {bar:.3g}"
    return "valid"


def new_counts():
    return {"all": 0, "required": 0, "equal": 0, "valid": 0}


def report(name, counts):
    """Prints the row classification of one test (shown with pytest -s or on failure)."""
    n = sum(counts.values())
    print(f"[topk parity] {name}: {n} rows: {counts}")
    return counts
