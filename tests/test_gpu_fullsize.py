"""Full-size parity of the long (n = 131072, k = 2048) and ragged (16 packed
sequences, k = 1024) prefill workloads, in the launch configuration bench.py
times.  Every compressed entry and indexer key is compared; top-k sets and
outputs are checked on at least 128 sampled rows per workload (the first 2m
rows of the first sequences, every sequence's k-clamp transition t = m k - 1
.. m k + m and last row, and seeded random rows), against the memory-light
oracle form on the same seeded inputs, under the protocol of parity.py."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth
from oracle import csa_oracle as orc
from parity import check_topk_row, compare_dense, f64, gpu_pack, new_counts, report, score_delta, weights_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_forward_rows(dims, W, H_cpu, seqlens, rows):
    """csa_forward on the device; returns C^Comp, K^IComp and the sampled rows of O and idx."""
    T = H_cpu.shape[0]
    cu, cb = csa.cu_from_lengths(seqlens, dims.m)
    NB = int(cb[-1])
    packed = gpu_pack(dims, W)
    H = H_cpu.to(DEV)
    O = torch.empty(T, dims.nh * dims.c, dtype=H.dtype, device=DEV)
    Cc = torch.empty(NB, dims.c, dtype=H.dtype, device=DEV)
    KI = torch.empty(NB, dims.cI, dtype=H.dtype, device=DEV)
    idx = torch.empty(T, dims.topk, dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.csa_forward_workspace_bytes(dims, T, len(seqlens)), dtype=torch.uint8, device=DEV)
    csa.csa_forward(dims, packed, H, cu.to(DEV), cb.to(DEV), len(seqlens), T, NB, max(seqlens), O, Cc, KI, idx, ws)
    st = csa.csa_get_device_status()
    assert st == 0, csa.status_string(st)
    r = torch.as_tensor(rows, device=DEV)
    out = {"C_comp": Cc.cpu(), "K_icomp": KI.cpu(), "O": O[r].cpu().view(len(rows), dims.nh, dims.c),
           "idx": idx[r].cpu()}
    del O, ws, idx, H
    torch.cuda.empty_cache()
    return out


def sample_rows(seqlens, m, k, seed, n_rows=128):
    cu = np.concatenate([[0], np.cumsum(seqlens)])
    rng = np.random.default_rng(seed)
    rows = set()
    for b, L in enumerate(seqlens):
        if b < 2:
            rows |= {int(cu[b]) + t for t in range(min(L, 2 * m))}
        rows |= {int(cu[b]) + t for t in range(m * k - 1, m * k + m + 1) if t < L}   # around the k clamp
        rows.add(int(cu[b + 1]) - 1)
    while len(rows) < n_rows:
        rows.add(int(rng.integers(0, int(cu[-1]))))
    return sorted(rows)


def run_fullsize(name):
    w = synth.workloads()[name]
    dims, lens = w.dims, list(w.seqlens)
    W = synth.make_weights(dims, w.seed)
    H = synth.make_hidden(sum(lens), dims, w.seed)
    rows = sample_rows(lens, dims.m, dims.topk, w.seed)
    g = gpu_forward_rows(dims, W, H, lens, rows)
    od = dict(m=dims.m, topk=dims.topk, nh=dims.nh, nhI=dims.nhI, c=dims.c, cI=dims.cI)
    W64 = weights_f64(W)
    o = orc.csa_forward_sampled(H, W64, od, lens, rows, store="bf16")
    compare_dense(f64(g["C_comp"]), o["C_comp"], dims.dtype, "C_comp")
    compare_dense(f64(g["K_icomp"]), o["K_icomp"], dims.dtype, "K_icomp")
    ox = orc.csa_forward_sampled(H, W64, od, lens, rows, store="exact")
    cu = np.concatenate([[0], np.cumsum(lens)])
    counts = new_counts()
    want = np.zeros((len(rows), dims.nh, dims.c))
    for r, t in enumerate(rows):
        gi = g["idx"][r].numpy()
        b = int(np.searchsorted(cu, t, side="right") - 1)
        base, avail = int(o["cu_blocks"][b]), int(t - cu[b]) // dims.m
        delta = score_delta(o["scores"][r], ox["scores"][r], o["qI"][r], o["wI"][r],
                            o["K_icomp"][base:base + avail])
        counts[check_topk_row(gi, o["scores"][r], dims.topk, delta)] += 1
        sel = gi[gi >= 0]
        want[r] = orc.core_attn(o["q"][r], o["C_comp"][base + sel])
    compare_dense(f64(g["O"]), want, dims.dtype, "O")
    assert sum(counts.values()) == len(rows) >= 128
    return report(f"{name} full size", counts)


def test_long_prefill_full_size_sampled_rows():
    c = run_fullsize("long")
    # k = 2048 of up to 32768 blocks: the k / (k+1) gap is almost always below
    # the candidates' bf16-storage perturbation (oracle alone: 1 stable set in
    # 106 selection rows); every other row must pass the validity rule
    assert c["required"] >= 1, c


def test_ragged_prefill_full_size_sampled_rows():
    c = run_fullsize("ragged")
    assert c["required"] >= 0.4 * (c["required"] + c["equal"] + c["valid"]), c   # oracle alone: 16 of 32
