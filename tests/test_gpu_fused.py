"""The H-side projection with the compression in its epilogue
(csa_project_hidden_compress, eqs. 1-5 and 7 of "Compressed Sparse
Attention", cnblogs), against the unfused pair csa_project_hidden +
csa_compress_kv on the same inputs (bit-identical: same bf16 storage point,
same per-channel arithmetic) and against the oracle's compression of its
own projections.  The packings put block windows across 128-token tile
boundaries at many offsets: ragged tails, sequences shorter than m,
sequences that start mid-tile, i = 0 entries on both sides of a boundary."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth
from oracle import csa_oracle as orc
from parity import compare_dense, f64, gpu_pack

pytestmark = pytest.mark.gpu
DEV = "cuda"

LENS = [517, 3, 130, 1031, 255, 129, 1, 4, 8, 600, 121, 7]

H_SIDE = ("W_aKV", "W_bKV", "W_aZ", "W_bZ", "W_aKV_I", "W_bKV_I", "W_aZ_I", "W_bZ_I")


def run_both(dims, lens, seed):
    T = sum(lens)
    W = synth.make_weights(dims, seed)
    packed = gpu_pack(dims, W)
    H = synth.make_hidden(T, dims, seed)
    Hd = H.to(DEV)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    cu, cb = cu.to(DEV), cb.to(DEV)
    N1b = csa.csa_hidden_row_elems(dims)
    # unfused: projection rows, then both key sets
    Y1 = torch.empty(T, N1b, dtype=torch.bfloat16, device=DEV)
    wI = torch.empty(T, dims.nhI, dtype=torch.float32, device=DEV)
    Cc = torch.empty(max(NB, 1), dims.c, dtype=torch.bfloat16, device=DEV)
    KI = torch.empty(max(NB, 1), dims.cI, dtype=torch.bfloat16, device=DEV)
    csa.csa_project_hidden(dims, packed, Hd, T, Y1, wI)
    csa.csa_compress_kv(dims, packed, Y1, T, cu, cb, len(lens), NB, Cc, KI)
    # fused (outputs pre-filled with a pattern that must be overwritten)
    fY1 = torch.full((T, N1b), 7.0, dtype=torch.bfloat16, device=DEV)
    fwI = torch.full((T, dims.nhI), 7.0, dtype=torch.float32, device=DEV)
    fCc = torch.full((max(NB, 1), dims.c), 7.0, dtype=torch.bfloat16, device=DEV)
    fKI = torch.full((max(NB, 1), dims.cI), 7.0, dtype=torch.bfloat16, device=DEV)
    ws = torch.full((csa.csa_project_compress_workspace_bytes(dims, T),), 0x5A, dtype=torch.uint8, device=DEV)
    for _ in range(2):   # twice: the boundary counters must come back to zero
        csa.csa_project_hidden_compress(dims, packed, Hd, T, cu, cb, len(lens), NB, fY1, fwI, fCc, fKI, ws)
    assert csa.csa_get_device_status() == 0
    q0 = 4 * dims.c + 4 * dims.cI
    assert torch.equal(fCc[:NB], Cc[:NB]), "C^Comp differs from the unfused path"
    assert torch.equal(fKI[:NB], KI[:NB]), "K^IComp differs from the unfused path"
    assert torch.equal(fY1[:, q0:], Y1[:, q0:]), "c^Q differs from the unfused path"
    assert torch.equal(fwI, wI), "w^I differs from the unfused path"
    # against the oracle's compression of its own (bf16-stored) projections
    W64 = {k: f64(v) for k, v in W.items()}
    proj = [orc.storage_round(orc.project(f64(H), W64[n]), "bf16") for n in H_SIDE]
    cuh = np.concatenate([[0], np.cumsum(lens)])
    wantC, wantK = [], []
    for b in range(len(lens)):
        sl = slice(int(cuh[b]), int(cuh[b + 1]))
        wantC.append(orc.compress(*(p[sl] for p in proj[:4]), W64["B_a"], W64["B_b"], dims.m))
        wantK.append(orc.compress(*(p[sl] for p in proj[4:]), W64["B_a_I"], W64["B_b_I"], dims.m))
    compare_dense(f64(fCc[:NB].cpu()), orc.round_bf16(np.concatenate(wantC)), dims.dtype, "C_comp")
    compare_dense(f64(fKI[:NB].cpu()), orc.round_bf16(np.concatenate(wantK)), dims.dtype, "K_icomp")
    return NB


@pytest.mark.parametrize("m", [1, 2, 4, 8])
def test_fused_projection_compression_matches_unfused(m):
    dims = csa.Dims(d=256, c=128, m=m, cI=64, nhI=16, nh=4, dc=128, topk=8, dtype=csa.CSA_BF16)
    assert run_both(dims, LENS, 300 + m) > 0


def test_fused_projection_compression_full_widths():
    """c = 512, c^I = 128 (ten channel groups), d = 4096, d_c = 1536, n_h^I = 64."""
    w = synth.workloads()["prefill"]
    assert run_both(w.dims, [1500, 77, 2048, 130], 311) > 0


def test_fused_projection_compression_single_tile_and_empty_tail():
    dims = csa.Dims(d=256, c=64, m=4, cI=64, nhI=16, nh=4, dc=128, topk=8, dtype=csa.CSA_BF16)
    run_both(dims, [3], 312)            # no block at all
    run_both(dims, [128], 313)          # one full tile
    run_both(dims, [127, 1, 128], 314)  # a boundary between two sequences
