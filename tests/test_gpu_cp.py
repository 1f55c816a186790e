"""Context-parallel prefill on the GPU (csa_cp_compress / csa_cp_queries
driven by cp.CpPrefill): the ranks of a 2- and 4-way split run one after
another in this process (their kernels never wait on one another; the
all-gather is stood in for by stacking every rank's send buffer), and the
result must be bit-identical to csa_forward over the whole sequence:
outputs, top-k rows and the assembled C^Comp / K^IComp."""
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import cp, synth
from parity import gpu_pack

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_cp(dims, n, world, seed):
    W = synth.make_weights(dims, seed)
    packed = gpu_pack(dims, W)
    H = synth.make_hidden(n, dims, seed).to(DEV)
    # whole-sequence reference
    cu, cb = csa.cu_from_lengths([n], dims.m)
    NB = int(cb[-1])
    dt = H.dtype
    O = torch.empty(n, dims.nh * dims.c, dtype=dt, device=DEV)
    Cc = torch.empty(NB, dims.c, dtype=dt, device=DEV)
    KI = torch.empty(NB, dims.cI, dtype=dt, device=DEV)
    idx = torch.empty(n, dims.topk, dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.csa_forward_workspace_bytes(dims, n, 1), dtype=torch.uint8, device=DEV)
    csa.csa_forward(dims, packed, H, cu.to(DEV), cb.to(DEV), 1, n, NB, n, O, Cc, KI, idx, ws)
    assert csa.csa_get_device_status() == 0
    # every rank in turn: compress, then (after all ranks) the gather, then queries
    ranks = [cp.CpPrefill(dims, packed, n, world, r, DEV) for r in range(world)]
    sends = {}
    chunks, owner = cp.zigzag_plan(n, world, dims.m)
    max_blocks = max(ch.length // dims.m for ch in chunks)
    for r, rk in enumerate(ranks):
        ent = [rk.compress(H, chunks[j]) for j in owner[r]]
        sends[r] = cp.pack_entries(ent, max_blocks)
    gathered = torch.stack([sends[r] for r in range(world)])
    for r, rk in enumerate(ranks):
        out = rk.forward(H, gather_fn=lambda send: gathered)
        assert torch.equal(rk.C, Cc) and torch.equal(rk.KI, KI)
        for j, Oj in out.items():
            ch = chunks[j]
            sl = slice(ch.start, ch.start + ch.length)
            assert torch.equal(rk.bufs[j]["idx"], idx[sl]), f"rank {r} chunk {j}: top-k rows differ"
            assert torch.equal(Oj, O[sl]), f"rank {r} chunk {j}: outputs differ"
    assert csa.csa_get_device_status() == 0


@pytest.mark.parametrize("world", [2, 4])
def test_cp_bf16_tensor_core_matches_whole_sequence(world):
    dims = csa.Dims(d=256, c=512, m=4, cI=128, nhI=64, nh=64, dc=128, topk=64, dtype=csa.CSA_BF16)
    run_cp(dims, 2048 + 37, world, 401)


def test_cp_bf16_small_dims_matches_whole_sequence():
    dims = csa.Dims(d=256, c=128, m=4, cI=64, nhI=16, nh=4, dc=128, topk=24, dtype=csa.CSA_BF16)
    run_cp(dims, 1501, 2, 402)


def test_cp_fp32_matches_whole_sequence():
    dims = csa.Dims(d=128, c=64, m=2, cI=32, nhI=4, nh=4, dc=64, topk=8, dtype=csa.CSA_F32)
    run_cp(dims, 403, 2, 403)


def test_cp_prefill_full_size_matches_whole_sequence():
    """The n = 8192 prefill workload split over 4 ranks."""
    w = synth.workloads()["prefill"]
    run_cp(w.dims, 8192, 4, w.seed)
