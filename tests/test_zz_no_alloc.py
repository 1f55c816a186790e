"""GPU test of csa_indexer_topk_noalloc, the indexer entry point for callers
that cannot allocate device memory (e.g. code whose device memory belongs to
another framework's pool, or a loop that must not allocate after start-up).

It calls the entry point through the C ABI twice in a row, on two different
seeded problems, and checks each result against csa_indexer_topk (the
workspace entry point) on the same inputs.  Both run the same tensor-core
kernel, so the index rows must be identical.  The second call also shows
that the scratch contents the first call left behind do not leak into the
next result.  This file is collected last on purpose (its name sorts last)."""
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(dims, lens, seed):
    T = sum(lens)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    qI = synth.make_normal((T, dims.nhI * dims.cI), dims, seed).to(DEV)
    wI = synth.make_normal((T, dims.nhI), dims, seed + 1).float().to(DEV)
    KI = synth.make_normal((NB, dims.cI), dims, seed + 2, std=0.5).to(DEV)
    return T, NB, cu.to(DEV), cb.to(DEV), qI, wI, KI


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_indexer_matches_workspace_entry(call):
    dims = csa.Dims(d=64, c=64, m=4, cI=128, nhI=64, nh=2, dc=64, topk=100, dtype=csa.CSA_BF16)
    cases = [([3000, 517, 9], 301), ([2048, 13, 4000], 302)]
    for lens, seed in cases:          # two calls in a row, different inputs
        T, NB, cu, cb, qI, wI, KI = _problem(dims, lens, seed + 10 * call)
        args = (dims, qI, dims.nhI * dims.cI, wI, dims.nhI, KI, cu, cb, len(lens), T, NB, max(lens))
        want = torch.full((T, dims.topk), -7, dtype=torch.int32, device=DEV)
        ws = torch.empty(csa.csa_indexer_workspace_bytes(dims, T, len(lens), max(lens)), dtype=torch.uint8,
                         device=DEV)
        csa.csa_indexer_topk(*args, want, ws)
        got = torch.full((T, dims.topk), -7, dtype=torch.int32, device=DEV)
        csa.csa_indexer_topk_noalloc(*args, got)
        assert csa.csa_get_device_status() == 0
        assert torch.equal(got, want)


def test_noalloc_indexer_rejects_sizes_beyond_its_scratch():
    dims = csa.Dims(d=64, c=64, m=4, cI=128, nhI=64, nh=2, dc=64, topk=100, dtype=csa.CSA_BF16)
    T, NB, cu, cb, qI, wI, KI = _problem(dims, [64], 303)
    idx = torch.empty((T, dims.topk), dtype=torch.int32, device=DEV)
    with pytest.raises(csa.CsaError) as e:
        csa.csa_indexer_topk_noalloc(dims, qI, dims.nhI * dims.cI, wI, dims.nhI, KI, cu, cb, 1, T, NB,
                                     4 * 4096, idx)     # max_seqlen beyond the fixed scratch
    assert e.value.status == 2   # CSA_ERR_UNSUPPORTED


def test_noalloc_indexer_understated_max_seqlen_is_flagged():
    """A max_seqlen below a sequence's real length would make the later
    queries' score rows overrun the fixed scratch rows; those items are
    skipped and flagged instead, and the next call works normally."""
    dims = csa.Dims(d=64, c=64, m=4, cI=128, nhI=64, nh=2, dc=64, topk=100, dtype=csa.CSA_BF16)
    T, NB, cu, cb, qI, wI, KI = _problem(dims, [6000], 304)
    idx = torch.empty((T, dims.topk), dtype=torch.int32, device=DEV)
    csa.csa_indexer_topk_noalloc(dims, qI, dims.nhI * dims.cI, wI, dims.nhI, KI, cu, cb, 1, T, NB, 1000, idx)
    assert csa.csa_get_device_status() == 6   # CSA_ERR_BAD_METADATA
    args = (dims, qI, dims.nhI * dims.cI, wI, dims.nhI, KI, cu, cb, 1, T, NB, T)
    want = torch.empty_like(idx)
    ws = torch.empty(csa.csa_indexer_workspace_bytes(dims, T, 1, T), dtype=torch.uint8, device=DEV)
    csa.csa_indexer_topk(*args, want, ws)
    csa.csa_indexer_topk_noalloc(*args, idx)
    assert csa.csa_get_device_status() == 0
    assert torch.equal(idx, want)
