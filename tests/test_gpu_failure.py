"""GPU tests of the failure detection: a bounded device wait that runs out
ends with CSA_ERR_DEVICE_TIMEOUT and leaves the context usable, and
inconsistent sequence metadata is flagged (CSA_ERR_BAD_METADATA) without any
access outside the buffers.  Nothing here faults, traps or hangs the GPU:
the wait that runs out waits on a barrier nothing arrives on, under a 2 ms
limit, and the bad metadata is clamped or skipped by the kernels."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
DEFAULT_WAIT_NS = 1_500_000_000


def _small_mqa(dims, lens, cu_blocks=None):
    T = sum(lens)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    if cu_blocks is not None:
        cb = torch.as_tensor(cu_blocks, dtype=torch.int32)
    q = synth.make_normal((T, dims.nh * dims.c), dims, 91).to(DEV)
    C = synth.make_normal((max(NB, 1), dims.c), dims, 92).to(DEV)
    idx = torch.full((T, dims.topk), -1, dtype=torch.int32)
    for b, L in enumerate(lens):
        for t in range(L):
            a = min(t // dims.m, dims.topk)
            idx[int(cu[b]) + t, :a] = torch.arange(a)
    O = torch.empty(T, dims.nh * dims.c, dtype=q.dtype, device=DEV)
    csa.csa_sparse_mqa(dims, q, dims.nh * dims.c, C, idx.to(DEV), cu.to(DEV), cb.to(DEV), len(lens), T, NB, O)
    return csa.csa_get_device_status(), O


def test_bounded_wait_runs_out_and_reports_timeout():
    csa.csa_set_wait_limit_ns(2_000_000)          # 2 ms
    try:
        out = torch.full((3,), 7, dtype=torch.int64, device=DEV)
        csa.csa_check_wait_timeout(out)
        status = csa.csa_get_device_status()
    finally:
        csa.csa_set_wait_limit_ns(DEFAULT_WAIT_NS)
    claimed, waited_ns, other = out.cpu().tolist()
    assert status == 4, csa.status_string(status)   # CSA_ERR_DEVICE_TIMEOUT
    assert claimed == 0, "a wait on a barrier nothing arrives on claimed completion"
    assert other == 1, "a wait on a completed barrier did not return success"
    assert 2_000_000 <= waited_ns < 500_000_000, waited_ns
    # the context is still usable and the status word was cleared by the read
    dims = csa.Dims(d=64, c=512, m=4, cI=32, nhI=4, nh=64, dc=64, topk=40, dtype=csa.CSA_BF16)
    status, _ = _small_mqa(dims, [300])
    assert status == 0


def test_wait_limit_rejects_out_of_range_values():
    for bad in (0, 999, 60_000_000_001):
        with pytest.raises(csa.CsaError) as e:
            csa.csa_set_wait_limit_ns(bad)
        assert e.value.status == 1   # CSA_ERR_INVALID_ARG


@pytest.mark.parametrize("nh,c", [(64, 512), (2, 64)])
def test_inconsistent_cu_blocks_flagged_by_mqa(nh, c):
    """cu_blocks claiming fewer blocks than the first sequence has: its later
    rows are clamped to the blocks that exist and the condition is flagged
    (tensor-core kernel for c = 512, CUDA-core kernel otherwise)."""
    dims = csa.Dims(d=64, c=c, m=4, cI=32, nhI=4, nh=nh, dc=64, topk=40, dtype=csa.CSA_BF16)
    lens = [300, 200]
    status, O = _small_mqa(dims, lens, cu_blocks=[0, 20, 125])
    assert status == 6, csa.status_string(status)  # CSA_ERR_BAD_METADATA
    assert bool(torch.isfinite(O.float()).all())
    assert csa.csa_get_device_status() == 0        # cleared by the read


def test_inconsistent_cu_blocks_flagged_by_indexer():
    dims = csa.Dims(d=64, c=64, m=4, cI=128, nhI=64, nh=2, dc=64, topk=16, dtype=csa.CSA_BF16)
    lens = [600, 300]
    T = sum(lens)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    qI = synth.make_normal((T, dims.nhI * dims.cI), dims, 93).to(DEV)
    wI = synth.make_normal((T, dims.nhI), dims, 94).float().to(DEV)
    KI = synth.make_normal((NB, dims.cI), dims, 95, std=0.5).to(DEV)
    bad = torch.as_tensor([0, 100, NB], dtype=torch.int32, device=DEV)   # the first sequence has 150 blocks
    idx = torch.full((T, dims.topk), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.csa_indexer_workspace_bytes(dims, T, 2, max(lens)), dtype=torch.uint8, device=DEV)
    csa.csa_indexer_topk(dims, qI, dims.nhI * dims.cI, wI, dims.nhI, KI, cu.to(DEV), bad, 2, T, NB, max(lens),
                         idx, ws)
    assert csa.csa_get_device_status() == 6
    got = idx.cpu().numpy()
    assert np.all((got >= -7) & (got < NB))
