"""GPU parity of the projection stage (eqs. 1, 2, 5, 6, 7, 10): the tcgen05
GEMM (bf16) and the CUDA-core GEMM (fp32) through csa_project_hidden /
csa_project_query, against fp64 products of the same inputs.

A bf16 output must be the fp64 product rounded to bf16, up to one bf16 ulp
(the fp32 accumulation can move a value across a rounding boundary) plus a
small absolute term for values near 0; fp32 outputs within 1e-5 relative to
the row scale.  Each GEMM gets seeded inputs that both sides share (H for the
first, a seeded c^Q with a padded row stride for the second)."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth
from oracle import csa_oracle as orc
from parity import f64, gpu_pack

pytestmark = pytest.mark.gpu
DEV = "cuda"

H_SIDE = ("W_aKV", "W_bKV", "W_aZ", "W_bZ", "W_aKV_I", "W_bKV_I", "W_aZ_I", "W_bZ_I", "W_DQ")


def check(got, want, dtype, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    if dtype == csa.CSA_BF16:
        ulp = np.ldexp(1.0, np.frexp(np.abs(want))[1] - 8)     # bf16 ulp of each value
        bad = np.abs(got - want) > ulp + 1e-3
    else:
        scale = np.abs(want).max(axis=-1, keepdims=True) + 1e-30
        bad = np.abs(got - want) > 1e-5 * scale
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance, worst at {np.argwhere(bad)[0]}"


@pytest.mark.parametrize("dtype", [csa.CSA_BF16, csa.CSA_F32])
@pytest.mark.parametrize("T", [1, 37, 64, 129, 300])
def test_projections(dtype, T):
    dims = csa.Dims(d=200 if dtype == csa.CSA_BF16 else 196, c=64, m=4, cI=32, nhI=16, nh=4, dc=192, topk=8,
                    dtype=dtype)
    W = synth.make_weights(dims, 90 + T)
    H = synth.make_hidden(T, dims, 90 + T)
    packed = gpu_pack(dims, W)
    N1b, N2 = csa.csa_hidden_row_elems(dims), csa.csa_query_row_elems(dims)
    Y1 = torch.empty(T, N1b, dtype=H.dtype, device=DEV)
    wI = torch.empty(T, dims.nhI, dtype=torch.float32, device=DEV)
    Y2 = torch.empty(T, N2, dtype=H.dtype, device=DEV)
    csa.csa_project_hidden(dims, packed, H.to(DEV), T, Y1, wI)
    # the second GEMM gets a seeded c^Q (row stride ld_cq), identical on both sides
    ld_cq = dims.dc + 24
    cQ = synth.make_normal((T, ld_cq), dims, 190 + T)
    csa.csa_project_query(dims, packed, cQ.to(DEV), ld_cq, T, Y2)
    assert csa.csa_get_device_status() == 0
    W64 = {k: f64(v) for k, v in W.items()}
    H64 = f64(H)
    store = "bf16" if dtype == csa.CSA_BF16 else "exact"
    want1 = orc.storage_round(np.concatenate([orc.project(H64, W64[n]) for n in H_SIDE], axis=1), store)
    check(f64(Y1.cpu()), want1, dtype, "Y1")
    check(wI.cpu().double().numpy(), orc.project(H64, W64["W_w"]), csa.CSA_F32, "wI")   # fp32 output
    cQ64 = f64(cQ)[:, :dims.dc]
    want2 = orc.storage_round(np.concatenate([orc.project(cQ64, W64["W_IUQ"]), orc.project(cQ64, W64["W_UQ"])],
                                             axis=1), store)
    check(f64(Y2.cpu()), want2, dtype, "Y2")
