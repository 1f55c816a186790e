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
@pytest.mark.parametrize("T", [1, 37, 64, 65, 100, 127, 128, 129, 300])
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


@pytest.mark.parametrize("name", ["prefill", "long"])
def test_projections_full_size_sampled_rows(name):
    """Both projection GEMMs at the full sizes of the prefill (T = 8192) and
    long (T = 131072) workloads, in the launch configuration the forward
    uses: H (64 MB / 1 GB) and c^Q exceed the 32 MB bound above which tiles
    run in groups of row tiles, A1 (N = 4160) takes 192-column tiles, and
    every CTA runs many tiles.  64 sampled rows (first, last, seeded) of Y1,
    w^I and Y2 are compared with fp64 products of the same inputs."""
    w = synth.workloads()[name]
    dims = w.dims
    T = sum(w.seqlens)
    W = synth.make_weights(dims, w.seed)
    packed = gpu_pack(dims, W)
    H = synth.make_hidden(T, dims, w.seed)
    N1b, N2 = csa.csa_hidden_row_elems(dims), csa.csa_query_row_elems(dims)
    Y1 = torch.empty(T, N1b, dtype=H.dtype, device=DEV)
    wI = torch.empty(T, dims.nhI, dtype=torch.float32, device=DEV)
    csa.csa_project_hidden(dims, packed, H.to(DEV), T, Y1, wI)
    cQ = synth.make_normal((T, dims.dc), dims, w.seed + 77)
    Y2 = torch.empty(T, N2, dtype=H.dtype, device=DEV)
    csa.csa_project_query(dims, packed, cQ.to(DEV), dims.dc, T, Y2)
    assert csa.csa_get_device_status() == 0
    rng = np.random.default_rng(w.seed)
    rows = sorted({0, 1, 127, 128, T - 129, T - 1} | set(rng.integers(0, T, 58).tolist()))
    r = torch.as_tensor(rows, device=DEV)
    got1, gotw, got2 = f64(Y1[r].cpu()), wI[r].cpu().double().numpy(), f64(Y2[r].cpu())
    del Y1, Y2, wI
    torch.cuda.empty_cache()
    W64 = {k: f64(v) for k, v in W.items()}
    H64 = f64(H[rows])
    want1 = orc.storage_round(np.concatenate([orc.project(H64, W64[n]) for n in H_SIDE], axis=1), "bf16")
    check(got1, want1, dims.dtype, f"{name} Y1")
    # w^I is stored in fp32: within the worst-case error of a d-term fp32 sum
    # (gamma_d sum |h||W|, rounding unit 2^-23 to cover truncating adders)
    u = 2.0 ** -23
    bound = dims.d * u / (1 - dims.d * u) * (np.abs(H64) @ np.abs(W64["W_w"])) + 2 * u * np.abs(gotw)
    err = np.abs(gotw - orc.project(H64, W64["W_w"]))
    assert (err <= bound).all(), f"{name} wI: worst error {err.max():.3e} (bound {bound.min():.3e})"
    cQ64 = f64(cQ[rows])
    want2 = orc.storage_round(np.concatenate([orc.project(cQ64, W64["W_IUQ"]), orc.project(cQ64, W64["W_UQ"])],
                                             axis=1), "bf16")
    check(got2, want2, dims.dtype, f"{name} Y2")
