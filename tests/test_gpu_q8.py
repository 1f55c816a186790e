"""Decode over the quantised indexer-key cache (E4M3 codes + one fp32 scale
per entry; csa_quantize_keys_e4m3, csa_decode_q8): the quantiser bit for bit
against the oracle's quantize_e4m3_rows, and decode steps across cache
appends against the oracle's decode step in its e4m3 key-cache mode (the
protocol of parity.py: top-k rows, outputs on the GPU's own index set, the
caches after the appends)."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth
from oracle import csa_oracle as orc
from test_gpu_parity import decode_case, e4m3_codes_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_quantize_keys_match_the_oracle_bit_for_bit():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1000, 128)) * rng.uniform(1e-3, 300, (1000, 1))
    x[7] = 0.0
    x[8, 5] = 1e-30                                     # a row of one tiny value
    rows = torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)
    codes = torch.empty(1000, 128, dtype=torch.uint8, device=DEV)
    scale = torch.empty(1000, dtype=torch.float32, device=DEV)
    pad = torch.zeros(1000, 160, dtype=torch.bfloat16)  # row stride 160: a strided source
    pad[:, :128] = rows
    csa.csa_quantize_keys_e4m3(pad.to(DEV), 160, 1000, 128, codes, scale)
    torch.cuda.synchronize()
    oc, osc = orc.quantize_e4m3_rows(rows.double().numpy())
    assert np.array_equal(e4m3_codes_f64(codes), oc)
    assert np.array_equal(scale.cpu().double().numpy(), osc)


def test_decode_q8_small_across_appends():
    dims = csa.Dims(d=256, c=128, m=4, cI=128, nhI=64, nh=4, dc=128, topk=16, dtype=csa.CSA_BF16)
    c = decode_case(dims, B=5, pos0=301, cap=400, steps=6, seed=81, check=[0, 3, 4], q8=True)
    assert c["required"] >= 1, c


def test_decode_q8_nhI_32_from_the_start():
    dims = csa.Dims(d=256, c=128, m=4, cI=128, nhI=32, nh=4, dc=128, topk=8, dtype=csa.CSA_BF16)
    decode_case(dims, B=3, pos0=0, cap=64, steps=11, seed=82, check=[0, 1, 2], q8=True)


def test_decode_q8_full_size_sampled_sequences():
    """The decode workload (64 sequences, 16384 cached entries, n_h = 128,
    k = 2048) with the E4M3 key cache, four steps across an append."""
    w = synth.workloads()["decode"]
    decode_case(w.dims, B=w.decode_batch, pos0=w.decode_pos, cap=w.cache_cap, steps=4, seed=w.seed,
                check=[0, 21, 42, 63], q8=True)


def test_decode_q8_rejects_unsupported_dims():
    dims = csa.Dims(d=256, c=128, m=4, cI=64, nhI=64, nh=4, dc=128, topk=8, dtype=csa.CSA_BF16)
    B, cap = 2, 64
    z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device=DEV)  # noqa: E731
    ws = torch.empty(csa.csa_decode_workspace_bytes(dims, B, cap), dtype=torch.uint8, device=DEV)
    packed = torch.zeros(csa.csa_packed_weights_bytes(dims), dtype=torch.uint8, device=DEV)
    with pytest.raises(csa.CsaError) as e:
        csa.csa_decode_q8(dims, packed, z(B, dims.d), z(B, dt=torch.int32), z(B, 8, 768), z(B, cap, 128),
                          z(B, cap, 64, dt=torch.uint8), z(B, cap, dt=torch.float32), z(B, dt=torch.int32), cap, B,
                          z(B, 4 * 128), None, ws)
    assert e.value.status == 2   # CSA_ERR_UNSUPPORTED
