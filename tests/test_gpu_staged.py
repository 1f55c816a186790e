"""The staged entry points (csa_forward_staged, csa_decode_staged) launch the
same kernels as csa_forward / csa_decode and add only CUDA events between
the stages: their results must be bit-identical and the events ordered."""
import pytest
import torch

import compressed_sparse_attention_09_b200 as csa
from compressed_sparse_attention_09_b200 import synth
from parity import gpu_pack

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _events(n):
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in ev:          # create the handles
        e.record()
    return ev


def test_forward_staged_matches_forward():
    dims = csa.Dims(d=256, c=512, m=4, cI=128, nhI=64, nh=64, dc=128, topk=16, dtype=csa.CSA_BF16)
    lens = [300, 57]
    T = sum(lens)
    W = synth.make_weights(dims, 11)
    packed = gpu_pack(dims, W)
    H = synth.make_hidden(T, dims, 11).to(DEV)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    cu, cb = cu.to(DEV), cb.to(DEV)
    ws = torch.empty(csa.csa_forward_workspace_bytes(dims, T, 2), dtype=torch.uint8, device=DEV)
    outs = []
    for staged in (False, True):
        O = torch.empty(T, dims.nh * dims.c, dtype=torch.bfloat16, device=DEV)
        idx = torch.empty(T, dims.topk, dtype=torch.int32, device=DEV)
        if staged:
            ev = _events(6)
            csa.csa_forward_staged(dims, packed, H, cu, cb, 2, T, NB, max(lens), O, None, None, idx, ws, ev)
        else:
            csa.csa_forward(dims, packed, H, cu, cb, 2, T, NB, max(lens), O, None, None, idx, ws)
        assert csa.csa_get_device_status() == 0
        outs.append((O, idx))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(5)]
    assert all(x >= 0 for x in ms), ms
    with pytest.raises(csa.CsaError):
        csa.csa_forward_staged(dims, packed, H, cu, cb, 2, T, NB, max(lens), O, None, None, idx, ws, [0] * 6)


def test_decode_staged_matches_decode():
    dims = csa.Dims(d=256, c=512, m=4, cI=128, nhI=64, nh=128, dc=128, topk=64, dtype=csa.CSA_BF16)
    B, cap, pos0 = 4, 600, 2047
    W = synth.make_weights(dims, 12)
    packed = gpu_pack(dims, W)
    Cc0 = synth.make_normal((B, cap, dims.c), dims, 13).to(DEV)
    Kc0 = synth.make_normal((B, cap, dims.cI), dims, 14).to(DEV)
    ring0 = synth.make_normal((B, 2 * dims.m, csa.csa_ring_row_elems(dims)), dims, 15).to(DEV)
    h = synth.make_normal((B, dims.d), dims, 16).to(DEV)
    pos = torch.full((B,), pos0, dtype=torch.int32, device=DEV)
    ws = torch.empty(csa.csa_decode_workspace_bytes(dims, B, cap), dtype=torch.uint8, device=DEV)
    outs = []
    for staged in (False, True):
        Cc, Kc, ring = Cc0.clone(), Kc0.clone(), ring0.clone()
        clen = torch.full((B,), pos0 // dims.m, dtype=torch.int32, device=DEV)
        O = torch.empty(B, dims.nh * dims.c, dtype=torch.bfloat16, device=DEV)
        idx = torch.empty(B, dims.topk, dtype=torch.int32, device=DEV)
        if staged:
            ev = _events(7)
            csa.csa_decode_staged(dims, packed, h, pos, ring, Cc, Kc, clen, cap, B, O, idx, ws, ev)
        else:
            csa.csa_decode(dims, packed, h, pos, ring, Cc, Kc, clen, cap, B, O, idx, ws)
        assert csa.csa_get_device_status() == 0
        outs.append((O, idx, Cc, Kc, clen))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(6)]
    assert all(x >= 0 for x in ms), ms
