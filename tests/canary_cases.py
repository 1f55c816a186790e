"""Canary-padded runs of the library's entry points on small seeded inputs.

Every buffer a call writes (outputs, caches, ring, workspace) sits inside a
larger allocation whose PAD bytes on each side hold the byte CANARY; after the
call the pads must be intact, so a write outside any buffer shows up as a
changed pad.  The cases take the tensor-core kernels (c = 512, n_h = 64,
n_h^I = 64, c^I = 128) and the fp32 SIMT kernels, prefill and decode (bf16 and
E4M3 key caches), and the fused projection + compression.

run_all() returns {name: numpy array} of every written buffer plus the
device status after each case.  tests/test_gpu_canary.py runs it with the
release library; the same function runs in a child process with
CSA_DEBUG=1 (the debug build, whose kernels check the indices they compute)
and the two results must be bit-identical.
"""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:   # run as a script (the debug-build child process)
    sys.path.insert(0, ROOT)

import compressed_sparse_attention_09_b200 as csa  # noqa: E402
from compressed_sparse_attention_09_b200 import synth  # noqa: E402

DEV = "cuda"
PAD = 4096          # canary bytes on each side of a buffer (a multiple of 256: alignment kept)
CANARY = 0xA5

TC = csa.Dims(d=256, c=512, m=4, cI=128, nhI=64, nh=64, dc=128, topk=16, dtype=csa.CSA_BF16)
SIMT = csa.Dims(d=128, c=64, m=2, cI=32, nhI=4, nh=4, dc=64, topk=8, dtype=csa.CSA_F32)


class Padded:
    """A tensor of `shape`/`dtype` in the middle of a canary-filled byte buffer."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((PAD + n + PAD,), CANARY, dtype=torch.uint8, device=DEV)
        self.t = self.buf[PAD:PAD + n].view(dtype).view(*shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        return bool((self.buf[:PAD] == CANARY).all()) and bool((self.buf[PAD + self.n:] == CANARY).all())


def _pack(dims, W):
    packed = Padded((csa.csa_packed_weights_bytes(dims),), torch.uint8)
    csa.csa_pack_weights(dims, {k: v.to(DEV) for k, v in W.items()}, packed.t)
    return packed


def _finish(name, bufs, out):
    status = csa.csa_get_device_status()
    out[f"{name}/status"] = np.array([status])
    for k, b in bufs.items():
        out[f"{name}/{k}/pads_intact"] = np.array([b.intact()])
        if k != "ws":   # the workspace holds scratch whose unused bytes are unspecified
            out[f"{name}/{k}"] = b.t.cpu().view(torch.uint8).numpy().copy()


def forward_case(dims, lens, seed, name, out):
    W = synth.make_weights(dims, seed)
    T = sum(lens)
    H = synth.make_hidden(T, dims, seed)
    packed = _pack(dims, W)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    dt = H.dtype
    b = {"O": Padded((T, dims.nh * dims.c), dt), "C": Padded((NB, dims.c), dt), "KI": Padded((NB, dims.cI), dt),
         "idx": Padded((T, dims.topk), torch.int32),
         "ws": Padded((csa.csa_forward_workspace_bytes(dims, T, len(lens)),), torch.uint8)}
    csa.csa_forward(dims, packed.t, H.to(DEV), cu.to(DEV), cb.to(DEV), len(lens), T, NB, max(lens), b["O"].t,
                    b["C"].t, b["KI"].t, b["idx"].t, b["ws"].t)
    b["packed"] = packed
    _finish(name, b, out)


def fused_projection_case(dims, lens, seed, name, out):
    W = synth.make_weights(dims, seed)
    T = sum(lens)
    H = synth.make_hidden(T, dims, seed)
    packed = _pack(dims, W)
    cu, cb = csa.cu_from_lengths(lens, dims.m)
    NB = int(cb[-1])
    b = {"Y1": Padded((T, csa.csa_hidden_row_elems(dims)), H.dtype), "wI": Padded((T, dims.nhI), torch.float32),
         "C": Padded((NB, dims.c), H.dtype), "KI": Padded((NB, dims.cI), H.dtype),
         "ws": Padded((csa.csa_project_compress_workspace_bytes(dims, T),), torch.uint8)}
    csa.csa_project_hidden_compress(dims, packed.t, H.to(DEV), T, cu.to(DEV), cb.to(DEV), len(lens), NB, b["Y1"].t,
                                    b["wI"].t, b["C"].t, b["KI"].t, b["ws"].t)
    # the fused call writes the c^Q columns of Y1 (after the 4c + 4cI C/Z columns), not the C/Z
    # columns themselves: compare only what it defines
    _finish(name, {k: v for k, v in b.items() if k != "Y1"}, out)
    q0 = 4 * dims.c + 4 * dims.cI
    out[f"{name}/Y1/pads_intact"] = np.array([b["Y1"].intact()])
    out[f"{name}/cQ"] = b["Y1"].t[:, q0:q0 + dims.dc].cpu().view(torch.uint8).numpy().copy()


def decode_case(dims, B, pos0, cap, steps, seed, name, out, q8=False):
    m = dims.m
    W = synth.make_weights(dims, seed)
    packed = _pack(dims, W)
    RW = csa.csa_ring_row_elems(dims)
    dt = torch.bfloat16 if dims.dtype == csa.CSA_BF16 else torch.float32
    b = {"Cc": Padded((B, cap, dims.c), dt, synth.make_normal((B, cap, dims.c), dims, seed + 1)),
         "ring": Padded((B, 2 * m, RW), dt, synth.make_normal((B, 2 * m, RW), dims, seed + 3)),
         "clen": Padded((B,), torch.int32, torch.full((B,), pos0 // m, dtype=torch.int32)),
         "ws": Padded((csa.csa_decode_workspace_bytes(dims, B, cap),), torch.uint8)}
    Kc = synth.make_normal((B, cap, dims.cI), dims, seed + 2)
    if q8:
        b["codes"] = Padded((B, cap, dims.cI), torch.uint8)
        b["scale"] = Padded((B, cap), torch.float32)
        Kd = Kc.to(DEV)
        csa.csa_quantize_keys_e4m3(Kd, dims.cI, B * cap, dims.cI, b["codes"].t, b["scale"].t)
    else:
        b["Kc"] = Padded((B, cap, dims.cI), dt, Kc)
    pos = torch.full((B,), pos0, dtype=torch.int32)
    for step in range(steps):
        h = synth.make_normal((B, dims.d), dims, seed + 100 + step).to(DEV)
        b[f"O{step}"] = Padded((B, dims.nh * dims.c), dt)
        b[f"idx{step}"] = Padded((B, dims.topk), torch.int32)
        if q8:
            csa.csa_decode_q8(dims, packed.t, h, pos.to(DEV), b["ring"].t, b["Cc"].t, b["codes"].t, b["scale"].t,
                              b["clen"].t, cap, B, b[f"O{step}"].t, b[f"idx{step}"].t, b["ws"].t)
        else:
            csa.csa_decode(dims, packed.t, h, pos.to(DEV), b["ring"].t, b["Cc"].t, b["Kc"].t, b["clen"].t, cap, B,
                           b[f"O{step}"].t, b[f"idx{step}"].t, b["ws"].t)
        pos += 1
    _finish(name, b, out)


def run_all():
    out = {}
    forward_case(TC, [300, 57, 130], 11, "forward_tc", out)
    forward_case(SIMT, [70, 33], 12, "forward_simt", out)
    fused_projection_case(TC, [300, 57, 130], 13, "fused_projection", out)
    decode_case(TC, B=5, pos0=2045, cap=640, steps=5, seed=14, name="decode_tc", out=out)
    decode_case(TC, B=5, pos0=2045, cap=640, steps=5, seed=15, name="decode_q8", out=out, q8=True)
    decode_case(SIMT, B=3, pos0=37, cap=40, steps=4, seed=16, name="decode_simt", out=out)
    return out


if __name__ == "__main__":
    np.savez(sys.argv[1], **run_all())
