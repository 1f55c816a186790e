"""Context-parallel prefill of one sequence over the ranks of a process group.

The split follows the structure of the equations of "Compressed Sparse
Attention" (cnblogs): compressed entry i needs only tokens m(i-1) .. m(i+1)-1
(eqs. 3-4), and query t needs every entry s < floor(t/m) (the causal set of
eq. 8) but nothing else of the other tokens.  So:

1. the sequence is cut into 2 x world chunks on block boundaries; rank r
   owns chunks r and 2 world - 1 - r (zig-zag: early and late positions in
   each rank's share even out the causal work);
2. each rank compresses its chunks (csa_cp_compress: the H-side projection
   over the chunk plus the m tokens before it, compression of the chunk's
   blocks);
3. ONE all-gather exchanges every rank's C^Comp / K^IComp entries (the only
   data-path collective: NB x (c + c^I) bf16 values, 2.6 MB at n = 8192);
4. each rank runs A2, the indexer + top-k and the MQA for its chunks' queries
   over all entries (csa_cp_queries).

torch.distributed carries the all-gather (NCCL on GPUs); everything else is
calls of libcsa.  The plan, packing and assembly are plain functions so that
host-side tests can drive them with any per-chunk computation.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import capi
from .capi import Dims


@dataclass(frozen=True)
class Chunk:
    index: int      # position in the sequence order
    start: int      # first token
    length: int     # tokens

    def blocks(self, m):
        """(first block, number of complete blocks) of the chunk."""
        return self.start // m, self.length // m


def zigzag_plan(n: int, world: int, m: int):
    """2 x world chunks covering [0, n), each a multiple of m tokens except
    the last (which takes the remainder).  Returns (chunks, owner), where
    owner[r] lists the chunk indices of rank r: r and 2 world - 1 - r."""
    parts = 2 * world
    base = (n // parts) // m * m
    if base == 0:
        raise ValueError(f"sequence of {n} tokens is too short for {parts} chunks of whole blocks of {m}")
    sizes = [base] * parts
    sizes[-1] += n - base * parts
    chunks, start = [], 0
    for i, L in enumerate(sizes):
        chunks.append(Chunk(i, start, L))
        start += L
    owner = [[r, parts - 1 - r] for r in range(world)]
    return chunks, owner


def pack_entries(entries, max_blocks):
    """One rank's send buffer: its chunks' [C^Comp | K^IComp] rows, each
    chunk padded to max_blocks rows.  entries: list of (C [b, c], KI [b, cI])."""
    c, cI = entries[0][0].shape[1], entries[0][1].shape[1]
    buf = entries[0][0].new_zeros(len(entries) * max_blocks, c + cI)
    for k, (C, KI) in enumerate(entries):
        b = C.shape[0]
        buf[k * max_blocks:k * max_blocks + b, :c] = C
        buf[k * max_blocks:k * max_blocks + b, c:] = KI
    return buf


def assemble(gathered, chunks, owner, m, c, max_blocks):
    """Full C^Comp [NB, c] and K^IComp [NB, cI] from the gathered send
    buffers of every rank ([world, chunks per rank x max_blocks, c + cI])."""
    NB = sum(ch.length for ch in chunks) // m
    C = gathered.new_empty(NB, c)
    KI = gathered.new_empty(NB, gathered.shape[-1] - c)
    for r, mine in enumerate(owner):
        for k, j in enumerate(mine):
            b0, nb = chunks[j].blocks(m)
            rows = gathered[r, k * max_blocks:k * max_blocks + nb]
            C[b0:b0 + nb] = rows[:, :c]
            KI[b0:b0 + nb] = rows[:, c:]
    return C, KI


def all_gather_entries(send, world, group=None):
    """The one collective: every rank's send buffer to every rank."""
    import torch.distributed as dist
    out = send.new_empty(world, *send.shape)
    dist.all_gather_into_tensor(out, send.contiguous(), group=group)
    return out


def run_plan(n, m, c, world, rank, compress_fn, queries_fn, gather_fn):
    """Drives one context-parallel prefill: compress_fn(chunk) -> (C, KI) of
    its blocks; gather_fn(send) -> [world, ...] gathered buffers;
    queries_fn(chunk, C_full, KI_full) -> that chunk's outputs.  Returns
    {chunk index: output} for this rank's chunks."""
    chunks, owner = zigzag_plan(n, world, m)
    max_blocks = max(ch.length // m for ch in chunks)
    mine = owner[rank]
    entries = [compress_fn(chunks[j]) for j in mine]
    gathered = gather_fn(pack_entries(entries, max_blocks))
    C, KI = assemble(gathered, chunks, owner, m, c, max_blocks)
    return {j: queries_fn(chunks[j], C, KI) for j in mine}


class CpPrefill:
    """Context-parallel prefill on this rank's GPU through libcsa.

    H: the whole sequence's hidden states on this device, or any tensor whose
    rows [chunk.start - m, chunk.start + chunk.length) are valid for this
    rank's chunks (only those rows are read).  forward() returns
    {chunk index: O [length, nh*c]} for this rank's chunks and keeps the
    assembled C^Comp / K^IComp in .C / .KI."""

    def __init__(self, dims: Dims, packed, n: int, world: int, rank: int, device, group=None):
        self.dims, self.packed, self.n, self.world, self.rank = dims, packed, n, world, rank
        self.device, self.group = device, group
        self.chunks, self.owner = zigzag_plan(n, world, dims.m)
        d = dims
        dt = torch.bfloat16 if d.dtype == capi.CSA_BF16 else torch.float32
        self.N1b = capi.csa_hidden_row_elems(d)
        self.bufs = {}
        for j in self.owner[rank]:
            ch = self.chunks[j]
            Tp = ch.length + (d.m if ch.start > 0 else 0)
            nb = ch.length // d.m
            self.bufs[j] = {
                "Y1": torch.empty(Tp, self.N1b, dtype=dt, device=device),
                "wI": torch.empty(Tp, d.nhI, dtype=torch.float32, device=device),
                "C": torch.empty(max(nb, 1), d.c, dtype=dt, device=device),
                "KI": torch.empty(max(nb, 1), d.cI, dtype=dt, device=device),
                "O": torch.empty(ch.length, d.nh * d.c, dtype=dt, device=device),
                "idx": torch.empty(ch.length, d.topk, dtype=torch.int32, device=device),
                "ws": torch.empty(capi.csa_cp_workspace_bytes(d, ch.length, ch.start + ch.length),
                                  dtype=torch.uint8, device=device),
            }
        self.C = self.KI = None

    def compress(self, H, ch):
        d, b = self.dims, self.bufs[ch.index]
        halo = d.m if ch.start > 0 else 0
        capi.csa_cp_compress(d, self.packed, H[ch.start - halo:ch.start + ch.length], ch.length, ch.start,
                             b["Y1"], b["wI"], b["C"], b["KI"], b["ws"])
        nb = ch.length // d.m
        return b["C"][:nb], b["KI"][:nb]

    def queries(self, ch, C, KI):
        d, b = self.dims, self.bufs[ch.index]
        halo = d.m if ch.start > 0 else 0
        capi.csa_cp_queries(d, self.packed, b["Y1"][halo:], b["wI"][halo:], ch.length, ch.start, C, KI, C.shape[0],
                            b["O"], b["idx"], b["ws"])
        return b["O"]

    def forward(self, H, gather_fn=None):
        if gather_fn is None:
            gather_fn = lambda send: all_gather_entries(send, self.world, self.group)  # noqa: E731
        keep = {}

        def q(ch, C, KI):
            keep["C"], keep["KI"] = C, KI
            return self.queries(ch, C, KI)

        out = run_plan(self.n, self.dims.m, self.dims.c, self.world, self.rank, lambda ch: self.compress(H, ch), q,
                       gather_fn)
        self.C, self.KI = keep.get("C"), keep.get("KI")
        return out
