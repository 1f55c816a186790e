"""Host-side logic of the context-parallel prefill (cp.py), on CPU: the
zig-zag plan, and a two-rank gloo run of run_plan with the oracle as the
per-chunk computation.  Each rank compresses its chunks from the chunk
plus the m tokens before it, one all-gather exchanges the entries, and
each rank evaluates its chunks' queries over all entries.  Everything must
equal the oracle's single-process forward exactly (same fp64 arithmetic
per entry and per row)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, REPO)
from compressed_sparse_attention_09_b200 import cp, synth  # noqa: E402
from compressed_sparse_attention_09_b200.capi import CSA_F32, Dims  # noqa: E402
from oracle import csa_oracle as orc  # noqa: E402

DIMS = Dims(d=64, c=32, m=4, cI=16, nhI=4, nh=2, dc=32, topk=6, dtype=CSA_F32)
N = 203


def _od(d):
    return dict(m=d.m, topk=d.topk, nh=d.nh, nhI=d.nhI, c=d.c, cI=d.cI)


@pytest.mark.parametrize("n,world,m", [(203, 2, 4), (8192, 4, 4), (1000, 3, 8), (65, 2, 2)])
def test_zigzag_plan_covers_the_sequence(n, world, m):
    chunks, owner = cp.zigzag_plan(n, world, m)
    assert len(chunks) == 2 * world and chunks[0].start == 0
    assert sum(ch.length for ch in chunks) == n
    for a, b in zip(chunks, chunks[1:]):
        assert b.start == a.start + a.length and a.length % m == 0
    assert sorted(j for r in owner for j in r) == list(range(2 * world))
    assert all(len(set(o)) == 2 for o in owner)


def test_zigzag_plan_rejects_too_short_sequences():
    with pytest.raises(ValueError):
        cp.zigzag_plan(10, 4, 4)


def _oracle_fns(H, W, d):
    od = _od(d)

    def compress(ch):
        halo = d.m if ch.start > 0 else 0
        rows = H[ch.start - halo:ch.start + ch.length]
        C, KI, _, _ = orc.compressed_entries(rows, W, od, [rows.shape[0]], "exact")
        skip = halo // d.m
        return torch.as_tensor(C[skip:]), torch.as_tensor(KI[skip:])

    def queries(ch, C, KI):
        NB = C.shape[0]
        # the chunk's queries over the whole sequence's entries: rows of the
        # full sequence, evaluated by the oracle's per-query half
        rows = np.arange(ch.start, ch.start + ch.length)
        out = orc.query_rows(H, W, od, C.numpy(), KI.numpy(), np.array([0, H.shape[0]]), np.array([0, NB]), rows,
                             "exact")
        return torch.as_tensor(out["O"]), torch.as_tensor(out["idx"])

    return compress, queries


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = {k: v.double().numpy() for k, v in synth.make_weights(DIMS, 5).items()}
        H = synth.make_hidden(N, DIMS, 5).double().numpy()
        compress, queries = _oracle_fns(H, W, DIMS)

        def gather(send):
            out = [torch.empty_like(send) for _ in range(world)]
            dist.all_gather(out, send)
            return torch.stack(out)

        res = cp.run_plan(N, DIMS.m, DIMS.c, world, rank, compress, queries, gather)
        q.put((rank, {j: (o.numpy(), i.numpy()) for j, (o, i) in res.items()}))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_equal_the_single_process_oracle():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, res = q.get(timeout=300)
        got.update(res)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W = {k: v.double().numpy() for k, v in synth.make_weights(DIMS, 5).items()}
    H = synth.make_hidden(N, DIMS, 5).double().numpy()
    ref = orc.csa_forward(H, W, _od(DIMS), [N], store="exact")
    chunks, _ = cp.zigzag_plan(N, 2, DIMS.m)
    assert sorted(got) == list(range(4))
    for ch in chunks:
        O, idx = got[ch.index]
        sl = slice(ch.start, ch.start + ch.length)
        assert np.array_equal(idx, ref["idx"][sl])
        assert np.array_equal(O, ref["O"][sl])
