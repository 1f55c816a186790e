"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test names the passage of "Compressed Sparse Attention (压缩稀疏注意力)"
(cnblogs) it follows.  The pins are closed forms worked by hand, invariants the
equations fix, special cases that reduce to a library routine (torch's
scaled-dot-product attention, torch's bf16 conversion) and brute force on tiny
inputs.  They are chosen so that a dropped term, a wrong sign, a shifted block
index or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import csa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- rounding

def test_round_bf16_matches_torch_conversion():
    """Storage rounding equals torch's fp32->bf16 conversion (RNE) on fp32 inputs."""
    r = rng(0)
    x = np.concatenate([r.standard_normal(100000) * 10.0 ** r.integers(-6, 6, 100000),
                        # exact ties between two bf16 neighbours: both directions of even
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)]),
                        np.array([0.0, -0.0, 1.0, -3.5])])
    x32 = x.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = orc.round_bf16(x32.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_f32_is_fp32_cast():
    x = rng(1).standard_normal(1000)
    assert np.array_equal(orc.round_f32(x), x.astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------- eqs. (3)-(4)

def _random_block_inputs(L, w, m, seed):
    r = rng(seed)
    return [r.standard_normal((L, w)) for _ in range(4)] + [r.standard_normal((m, w)) * 0.3 for _ in range(2)]


def test_compress_weights_sum_to_one():
    """Eq. (3): the 2m softmax weights of each channel sum to 1 (and the m
    weights at i=0), so constant C rows compress to that constant."""
    L, w, m = 37, 5, 4
    Ca, Cb, Za, Zb, Ba, Bb = _random_block_inputs(L, w, m, 2)
    ones = np.full((L, w), 3.25)
    out = orc.compress(ones, ones, Za, Zb, Ba, Bb, m)
    assert out.shape == (L // m, w)
    np.testing.assert_allclose(out, 3.25, rtol=0, atol=1e-13)


def test_compress_constant_logits_give_block_means():
    """B = 0 and a constant Z make every weight equal: entry i >= 1 is the mean
    of the 2m rows C^a[mi..mi+m-1], C^b[m(i-1)..mi-1]; entry 0 is the mean of
    the m rows C^a[0..m-1] (i = 0 padding)."""
    L, w, m = 24, 6, 3
    Ca, Cb, _, _, _, _ = _random_block_inputs(L, w, m, 3)
    Z = np.full((L, w), -0.7)
    B0 = np.zeros((m, w))
    out = orc.compress(Ca, Cb, Z, Z, B0, B0, m)
    np.testing.assert_allclose(out[0], Ca[0:m].mean(axis=0), atol=1e-14)
    for i in range(1, L // m):
        want = np.concatenate([Ca[m * i:m * (i + 1)], Cb[m * (i - 1):m * i]]).mean(axis=0)
        np.testing.assert_allclose(out[i], want, atol=1e-14)


def test_compress_worked_example():
    """Hand-worked case of eqs. (3)-(4) with m = 4, one channel.

    Z = 0 everywhere, B^a rows = ln 1, ln 2, ln 3, ln 4 and B^b rows =
    ln 5, ln 6, ln 7, ln 8, so the softmax weights of entry i >= 1 are
    (1, 2, 3, 4)/36 on the block's own C^a rows and (5, 6, 7, 8)/36 on the
    previous block's C^b rows; entry 0 has weights (1, 2, 3, 4)/10 on C^a.
    With C^a[t] = t and C^b[t] = 1000 + t:
      entry 0 = (0*1 + 1*2 + 2*3 + 3*4)/10 = 2
      entry 1 = (4*1 + 5*2 + 6*3 + 7*4)/36 + (1000*26 + 0*5 + 1*6 + 2*7 + 3*8)/36
              = 60/36 + 26044/36 = 26104/36
      entry 2 = (8*1 + 9*2 + 10*3 + 11*4)/36 + (1004*5 + 1005*6 + 1006*7 + 1007*8)/36
              = 100/36 + 26148/36 = 26248/36
    """
    m, L = 4, 12
    Ca = np.arange(L, dtype=np.float64)[:, None]
    Cb = 1000.0 + np.arange(L, dtype=np.float64)[:, None]
    Z = np.zeros((L, 1))
    Ba = np.log(np.array([1.0, 2, 3, 4]))[:, None]
    Bb = np.log(np.array([5.0, 6, 7, 8]))[:, None]
    out = orc.compress(Ca, Cb, Z, Z, Ba, Bb, m)[:, 0]
    want = [2.0, float(Fraction(26104, 36)), float(Fraction(26248, 36))]
    np.testing.assert_allclose(out, want, rtol=1e-14)


def test_compress_golden_fixture():
    """Fixture tests/golden/compress_m2.json: a second hand-worked case (m = 2,
    two channels, nonzero Z) whose expected values were derived by hand in the
    fixture's own notes."""
    with open(os.path.join(GOLDEN, "compress_m2.json")) as f:
        g = json.load(f)
    out = orc.compress(*(np.array(g[k], dtype=np.float64) for k in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")),
                       g["m"])
    np.testing.assert_allclose(out, np.array(g["expected"]), rtol=1e-13)


def test_compress_overlap_and_i0_padding():
    """The C^b/Z^b rows of block i feed entry i+1 only and the C^a/Z^a rows of
    block i feed entry i only (the overlap statement after eq. (4)); the Z^b,
    C^b rows of the last block and the ragged tail feed nothing."""
    L, w, m = 22, 3, 4            # 5 full blocks, tail of 2 tokens
    base = _random_block_inputs(L, w, m, 4)
    ref = orc.compress(*base, m)
    assert ref.shape[0] == 5
    for arr_id, tok in itertools.product(range(4), range(L)):
        pert = [a.copy() for a in base]
        pert[arr_id][tok] += 1.0
        out = orc.compress(*pert, m)
        changed = set(np.nonzero(np.any(out != ref, axis=1))[0].tolist())
        blk = tok // m
        if blk >= 5:
            expect = set()                                    # dropped tail
        elif arr_id in (0, 2):                               # C^a, Z^a
            expect = {blk}
        else:                                                 # C^b, Z^b
            expect = {blk + 1} if blk + 1 < 5 else set()
        assert changed == expect, (arr_id, tok, changed, expect)


def test_compress_bias_rows_follow_token_position():
    """Row r of B^a / B^b is added to the r-th token of its block (eq. 3):
    raising B^a[r] by ln 2 doubles the weight of token mi+r in every entry."""
    L, w, m = 16, 2, 4
    Ca, Cb, Za, Zb, Ba, Bb = _random_block_inputs(L, w, m, 5)
    r0 = 2
    Ba2 = Ba.copy()
    Ba2[r0] += math.log(2.0)
    out = orc.compress(Ca, Cb, Za, Zb, Ba2, Bb, m)
    # Same result from doubling the weight directly: Z^a[m i + r0] += ln 2.
    Za2 = Za.copy()
    Za2[r0::m] += math.log(2.0)
    np.testing.assert_allclose(out, orc.compress(Ca, Cb, Za2, Zb, Ba, Bb, m), atol=1e-13)


# ---------------------------------------------------------------- eq. (8)

def test_indexer_scores_one_hot_heads():
    """Eq. (8) with one-hot queries: head 0 reads channel 0 and head 1 reads
    channel 1 of each K^IComp_s, so I_s = w_0 ReLU(K_s[0]) + w_1 ReLU(K_s[1])."""
    cI = 4
    q = np.zeros((2, cI))
    q[0, 0] = 1.0
    q[1, 1] = 1.0
    w = np.array([2.0, -3.0])
    K = np.array([[1.0, 1.0, 9.0, 9.0],
                  [-1.0, 2.0, 9.0, 9.0],
                  [0.5, -4.0, 9.0, 9.0]])
    got = orc.indexer_scores(q, w, K)
    np.testing.assert_allclose(got, [2.0 - 3.0, -6.0, 1.0], atol=0)


def test_indexer_scores_no_visible_block():
    assert orc.indexer_scores(np.ones((3, 2)), np.ones(3), np.zeros((0, 2))).shape == (0,)


# ---------------------------------------------------------------- eq. (9)

def test_topk_brute_force():
    """For distinct scores the top-k set is the unique k-subset with the
    largest score sum: enumerate every subset of tiny candidate sets."""
    r = rng(6)
    for avail in range(0, 8):
        for k in range(1, 7):
            s = r.standard_normal(avail)
            got = orc.topk_select(s, k)
            keff = min(k, avail)
            assert np.all(got[keff:] == -1) and got.shape == (k,)
            if keff == 0:
                continue
            best = max(itertools.combinations(range(avail), keff), key=lambda c: sum(s[list(c)]))
            assert sorted(got[:keff].tolist()) == list(best)


def test_topk_ties_prefer_lower_block():
    """Equal scores: the lower block index wins (W^w = 0 makes every score 0)."""
    assert orc.topk_select(np.zeros(10), 4).tolist() == [0, 1, 2, 3]
    assert orc.topk_select(np.array([1.0, 2, 2, 2, 0]), 2).tolist() == [1, 2]
    assert orc.topk_select(np.array([5.0, 2, 2, 2, 0]), 3).tolist() == [0, 1, 2]


def test_topk_clamps_to_available():
    assert orc.topk_select(np.array([0.3, -1.0]), 5).tolist() == [0, 1, -1, -1, -1]


# ---------------------------------------------------------------- eq. (11)

def test_core_attn_single_entry_is_identity():
    """One selected entry: the softmax over one element is 1, o = C^Comp_0."""
    r = rng(7)
    C = r.standard_normal((1, 16))
    q = r.standard_normal((5, 16)) * 10
    np.testing.assert_allclose(orc.core_attn(q, C), np.repeat(C, 5, axis=0), atol=1e-15)


def test_core_attn_two_orthogonal_entries():
    """Two entries C_0 = a e_0, C_1 = b e_1 and q = (x, y, 0, ...): the weights
    are the logistic of (x a - y b)/sqrt(c), worked by hand."""
    c = 9
    a, b, x, y = 2.0, -1.5, 0.7, 1.3
    C = np.zeros((2, c))
    C[0, 0], C[1, 1] = a, b
    q = np.zeros((1, c))
    q[0, 0], q[0, 1] = x, y
    p0 = 1.0 / (1.0 + math.exp(-(x * a - y * b) / 3.0))
    want = np.zeros(c)
    want[0], want[1] = p0 * a, (1.0 - p0) * b
    np.testing.assert_allclose(orc.core_attn(q, C)[0], want, atol=1e-15)


def test_core_attn_matches_torch_sdpa():
    """CoreAttn = softmax(q K^T / sqrt(c)) V with K = V: torch's library SDPA."""
    r = rng(8)
    q = r.standard_normal((6, 32))
    C = r.standard_normal((11, 32))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(C)[None], torch.from_numpy(C)[None])[0].numpy()
    np.testing.assert_allclose(orc.core_attn(q, C), want, atol=1e-13)


def test_core_attn_empty_is_zero():
    assert np.all(orc.core_attn(np.ones((3, 4)), np.zeros((0, 4))) == 0)


# ---------------------------------------------------------------- whole path

def small_problem(seed, seqlens, d=24, c=16, cI=8, m=4, nhI=3, nh=2, dc=12, topk=3):
    r = rng(seed)
    dims = dict(d=d, c=c, cI=cI, m=m, nhI=nhI, nh=nh, dc=dc, topk=topk)
    W = {}
    for n in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"):
        W[n] = r.standard_normal((d, c)) / math.sqrt(d)
    for n in ("W_aKV_I", "W_bKV_I", "W_aZ_I", "W_bZ_I"):
        W[n] = r.standard_normal((d, cI)) / math.sqrt(d)
    W["B_a"], W["B_b"] = (r.standard_normal((m, c)) * 0.3 for _ in range(2))
    W["B_a_I"], W["B_b_I"] = (r.standard_normal((m, cI)) * 0.3 for _ in range(2))
    W["W_DQ"] = r.standard_normal((d, dc)) / math.sqrt(d)
    W["W_IUQ"] = r.standard_normal((dc, nhI * cI)) / math.sqrt(dc)
    W["W_UQ"] = r.standard_normal((dc, nh * c)) / math.sqrt(dc)
    W["W_w"] = r.standard_normal((d, nhI)) / math.sqrt(d)
    H = r.standard_normal((sum(seqlens), d))
    return H, W, dims


def test_forward_dense_equivalence_when_k_covers_all_blocks():
    """k >= floor(t/m) selects every visible block, so eq. (11) becomes dense
    causal attention over C^Comp_0..C^Comp_{floor(t/m)-1}: checked against
    torch's SDPA with a block-causal mask.  Rows with no visible block are 0."""
    H, W, dims = small_problem(9, [41], topk=64)
    out = orc.csa_forward(H, W, dims, [41])
    Cc = torch.from_numpy(out["C_comp"])
    q = torch.from_numpy(out["q"])                       # [T, nh, c]
    T, nh, c = q.shape
    t = torch.arange(T)[:, None]
    s = torch.arange(Cc.shape[0])[None, :]
    mask = s < (t // dims["m"])                          # [T, NB]
    want = torch.zeros(T, nh, c, dtype=torch.float64)
    has = mask.any(dim=1)
    dense = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1)[:, has], Cc[None].expand(nh, -1, -1), Cc[None].expand(nh, -1, -1),
        attn_mask=mask[has][None])
    want[has] = dense.transpose(0, 1)
    np.testing.assert_allclose(out["O"], want.numpy(), atol=1e-12)
    assert np.all(out["O"][: dims["m"]] == 0)


def test_forward_single_block_rows_equal_entry0():
    """Tokens t in [m, 2m) see exactly one block: o_{t,h} = C^Comp_0 for all h."""
    H, W, dims = small_problem(10, [20])
    out = orc.csa_forward(H, W, dims, [20])
    m = dims["m"]
    for t in range(m, 2 * m):
        for h in range(dims["nh"]):
            np.testing.assert_allclose(out["O"][t, h], out["C_comp"][0], atol=1e-14)


def test_forward_brute_force_scores():
    """Brute force over the full score matrix: for every query, the chosen
    blocks are the k-subset of visible blocks with the largest score sum
    (scores of a random case are distinct)."""
    H, W, dims = small_problem(11, [30], topk=3)
    out = orc.csa_forward(H, W, dims, [30], keep_scores=True)
    for t in range(30):
        I = out["scores"][t]
        keff = min(3, len(I))
        got = sorted(out["idx"][t][:keff].tolist())
        if keff:
            best = max(itertools.combinations(range(len(I)), keff), key=lambda c: sum(I[list(c)]))
            assert got == list(best)


def test_forward_head_layout_with_one_hot_up_projection():
    """Eqs. (6) and (10) concatenate heads in order: with W^UQ = [1*I | 2*I]
    (d_c = c) head h of q_t is (h+1) c^Q_t; likewise for the indexer."""
    H, W, dims = small_problem(12, [12], dc=16, c=16, cI=8, nh=2, nhI=2)
    W["W_UQ"] = np.concatenate([np.eye(16), 2 * np.eye(16)], axis=1)
    W["W_IUQ"] = np.concatenate([np.eye(16)[:, :8], 3 * np.eye(16)[:, 8:]], axis=1)
    out = orc.csa_forward(H, W, dims, [12])
    np.testing.assert_allclose(out["q"][:, 0], out["cQ"], atol=1e-14)
    np.testing.assert_allclose(out["q"][:, 1], 2 * out["cQ"], atol=1e-14)
    np.testing.assert_allclose(out["qI"][:, 0], out["cQ"][:, :8], atol=1e-14)
    np.testing.assert_allclose(out["qI"][:, 1], 3 * out["cQ"][:, 8:], atol=1e-14)


def test_forward_zero_head_weights_pick_lowest_blocks():
    """W^w = 0 makes every index score 0, so each query keeps blocks 0..k_eff-1."""
    H, W, dims = small_problem(13, [33], topk=3)
    W["W_w"] = np.zeros_like(W["W_w"])
    out = orc.csa_forward(H, W, dims, [33])
    for t in range(33):
        keff = min(3, t // 4)
        assert out["idx"][t].tolist() == list(range(keff)) + [-1] * (3 - keff)


def test_forward_is_causal():
    """Perturbing H at tokens > t leaves idx_t, o_t and every entry s with
    m(s+1) <= t+1 unchanged (the causal condition s < floor(t/m))."""
    H, W, dims = small_problem(14, [29])
    ref = orc.csa_forward(H, W, dims, [29])
    for t0 in (5, 12, 20):
        H2 = H.copy()
        H2[t0 + 1:] += rng(t0).standard_normal(H2[t0 + 1:].shape)
        out = orc.csa_forward(H2, W, dims, [29])
        np.testing.assert_array_equal(out["idx"][: t0 + 1], ref["idx"][: t0 + 1])
        np.testing.assert_allclose(out["O"][: t0 + 1], ref["O"][: t0 + 1], atol=0)
        full = (t0 + 1) // dims["m"]
        np.testing.assert_allclose(out["C_comp"][:full], ref["C_comp"][:full], atol=0)


def test_forward_packed_equals_separate():
    """Packed ragged sequences give the same result as each sequence alone;
    compression blocks never cross a sequence boundary."""
    lens = [13, 4, 22, 3, 9]
    H, W, dims = small_problem(15, lens)
    packed = orc.csa_forward(H, W, dims, lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    for b, L in enumerate(lens):
        alone = orc.csa_forward(H[cu[b]:cu[b + 1]], W, dims, [L])
        np.testing.assert_allclose(packed["O"][cu[b]:cu[b + 1]], alone["O"], atol=1e-13)
        np.testing.assert_array_equal(packed["idx"][cu[b]:cu[b + 1]], alone["idx"])
        blk = slice(packed["cu_blocks"][b], packed["cu_blocks"][b + 1])
        np.testing.assert_allclose(packed["C_comp"][blk], alone["C_comp"], atol=1e-13)


def test_forward_rows_subset_matches_full():
    H, W, dims = small_problem(16, [10, 27])
    full = orc.csa_forward(H, W, dims, [10, 27])
    rows = [0, 9, 10, 25, 36]
    part = orc.csa_forward(H, W, dims, [10, 27], rows=rows)
    np.testing.assert_allclose(part["O"], full["O"][rows], atol=1e-14)
    np.testing.assert_array_equal(part["idx"], full["idx"][rows])


def test_forward_bf16_storage_close_to_exact():
    """Storage rounding only perturbs: bf16-stored compressed entries stay
    within bf16 precision of the exact ones (a check on the rounding hooks)."""
    H, W, dims = small_problem(17, [32])
    ex = orc.csa_forward(H, W, dims, [32], store="exact")
    bf = orc.csa_forward(H, W, dims, [32], store="bf16")
    np.testing.assert_allclose(bf["C_comp"], ex["C_comp"], atol=2e-2)
    assert np.array_equal(bf["C_comp"], orc.round_bf16(bf["C_comp"]))


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("t0", [8, 13])
def test_decode_steps_reproduce_prefill_rows(t0):
    """m + 1 decode steps starting at token t0, over a cache and ring built
    from the first t0 tokens, reproduce the prefill rows t0..t0+m and append
    exactly the entries that prefill computes."""
    L = t0 + 5
    H, W, dims = small_problem(18, [L], topk=2)
    m, c, cI = dims["m"], dims["c"], dims["cI"]
    full = orc.csa_forward(H, W, dims, [L])
    cap = L // m + 1
    C_cache = np.zeros((1, cap, c))
    K_cache = np.zeros((1, cap, cI))
    nb0 = t0 // m
    C_cache[0, :nb0] = full["C_comp"][:nb0]
    K_cache[0, :nb0] = full["K_icomp"][:nb0]
    cache_len = np.array([nb0])
    ring = np.zeros((1, 2 * m, 4 * c + 4 * cI))
    for tok in range(max(0, t0 - 2 * m), t0):
        ring[0, tok % (2 * m)] = np.concatenate(
            [orc.project(H[tok:tok + 1], W[n])[0] for n in orc._HSIDE])
    for t in range(t0, t0 + m + 1):
        O, idx = orc.csa_decode_step(H[t:t + 1], [t], C_cache, K_cache, cache_len, ring, W, dims)
        np.testing.assert_allclose(O[0], full["O"][t], atol=1e-13)
        np.testing.assert_array_equal(idx[0], full["idx"][t])
    nb1 = (t0 + m + 1) // m
    assert cache_len[0] == nb1
    np.testing.assert_allclose(C_cache[0, :nb1], full["C_comp"][:nb1], atol=1e-13)
    np.testing.assert_allclose(K_cache[0, :nb1], full["K_icomp"][:nb1], atol=1e-13)


def test_decode_first_block_uses_i0_padding():
    """Decoding from t = 0 builds entry 0 with the i = 0 padding."""
    H, W, dims = small_problem(19, [9], topk=2)
    m, c, cI = dims["m"], dims["c"], dims["cI"]
    full = orc.csa_forward(H, W, dims, [9])
    C_cache, K_cache = np.zeros((1, 3, c)), np.zeros((1, 3, cI))
    cache_len = np.array([0])
    ring = np.zeros((1, 2 * m, 4 * c + 4 * cI))
    for t in range(9):
        O, idx = orc.csa_decode_step(H[t:t + 1], [t], C_cache, K_cache, cache_len, ring, W, dims)
        np.testing.assert_allclose(O[0], full["O"][t], atol=1e-13)
    np.testing.assert_allclose(C_cache[0, :2], full["C_comp"], atol=1e-13)


@pytest.mark.parametrize("store", ["exact", "bf16"])
def test_forward_sampled_equals_forward(store):
    """The chunked, memory-light form gives the same rows as csa_forward."""
    lens = [37, 5, 60]
    H, W, dims = small_problem(20, lens, topk=4)
    rows = [0, 4, 36, 40, 41, 70, 101]
    full = orc.csa_forward(H, W, dims, lens, store=store, rows=rows, keep_scores=True)
    samp = orc.csa_forward_sampled(H, W, dims, lens, rows, store=store, chunk=16)
    np.testing.assert_allclose(samp["C_comp"], full["C_comp"], atol=1e-12)
    np.testing.assert_allclose(samp["K_icomp"], full["K_icomp"], atol=1e-12)
    np.testing.assert_array_equal(samp["idx"], full["idx"])
    np.testing.assert_allclose(samp["O"], full["O"], atol=1e-12)
    for a, b in zip(samp["scores"], full["scores"]):
        np.testing.assert_allclose(a, b, atol=1e-12)


# ---------------------------------------------------------------- FP8 E4M3 (quantised key cache)

def test_round_e4m3_matches_torch_float8_below_saturation():
    """round_e4m3 against torch's own float -> float8_e4m3fn conversion
    (round to nearest even) over magnitudes from subnormal to 448."""
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(4000) * s for s in (1e-3, 0.02, 1.0, 30.0, 200.0)])
    x = x[np.abs(x) <= 448]
    want = torch.as_tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(orc.round_e4m3(x.astype(np.float32).astype(np.float64)), want)


def test_round_e4m3_hand_values():
    # ties to even: 1.0625 lies halfway between 1.0 and 1.125, 1.1875 between 1.125 and 1.25
    assert orc.round_e4m3(1.0625) == 1.0 and orc.round_e4m3(1.1875) == 1.25
    # smallest normal 2^-6 and smallest subnormal 2^-9 are exact; half of 2^-9 rounds to 0 (even)
    assert orc.round_e4m3(2.0 ** -6) == 2.0 ** -6 and orc.round_e4m3(2.0 ** -9) == 2.0 ** -9
    assert orc.round_e4m3(2.0 ** -10) == 0.0 and orc.round_e4m3(3 * 2.0 ** -10) == 2.0 ** -8
    # saturation: 464 would round to 480, beyond the largest finite 448
    assert orc.round_e4m3(464.0) == 448.0 and orc.round_e4m3(-1000.0) == -448.0
    assert orc.round_e4m3(-3.4) == -3.5 and orc.round_e4m3(0.0) == 0.0


def test_quantize_e4m3_rows_scale_and_error():
    rng = np.random.default_rng(8)
    V = orc.round_bf16(rng.standard_normal((50, 128)) * rng.uniform(0.01, 10, (50, 1)))
    V[3] = 0.0
    codes, scale = orc.quantize_e4m3_rows(V)
    # each row's largest magnitude maps to the largest code
    rows = [r for r in range(50) if r != 3]
    assert np.all(np.abs(codes[rows]).max(axis=1) == 448.0)
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    # every code is an E4M3 value, and the reconstruction is within half a step
    assert np.array_equal(orc.round_e4m3(codes), codes)
    err = np.abs(codes * scale[:, None] - V)
    step = np.where(np.abs(codes) >= 2.0 ** -6, np.ldexp(1.0, np.frexp(np.abs(codes) + 1e-300)[1] - 4), 2.0 ** -9)
    assert np.all(err <= 0.5 * step * scale[:, None] * (1 + 1e-6) + 1e-12)
