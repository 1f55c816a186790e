"""Plain, slow, fp64 CPU oracle for the Compressed Sparse Attention (CSA) forward path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never calls
it, and this module imports nothing from the product package.

Source of every formula: the page "Compressed Sparse Attention (压缩稀疏注意力)"
(cnblogs), equations (1)-(11) and the paragraphs around them.  Each function
names the equation it restates.  Where the page is silent the reading taken is
stated in the docstring (and listed in the design notes of the repository).

Conventions
-----------
* Every array is ``numpy.float64``; inputs are widened exactly from the bf16 /
  fp32 tensors the GPU path sees.
* Matrices multiply as on the page: ``X @ W`` with ``W`` of shape [in, out].
* Token indices ``t`` are 0-based and local to their sequence.
* ``store`` selects what happens at the points where the GPU path stores an
  intermediate tensor: ``"exact"`` keeps fp64, ``"bf16"`` rounds to bf16
  (round-to-nearest-even), ``"f32"`` rounds to fp32.  In ``"bf16"`` mode the
  indexer head weights w^I are rounded to fp32, because they are kept in fp32.
  The arithmetic between storage points is always fp64.

Parity pins (what checks this oracle against something other than itself) are
in ``tests/test_oracle_pins.py``; every function below has at least one.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "round_bf16",
    "round_f32",
    "round_f16",
    "round_e4m3",
    "quantize_e4m3_rows",
    "storage_round",
    "project",
    "compress",
    "indexer_scores",
    "topk_select",
    "core_attn",
    "num_blocks",
    "compressed_entries",
    "query_rows",
    "csa_forward",
    "csa_forward_sampled",
    "csa_decode_step",
]


# --------------------------------------------------------------------------
# Storage rounding (not part of the method; mirrors where the GPU stores data)
# --------------------------------------------------------------------------

def round_bf16(x):
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    bf16 keeps 8 significant bits.  ``frexp`` gives x = f * 2**e with
    0.5 <= |f| < 1; scaling f by 2**8 puts the kept bits left of the binary
    point, ``np.round`` rounds half to even, and ``ldexp`` scales back.  This
    is exact for every normal bf16 magnitude (the only range the path uses).
    """
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)
    return np.ldexp(np.round(np.ldexp(f, 8)), e - 8)


def round_f32(x):
    """Round fp64 values to the nearest fp32 value (ties to even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_f16(x):
    """Round fp64 values to the nearest fp16 value (ties to even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


E4M3_MAX = 448.0


def round_e4m3(x):
    """Round fp64 values to the nearest FP8 E4M3 value (1 sign, 4 exponent bits
    with bias 7, 3 mantissa bits; ties to even), saturating to +-448, as fp64.

    Normal values (|x| >= 2^-6) have 8 steps per binade, i.e. a spacing of
    2^(e-3) for |x| in [2^e, 2^(e+1)); below 2^-6 the subnormal spacing is
    2^-9.  ``np.round`` rounds half to even on the scaled magnitude.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, E = np.frexp(a)                       # a = f 2^E, 0.5 <= f < 1, so the binade is 2^(E-1)
    e = np.maximum(E - 1, -6)                # subnormals share the spacing of the lowest binade
    step = np.ldexp(1.0, e - 3)
    r = np.round(a / step) * step
    return np.sign(x) * np.minimum(r, E4M3_MAX)


def quantize_e4m3_rows(V):
    """FP8 E4M3 codes and one fp32 scale per row, the quantised cache format.

    V: [N, w] values (the entries as stored in bf16).  Per row:
    scale = max_j |v_j| / 448 in fp32 (1 for an all-zero row), and
    code_j = round_e4m3(v_j / scale) with the division in fp32.  The row is
    represented as code_j * scale.  Returns (codes [N, w], scales [N]) as fp64.
    """
    V = np.asarray(V, dtype=np.float64)
    amax = np.abs(V).max(axis=-1).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    x = V.astype(np.float32) / scale[..., None]
    return round_e4m3(x.astype(np.float64)), scale.astype(np.float64)


def storage_round(x, store):
    """Apply the storage rounding named by ``store`` ("exact", "bf16" or "f32")."""
    if store == "exact":
        return np.asarray(x, dtype=np.float64)
    if store == "bf16":
        return round_bf16(x)
    if store == "f32":
        return round_f32(x)
    raise ValueError(f"unknown storage mode {store!r}")


# --------------------------------------------------------------------------
# Eqs. (1), (2), (5), (6), (7), (10): the projections
# --------------------------------------------------------------------------

def project(X, W):
    """Row-vector projection ``X @ W`` in fp64.

    Eq. (1) C^a = H W^aKV, C^b = H W^bKV; eq. (2) Z^a = H W^aZ, Z^b = H W^bZ;
    eq. (5) c^Q_t = h_t W^DQ; eq. (6) q^I_t = c^Q_t W^UQ (indexer up-projection);
    eq. (7) w^I_t = h_t W^w; eq. (10) q_t = c^Q_t W^UQ (attention up-projection).
    The matrix product is the library primitive the definition names.
    """
    return np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64)


# --------------------------------------------------------------------------
# Eqs. (3), (4): overlapping softmax compression of every m tokens
# --------------------------------------------------------------------------

def num_blocks(L, m):
    """Number of compressed entries of a sequence of L tokens: floor(L / m).

    The page compresses n tokens into n/m entries.  Reading for a length that
    m does not divide: only full blocks are compressed and the tail of
    L mod m tokens is dropped (no query of the sequence could see a partial
    block, because query t sees only blocks s < floor(t/m)).
    """
    return L // m


def compress(Ca, Cb, Za, Zb, Ba, Bb, m):
    """Compressed entries of ONE sequence, eqs. (3)-(4).

    Ca, Cb, Za, Zb: [L, w] (eqs. 1-2); Ba, Bb: [m, w] position biases.
    Returns C^Comp: [floor(L/m), w].

    For entry i and channel j the 2m logits are
        Z^a[m*i + r, j] + B^a[r, j]          (r = 0..m-1, the block itself)
        Z^b[m*(i-1) + r, j] + B^b[r, j]      (r = 0..m-1, the block before)
    Softmax_row normalises these 2m values jointly and independently for each
    channel j (eq. 3 and the paragraph after eq. 4: the row softmax spans the
    2m logits from Z^a and Z^b together).
    Eq. (4) then sums S^a * C^a over the block and S^b * C^b over the block
    before.  At i = 0 the Z^b logits are -inf and the C^b rows are 0, so the
    softmax runs over the m C^a logits only.  Row r of each bias is added to
    the r-th token of its block.
    """
    Ca, Cb, Za, Zb = (np.asarray(a, dtype=np.float64) for a in (Ca, Cb, Za, Zb))
    Ba, Bb = np.asarray(Ba, dtype=np.float64), np.asarray(Bb, dtype=np.float64)
    L, w = Ca.shape
    nb = num_blocks(L, m)
    out = np.zeros((nb, w), dtype=np.float64)
    for i in range(nb):
        a_rows = slice(m * i, m * (i + 1))
        logits_a = Za[a_rows] + Ba                       # [m, w]
        if i == 0:
            logits_b = np.full((m, w), -np.inf)          # padding at i = 0
            Cb_blk = np.zeros((m, w))
        else:
            b_rows = slice(m * (i - 1), m * i)
            logits_b = Zb[b_rows] + Bb
            Cb_blk = Cb[b_rows]
        logits = np.concatenate([logits_a, logits_b], axis=0)   # [2m, w]
        mx = logits.max(axis=0, keepdims=True)
        e = np.exp(logits - mx)                                 # exp(-inf) = 0
        S = e / e.sum(axis=0, keepdims=True)
        out[i] = (S[:m] * Ca[a_rows]).sum(axis=0) + (S[m:] * Cb_blk).sum(axis=0)
    return out


# --------------------------------------------------------------------------
# Eq. (8): lightning-indexer scores;  eq. (9): top-k selection
# --------------------------------------------------------------------------

def indexer_scores(qI_t, wI_t, KI_avail):
    """Index scores of one query token against its visible blocks, eq. (8).

    qI_t: [n_h^I, c^I] indexer queries of token t (eq. 6, heads in the order
    of the concatenation); wI_t: [n_h^I] head weights (eq. 7); KI_avail:
    [avail, c^I] the compressed indexer keys K^IComp_s for s < floor(t/m).
    Returns I[t, s] = sum_h w_{t,h} * ReLU(q^I_{t,h} . K^IComp_s), shape [avail].
    No scaling and no softmax are applied to the scores (the page has none).
    """
    qI_t = np.asarray(qI_t, dtype=np.float64)
    wI_t = np.asarray(wI_t, dtype=np.float64)
    KI_avail = np.asarray(KI_avail, dtype=np.float64)
    if KI_avail.shape[0] == 0:
        return np.zeros(0)
    dots = qI_t @ KI_avail.T                     # [n_h^I, avail]
    return wI_t @ np.maximum(dots, 0.0)


def topk_select(scores, k):
    """Top-k block indices of one query, eq. (9), padded with -1 to length k.

    Readings where the page is silent: k is clamped to the number of visible
    blocks; equal scores are ordered by the lower block index s.  The result
    lists the chosen indices in ascending s (a top-k result is a set).
    """
    scores = np.asarray(scores, dtype=np.float64)
    avail = scores.shape[0]
    keff = min(k, avail)
    s = np.arange(avail)
    order = np.lexsort((s, -scores))            # primary key -score, then s
    chosen = np.sort(order[:keff])
    out = np.full(k, -1, dtype=np.int64)
    out[:keff] = chosen
    return out


# --------------------------------------------------------------------------
# Eq. (11): shared-KV MQA
# --------------------------------------------------------------------------

def core_attn(q_t, C_sel):
    """Shared key-value multi-query attention of one token, eq. (11).

    q_t: [n_h, c] attention queries (eq. 10); C_sel: [k_eff, c] the selected
    compressed entries, each serving as key AND value for every head.
    CoreAttn is read as softmax(q . K^T / sqrt(c)) . V per head.
    With no selected entry the output is 0.
    """
    q_t = np.asarray(q_t, dtype=np.float64)
    C_sel = np.asarray(C_sel, dtype=np.float64)
    nh, c = q_t.shape
    if C_sel.shape[0] == 0:
        return np.zeros((nh, c))
    sc = (q_t @ C_sel.T) / math.sqrt(c)          # [n_h, k_eff]
    sc = sc - sc.max(axis=1, keepdims=True)
    p = np.exp(sc)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ C_sel


# --------------------------------------------------------------------------
# Whole forward pass over packed sequences
# --------------------------------------------------------------------------

_HSIDE = ("W_aKV", "W_bKV", "W_aZ", "W_bZ", "W_aKV_I", "W_bKV_I", "W_aZ_I", "W_bZ_I")


def compressed_entries(H, W, dims, seqlens, store="exact"):
    """The token-parallel half of the forward pass: eqs. (1), (2), the
    indexer-key projections, and eqs. (3), (4) per sequence.

    Returns (C_comp [NB, c], K_icomp [NB, c^I], cu [nseq+1], cu_blocks [nseq+1]).
    Arguments as for ``csa_forward``.
    """
    H = np.asarray(H, dtype=np.float64)
    m, c, cI = dims["m"], dims["c"], dims["cI"]
    assert sum(seqlens) == H.shape[0]
    rnd = lambda x: storage_round(x, store)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    cu_blocks = np.concatenate([[0], np.cumsum([num_blocks(L, m) for L in seqlens])]).astype(np.int64)
    proj = {name: rnd(project(H, W[name])) for name in _HSIDE}
    C_comp_parts, K_icomp_parts = [], []
    for b, L in enumerate(seqlens):
        sl = slice(cu[b], cu[b] + L)
        C_comp_parts.append(compress(proj["W_aKV"][sl], proj["W_bKV"][sl], proj["W_aZ"][sl],
                                     proj["W_bZ"][sl], W["B_a"], W["B_b"], m))
        K_icomp_parts.append(compress(proj["W_aKV_I"][sl], proj["W_bKV_I"][sl], proj["W_aZ_I"][sl],
                                      proj["W_bZ_I"][sl], W["B_a_I"], W["B_b_I"], m))
    C_comp = rnd(np.concatenate(C_comp_parts, axis=0)) if C_comp_parts else np.zeros((0, c))
    K_icomp = rnd(np.concatenate(K_icomp_parts, axis=0)) if K_icomp_parts else np.zeros((0, cI))
    return C_comp, K_icomp, cu, cu_blocks


def query_rows(H, W, dims, C_comp, K_icomp, cu, cu_blocks, rows, store="exact", keep_scores=False):
    """The per-query half of the forward pass for the global rows ``rows``:
    eqs. (5), (6), (7), (10), then eq. (8) over the visible blocks, eq. (9)
    and eq. (11), given the compressed entries of ``compressed_entries``.

    Returns a dict with, per row, idx [R, topk], O [R, n_h, c], cQ, wI, qI,
    q and, if keep_scores, the list of score rows.
    """
    H = np.asarray(H, dtype=np.float64)
    m, k = dims["m"], dims["topk"]
    nh, nhI, c, cI = dims["nh"], dims["nhI"], dims["c"], dims["cI"]
    rnd = lambda x: storage_round(x, store)
    rnd_w = (lambda x: round_f32(x)) if store == "bf16" else rnd
    rows = np.asarray(rows, dtype=np.int64)
    seq_of = np.searchsorted(cu, rows, side="right") - 1

    cQ = rnd(project(H[rows], W["W_DQ"]))                    # [R, d_c]
    wI = rnd_w(project(H[rows], W["W_w"]))                   # [R, n_h^I]
    qI = rnd(project(cQ, W["W_IUQ"])).reshape(len(rows), nhI, cI)
    q = rnd(project(cQ, W["W_UQ"])).reshape(len(rows), nh, c)

    idx = np.full((len(rows), k), -1, dtype=np.int64)
    O = np.zeros((len(rows), nh, c))
    scores = []
    for r, (tg, b) in enumerate(zip(rows, seq_of)):
        t = int(tg - cu[b])                                  # local token index
        avail = t // m                                       # blocks s < floor(t/m)
        base = int(cu_blocks[b])
        I_t = indexer_scores(qI[r], wI[r], K_icomp[base:base + avail])      # eq. (8)
        sel = topk_select(I_t, k)                                           # eq. (9)
        idx[r] = sel
        chosen = sel[sel >= 0]
        O[r] = core_attn(q[r], C_comp[base + chosen])                       # eq. (11)
        if keep_scores:
            scores.append(I_t)
    out = {"rows": rows, "idx": idx, "O": O, "cQ": cQ, "wI": wI, "qI": qI, "q": q}
    if keep_scores:
        out["scores"] = scores
    return out


def csa_forward(H, W, dims, seqlens, store="exact", rows=None, keep_scores=False):
    """CSA forward pass, eqs. (1)-(11), over packed sequences.

    H: [T, d] hidden states of all sequences, packed in order.
    W: dict of weights, shapes as on the page ([in, out]):
       W_aKV, W_bKV, W_aZ, W_bZ [d, c]; B_a, B_b [m, c];
       W_aKV_I, W_bKV_I, W_aZ_I, W_bZ_I [d, c^I]; B_a_I, B_b_I [m, c^I]
       (the page builds the indexer keys by the same kind of compression as
       C^Comp without naming its parameters; read as a separate parameter
       set of the same form with width c^I);
       W_DQ [d, d_c]; W_IUQ [d_c, n_h^I c^I] (eq. 6); W_UQ [d_c, n_h c]
       (eq. 10 -- the page reuses the symbol W^UQ with a second shape, read as
       a second matrix); W_w [d, n_h^I].
    dims: dict with keys m, topk, nh, nhI, c, cI.
    seqlens: lengths of the packed sequences (sum = T).  Compression blocks
       never cross a sequence boundary.
    store: storage rounding mode (module docstring).
    rows: global query rows to evaluate (default: all).  Compressed entries
       are always computed for every block.
    Returns a dict with C_comp [NB, c], K_icomp [NB, c^I], cu_blocks, and per
    evaluated row: idx [R, topk] (local block indices, -1 padded), O [R, n_h, c]
    and, if keep_scores, the list of score rows.
    The work is the two halves ``compressed_entries`` (eqs. 1-4) and
    ``query_rows`` (eqs. 5-11), in that order.
    """
    H = np.asarray(H, dtype=np.float64)
    C_comp, K_icomp, cu, cu_blocks = compressed_entries(H, W, dims, seqlens, store)
    if rows is None:
        rows = np.arange(H.shape[0])
    out = query_rows(H, W, dims, C_comp, K_icomp, cu, cu_blocks, rows, store, keep_scores)
    out.update({"C_comp": C_comp, "K_icomp": K_icomp, "cu_blocks": cu_blocks})
    return out


def csa_forward_sampled(H, W, dims, seqlens, rows, store="bf16", chunk=8192):
    """``csa_forward`` restricted to ``rows``, for inputs too large to hold in fp64.

    The same equations in the same order; only the bookkeeping differs:
    H (any array-like of shape [T, d], e.g. a bf16 torch tensor) is widened
    to fp64 ``chunk`` tokens at a time, and each chunk's eight H-side
    projections (eqs. 1, 2 and the indexer copies) are stored after storage
    rounding.  With ``store="bf16"`` they are kept in fp32, which holds every
    bf16 value exactly; with ``"exact"`` they stay fp64.  Compression, the
    indexer, top-k and CoreAttn then run as in ``csa_forward``.
    Returns the same keys as ``csa_forward`` for the requested rows.
    """
    m, k = dims["m"], dims["topk"]
    nh, nhI, c, cI = dims["nh"], dims["nhI"], dims["c"], dims["cI"]
    T = sum(seqlens)
    rnd = lambda x: storage_round(x, store)
    rnd_w = (lambda x: round_f32(x)) if store == "bf16" else rnd
    keep = np.float32 if store in ("bf16", "f32") else np.float64

    def rows_f64(a, b):
        x = H[a:b]
        if hasattr(x, "double"):               # a torch tensor
            x = x.double().numpy()
        return np.asarray(x, dtype=np.float64)

    Wcat = np.concatenate([np.asarray(W[n], dtype=np.float64) for n in _HSIDE], axis=1)
    widths = [c, c, c, c, cI, cI, cI, cI]
    offs = np.concatenate([[0], np.cumsum(widths)])
    proj = np.empty((T, int(offs[-1])), dtype=keep)
    for a in range(0, T, chunk):
        b = min(T, a + chunk)
        proj[a:b] = rnd(project(rows_f64(a, b), Wcat))
    part = lambda j, sl: proj[sl, offs[j]:offs[j + 1]]

    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    cu_blocks = np.concatenate([[0], np.cumsum([num_blocks(L, m) for L in seqlens])]).astype(np.int64)
    C_parts, K_parts = [], []
    for b, L in enumerate(seqlens):
        sl = slice(cu[b], cu[b] + L)
        C_parts.append(compress(part(0, sl), part(1, sl), part(2, sl), part(3, sl), W["B_a"], W["B_b"], m))
        K_parts.append(compress(part(4, sl), part(5, sl), part(6, sl), part(7, sl), W["B_a_I"], W["B_b_I"], m))
    del proj
    C_comp = rnd(np.concatenate(C_parts, axis=0))
    K_icomp = rnd(np.concatenate(K_parts, axis=0))

    rows = np.asarray(rows, dtype=np.int64)
    seq_of = np.searchsorted(cu, rows, side="right") - 1
    Hr = np.concatenate([rows_f64(int(t), int(t) + 1) for t in rows]) if len(rows) else np.zeros((0, H.shape[1]))
    cQ = rnd(project(Hr, W["W_DQ"]))
    wI = rnd_w(project(Hr, W["W_w"]))
    qI = rnd(project(cQ, W["W_IUQ"])).reshape(len(rows), nhI, cI)
    q = rnd(project(cQ, W["W_UQ"])).reshape(len(rows), nh, c)
    idx = np.full((len(rows), k), -1, dtype=np.int64)
    O = np.zeros((len(rows), nh, c))
    scores = []
    for r, (tg, b) in enumerate(zip(rows, seq_of)):
        t = int(tg - cu[b])
        avail = t // m
        base = int(cu_blocks[b])
        I_t = indexer_scores(qI[r], wI[r], K_icomp[base:base + avail])
        sel = topk_select(I_t, k)
        idx[r] = sel
        O[r] = core_attn(q[r], C_comp[base + sel[sel >= 0]])
        scores.append(I_t)
    return {"C_comp": C_comp, "K_icomp": K_icomp, "cu_blocks": cu_blocks, "rows": rows, "idx": idx, "O": O,
            "cQ": cQ, "wI": wI, "qI": qI, "q": q, "scores": scores}


# --------------------------------------------------------------------------
# One decode step over a compressed cache
# --------------------------------------------------------------------------

def csa_decode_step(h, pos, C_cache, K_cache, cache_len, ring, W, dims, store="exact", detail=None,
                    kcache="plain"):
    """One new token per sequence attending over a compressed cache.

    The same equations as ``csa_forward`` for a single query token t = pos[b]
    of each independent sequence b:
      * eqs. (1), (2), (5), (7) project h_t; the token's rows
        [C^a | C^b | Z^a | Z^b | C^aI | C^bI | Z^aI | Z^bI] are written into
        ring slot t mod 2m (the ring holds the raw rows of the last 2m tokens,
        which is what eqs. (3)-(4) need to build the next entry);
      * when t + 1 is a multiple of m, block i = (t + 1)/m - 1 is complete and
        eqs. (3)-(4) compress it (C^a rows of block i, C^b rows of block i-1,
        or the i = 0 padding) into cache entry i (C^Comp and K^IComp);
      * eqs. (8), (9), (10), (11) then run for t over the visible entries
        s < floor(t/m).  The entry appended at this step is never visible
        to t (it contains t).
    C_cache [B, cap, c], K_cache [B, cap, c^I], cache_len [B] and ring
    [B, 2m, 4c + 4c^I] are updated IN PLACE (copies are the caller's choice).
    cache_len[b] must equal floor(t/m) on entry.
    kcache="e4m3" is the quantised indexer-key cache (a format of this
    implementation, not of the page): K_cache then holds every entry as
    code * scale (quantize_e4m3_rows of its bf16 value), an appended entry is
    quantised the same way, and the indexer queries enter eq. (8) rounded to
    fp16, the precision the quantised kernels multiply them in.
    Returns (O [B, n_h, c], idx [B, topk]).  If ``detail`` is a dict it
    receives per sequence the scores I_t, the attention queries q_t and the
    indexer inputs q^I_t and w^I_t.
    """
    m, k = dims["m"], dims["topk"]
    nh, nhI, c, cI = dims["nh"], dims["nhI"], dims["c"], dims["cI"]
    h = np.asarray(h, dtype=np.float64)
    B = h.shape[0]
    rnd = lambda x: storage_round(x, store)
    rnd_w = (lambda x: round_f32(x)) if store == "bf16" else rnd
    widths = [c, c, c, c, cI, cI, cI, cI]
    offs = np.concatenate([[0], np.cumsum(widths)])

    O = np.zeros((B, nh, c))
    idx = np.full((B, k), -1, dtype=np.int64)
    for b in range(B):
        t = int(pos[b])
        assert cache_len[b] == t // m, "cache_len must equal floor(t/m)"
        row = np.concatenate([rnd(project(h[b:b + 1], W[name]))[0] for name in _HSIDE])
        ring[b, t % (2 * m)] = row
        if (t + 1) % m == 0:
            i = (t + 1) // m - 1
            part = lambda slot_tokens, j: np.stack(
                [ring[b, tok % (2 * m), offs[j]:offs[j + 1]] for tok in slot_tokens])
            a_tok = list(range(m * i, m * (i + 1)))
            if i == 0:
                # i = 0 has no block before it; compress() pads it itself.
                for j0, bias_a, bias_b, cache, wdt in ((0, "B_a", "B_b", C_cache, c),
                                                       (4, "B_a_I", "B_b_I", K_cache, cI)):
                    Ca, Za = part(a_tok, j0), part(a_tok, j0 + 2)
                    ent = compress(Ca, np.zeros((m, wdt)), Za, np.zeros((m, wdt)),
                                   W[bias_a], W[bias_b], m)[0]
                    cache[b, i] = rnd(ent)
            else:
                b_tok = list(range(m * (i - 1), m * i))
                for j0, bias_a, bias_b, cache in ((0, "B_a", "B_b", C_cache),
                                                  (4, "B_a_I", "B_b_I", K_cache)):
                    # Lay out the 2m tokens [block i-1 ; block i] as one short
                    # sequence and take its entry 1: eqs. (3)-(4) for entry i.
                    Ca = np.concatenate([part(b_tok, j0), part(a_tok, j0)])
                    Cb = np.concatenate([part(b_tok, j0 + 1), part(a_tok, j0 + 1)])
                    Za = np.concatenate([part(b_tok, j0 + 2), part(a_tok, j0 + 2)])
                    Zb = np.concatenate([part(b_tok, j0 + 3), part(a_tok, j0 + 3)])
                    ent = compress(Ca, Cb, Za, Zb, W[bias_a], W[bias_b], m)[1]
                    cache[b, i] = rnd(ent)
            if kcache == "e4m3":
                codes, scale = quantize_e4m3_rows(K_cache[b, i][None, :])
                K_cache[b, i] = codes[0] * scale[0]
            cache_len[b] = i + 1
        avail = t // m
        cQ = rnd(project(h[b:b + 1], W["W_DQ"]))
        wI = rnd_w(project(h[b:b + 1], W["W_w"]))[0]
        qI = rnd(project(cQ, W["W_IUQ"]))[0].reshape(nhI, cI)
        if kcache == "e4m3":
            qI = round_f16(qI)
        q = rnd(project(cQ, W["W_UQ"]))[0].reshape(nh, c)
        I_t = indexer_scores(qI, wI, K_cache[b, :avail])
        sel = topk_select(I_t, k)
        idx[b] = sel
        O[b] = core_attn(q, C_cache[b, sel[sel >= 0]])
        if detail is not None:
            detail.setdefault("scores", []).append(I_t)
            detail.setdefault("q", []).append(q)
            detail.setdefault("qI", []).append(qI)
            detail.setdefault("wI", []).append(wI)
    return O, idx
