"""Plain fp64 CPU oracle of the token-level sparse-attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
anything under ``oracle/``.  The product path (the CUDA library and its Python
binding) never reaches this file, and this file imports nothing from the
product package: it works on numpy arrays of raw input bytes.

Every function is the plain definition from the pages, in fp64, with library
primitives (matmul, stable sort, exp, log) as steps and no blocking or fusion:

* ``index_score``     LongCat Sparse Attention（LSA）完全拆解, §"DSA 基线：闪电索引器是怎么工作的",
                      equation I_{t,s} = sum_j w_{t,j} * ReLU(q_{t,j} . k_s), s <= t.
* ``topk_select``     same page, same section, S_t = arg topK({I_{t,s}}_{s<=t}, K); and
                      §"机制一：流式感知索引（SI）/ 预算分解": S_t = S_sink u S_swa u S_sparse with
                      S_sparse = arg topK over s not in S_sink u S_swa.
* ``pool_keys``       same page, §"机制三：层级索引（HI）" (mean of the member index keys,
                      computed once and cached); lecture "从两本账看懂长上下文注意力",
                      §"Qwen Sparse Attention" (index keys mean-pooled in 4-token micro-blocks).
* ``bucket_select``   "LSA 稀疏注意力會省顯存嗎", §二 steps 2-4 (buckets keep a
                      representative and member positions; Flat compares representatives,
                      expands to positions, adds sink and window); lecture §"Qwen Sparse
                      Attention" and §"尾部计数与 query 自身" (complete micro-blocks are ranked,
                      visible tokens of the incomplete tail block are read directly).
* ``hi_select_row``   LongCat page §"机制三：层级索引（HI）": page scores from the sub-blocks' mean
                      keys, top-M pages, then the token score and arg topK on the recalled tokens.
* ``msa_select_row``  lecture "从两本账看懂长上下文注意力", §"MiniMax Sparse Attention": block score = max of
                      its tokens' index scores, per-group top-k blocks, the local block always kept.
* ``tree_select_row`` "LSA 稀疏注意力會省顯存嗎", §二 step 3 (the Tree version searches level by level,
                      keeping candidates at each level); "超长上下文LSA注意力技术开源", §"Qwen LSA注意力优化原理与
                      核心创新" (keys clustered into a tree; the query scans only cluster centres, then picks
                      buckets).  Two levels over the Flat buckets; parity unpinned beyond the pins in the tests
                      (full beam = Flat, one child per parent = Flat, a hand-built case where a parent's mean
                      hides its best child).
* ``lse_merge``       LongCat page §"训练与 kernel：混合稀疏注意力算子（HFA）": partial attentions merged by
                      online-softmax (log-sum-exp) rescaling.
* ``softmax_attention`` / ``sparse_mla_attn``
                      LongCat page §"DSA 基线", u_t = Attn(h_t, {c_s | s in S_t}) in the absorbed
                      MQA form (one latent c_s shared by all heads; value = first 512 dims);
                      "LSA 稀疏注意力會省顯存嗎" §四 (score q.k/sqrt(d), softmax, weighted V).

Readings where the pages are silent:
  positions are 0-based; the window includes the query position itself; K counts
  only the dynamic part; ties at the K-th score go to the lower position / bucket
  id; fewer candidates than K means all are taken; an empty set gives output 0 and
  lse = -inf; in bucket / micro-block mode a bucket overlapping sink or window is
  allowed and the union is de-duplicated; members beyond q_pos are dropped.
"""

from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Input decoding (exact)
# ---------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16/int16) -> float64, exactly (bf16 = top half of fp32)."""
    b = np.asarray(bits).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 (e4m3fn) codes -> float64 from the format definition.

    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
    subnormal (m/8 * 2^-6); S.1111.111 is NaN; there are no infinities.
    """
    c = np.asarray(codes).view(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = np.where(e == 0, sub, normal) * sign
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


# ---------------------------------------------------------------------------
# a1: lightning-indexer score
# ---------------------------------------------------------------------------


def index_score(q_I: np.ndarray, w: np.ndarray, k_I: np.ndarray, q_pos: np.ndarray,
                chunk: int = 1 << 15) -> np.ndarray:
    """I[b, s] = sum_j w[b, j] * max(0, q_I[b, j, :] . k_I[s, :]) for s <= q_pos[b], else -inf.

    q_I [B, H_I, d] fp64, w [B, H_I] fp64, k_I [L, d] fp64 (already dequantized:
    in the FP8 mode q_I = code * q_scale[b, j] and k_I = code * k_scale[s]).
    """
    q_I = np.asarray(q_I, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k_I = np.asarray(k_I, dtype=np.float64)
    B, H, d = q_I.shape
    L = k_I.shape[0]
    out = np.full((B, L), -np.inf, dtype=np.float64)
    qf = q_I.reshape(B * H, d)
    for s0 in range(0, L, chunk):
        s1 = min(L, s0 + chunk)
        dots = k_I[s0:s1] @ qf.T  # [n, B*H]: q_{b,j} . k_s
        relu = np.maximum(dots, 0.0).reshape(s1 - s0, B, H)
        out[:, s0:s1] = np.einsum("nbh,bh->bn", relu, w)
    pos = np.arange(L)
    out[pos[None, :] > np.asarray(q_pos)[:, None]] = -np.inf
    return out


# ---------------------------------------------------------------------------
# a2: top-K with the sink / window union
# ---------------------------------------------------------------------------


def fixed_positions(q_pos: int, sink: int, window: int) -> tuple[np.ndarray, np.ndarray]:
    """S_sink = {0..sink-1} and S_swa = {q_pos-window+1..q_pos}, clipped to [0, q_pos]."""
    q_pos = int(q_pos)
    s_sink = np.arange(0, min(sink, q_pos + 1), dtype=np.int64)
    s_swa = np.arange(max(0, q_pos - window + 1), q_pos + 1, dtype=np.int64) if window > 0 else np.zeros(0, np.int64)
    return s_sink, s_swa


def topk_row(scores_row: np.ndarray, q_pos: int, K: int, sink: int, window: int):
    """One query: (sorted selected positions, K-th selected score, candidate count).

    Candidates are the visible positions outside sink u window; they are ordered
    by a stable sort on descending score, so equal scores keep ascending position.
    """
    s_sink, s_swa = fixed_positions(q_pos, sink, window)
    visible = np.arange(0, int(q_pos) + 1, dtype=np.int64)
    fixed = np.union1d(s_sink, s_swa)
    cand = np.setdiff1d(visible, fixed, assume_unique=True)
    order = np.argsort(-scores_row[cand], kind="stable")
    take = cand[order[: min(K, cand.size)]]
    kth = scores_row[take[-1]] if take.size else -np.inf
    sel = np.union1d(np.union1d(s_sink, take), s_swa)
    return sel.astype(np.int64), float(kth), int(cand.size)


def topk_select(scores: np.ndarray, q_pos: np.ndarray, K: int, sink: int = 0, window: int = 0):
    """All rows: list of sorted int64 position arrays, and the K-th scores."""
    sets, kths = [], []
    for b in range(scores.shape[0]):
        sel, kth, _ = topk_row(scores[b], int(q_pos[b]), K, sink, window)
        sets.append(sel)
        kths.append(kth)
    return sets, np.array(kths)


# ---------------------------------------------------------------------------
# a0 / a3: representatives and bucket / micro-block selection
# ---------------------------------------------------------------------------


def pool_keys(k_I: np.ndarray, members: np.ndarray | None = None, block: int | None = None) -> np.ndarray:
    """Representative of each bucket = mean of its members' index keys (fp64).

    members [NB, bsz] explicit positions (Flat buckets), or ``block`` for
    contiguous micro-blocks {n*block .. n*block+block-1}, complete blocks only.
    """
    k_I = np.asarray(k_I, dtype=np.float64)
    if members is not None:
        return k_I[np.asarray(members, dtype=np.int64)].mean(axis=1)
    nb = k_I.shape[0] // block
    return k_I[: nb * block].reshape(nb, block, -1).mean(axis=1)


def bucket_scores(q_I: np.ndarray, w: np.ndarray, reps: np.ndarray) -> np.ndarray:
    """Representative score with the indexer's formula: sum_j w_j ReLU(q_j . c)."""
    q_I = np.asarray(q_I, dtype=np.float64)
    B, H, d = q_I.shape
    dots = np.asarray(reps, dtype=np.float64) @ q_I.reshape(B * H, d).T  # [NB, B*H]
    relu = np.maximum(dots, 0.0).reshape(-1, B, H)
    return np.einsum("nbh,bh->bn", relu, np.asarray(w, dtype=np.float64))


def bucket_select_row(bscore_row: np.ndarray, q_pos: int, M: int, sink: int, window: int,
                      members: np.ndarray | None = None, block: int | None = None):
    """One query: (sorted positions, M-th bucket score, number of ranked buckets).

    Flat mode (``members``): every bucket is ranked.  Micro-block mode
    (``block``): only the floor((q_pos+1)/block) complete visible blocks are
    ranked, and the tail {block*floor((q_pos+1)/block) .. q_pos} is added directly.
    Top-M buckets by a stable sort on descending score (ties -> lower bucket id),
    expanded to their positions, union sink and window, clipped to [0, q_pos].
    """
    q_pos = int(q_pos)
    if members is not None:
        nrank = bscore_row.shape[0]
    else:
        nrank = min(bscore_row.shape[0], (q_pos + 1) // block)
    order = np.argsort(-bscore_row[:nrank], kind="stable")
    chosen = order[: min(M, nrank)]
    mth = float(bscore_row[chosen[-1]]) if chosen.size else -np.inf
    if members is not None:
        pos = np.asarray(members, dtype=np.int64)[chosen].reshape(-1)
        tail = np.zeros(0, np.int64)
    else:
        pos = (chosen[:, None] * block + np.arange(block)[None, :]).reshape(-1).astype(np.int64)
        tail = np.arange(((q_pos + 1) // block) * block, q_pos + 1, dtype=np.int64)
    s_sink, s_swa = fixed_positions(q_pos, sink, window)
    sel = np.unique(np.concatenate([s_sink, pos, tail, s_swa]))
    sel = sel[(sel >= 0) & (sel <= q_pos)]
    return sel.astype(np.int64), mth, int(nrank)


# ---------------------------------------------------------------------------
# HI: two-stage (page -> token) selection
# ---------------------------------------------------------------------------


def hi_select_row(q_I_b: np.ndarray, w_b: np.ndarray, k_I: np.ndarray, q_pos: int, P: int, Bsub: int, M: int,
                  K: int, sink: int, window: int):
    """One query of the hierarchical index: (sorted positions, K-th token score, M-th page score, recalled).

    LongCat page §"机制三：层级索引（HI）".  Stage one: the sequence is cut into pages of P tokens and
    sub-blocks of Bsub tokens; each sub-block n keeps the mean of its index keys; the page score is
    I_page(p) = sum_j w_j sum_{n in page p} ReLU(q_j . kmean_n); the M best pages among p <= q_pos/P
    (0-based: pages that start at or before the query) are recalled (stable sort on descending score:
    ties -> lower page id).  Stage two: the token score I_{t,s} (the indexer formula) on the recalled
    tokens only, and the same sink / window union and arg topK as ``topk_row`` over them.

    Readings: a page's score sums its complete sub-blocks that are entirely visible (end <= q_pos);
    the visible tokens of the sub-block holding q_pos that is not entirely visible, i.e.
    {Bsub*floor((q_pos+1)/Bsub) .. q_pos}, have no mean key and join the recalled tokens directly (as
    the micro-block tail).  Recalled tokens are clipped to [0, q_pos].
    """
    q_pos = int(q_pos)
    k_I = np.asarray(k_I, dtype=np.float64)
    L = k_I.shape[0]
    # stage one: sub-block means and their indexer scores, summed per page
    nvis = min(L // Bsub, (q_pos + 1) // Bsub)  # complete sub-blocks entirely visible
    kmean = pool_keys(k_I, block=Bsub)[:nvis]
    sub = bucket_scores(np.asarray(q_I_b, np.float64)[None], np.asarray(w_b, np.float64)[None], kmean)[0]
    per_page = P // Bsub
    npages = q_pos // P + 1
    page = np.zeros(npages)
    for p in range(npages):
        page[p] = sub[p * per_page: min((p + 1) * per_page, nvis)].sum()
    order = np.argsort(-page, kind="stable")
    chosen = order[: min(M, npages)]
    mth_page = float(page[chosen[-1]]) if chosen.size else -np.inf
    recalled = (chosen[:, None] * P + np.arange(P)[None, :]).reshape(-1)
    tail = np.arange(((q_pos + 1) // Bsub) * Bsub, q_pos + 1)
    recalled = np.union1d(recalled, tail).astype(np.int64)
    recalled = recalled[recalled <= q_pos]
    # stage two: token scores on the recalled tokens, sink / window union, arg topK
    scores = index_score(np.asarray(q_I_b)[None], np.asarray(w_b)[None], k_I[recalled],
                         np.array([len(recalled) - 1]))[0]
    s_sink, s_swa = fixed_positions(q_pos, sink, window)
    fixed = np.union1d(s_sink, s_swa)
    keep = ~np.isin(recalled, fixed)
    cand, cand_sc = recalled[keep], scores[keep]
    order = np.argsort(-cand_sc, kind="stable")
    take = cand[order[: min(K, cand.size)]]
    kth = float(cand_sc[order[min(K, cand.size) - 1]]) if cand.size else -np.inf
    sel = np.union1d(np.union1d(s_sink, take), s_swa)
    return sel.astype(np.int64), kth, mth_page, recalled


# ---------------------------------------------------------------------------
# MSA: group-wise block selection
# ---------------------------------------------------------------------------


def msa_select_row(q_I_b: np.ndarray, w_b: np.ndarray, k_I: np.ndarray, q_pos: int, G: int, block: int, KB: int):
    """One query of group-wise block selection: per group g, (sorted positions, KB-th block score).

    Lecture "从两本账看懂长上下文注意力", section "MiniMax Sparse Attention": the index branch scores tokens,
    a block's score is the max of its tokens' scores, each GQA group picks its own top-k blocks (its query
    heads share them) and the current local block is always kept.

    Readings: group g's token score is the indexer formula over its own index heads
    j in [g*H_I/G, (g+1)*H_I/G); the ranked blocks are those entirely before the local block (the block
    holding q_pos), i.e. c < q_pos // block; the top-KB of them (stable sort on descending score: ties ->
    lower block) plus the local block's visible tokens {block*(q_pos//block) .. q_pos} form the group's set.
    """
    q_pos = int(q_pos)
    H = q_I_b.shape[0]
    hg = H // G
    lb = q_pos // block
    out = []
    for g in range(G):
        sl = slice(g * hg, (g + 1) * hg)
        sc = index_score(np.asarray(q_I_b)[None, sl], np.asarray(w_b)[None, sl], np.asarray(k_I)[: lb * block],
                         np.array([lb * block - 1]))[0] if lb > 0 else np.zeros(0)
        bscore = sc.reshape(lb, block).max(axis=1) if lb > 0 else np.zeros(0)
        order = np.argsort(-bscore, kind="stable")
        chosen = order[: min(KB, lb)]
        kth = float(bscore[chosen[-1]]) if chosen.size else -np.inf
        pos = (chosen[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        pos = np.union1d(pos, np.arange(lb * block, q_pos + 1)).astype(np.int64)
        out.append((pos, kth))
    return out


# ---------------------------------------------------------------------------
# D-LSA Tree: level-by-level search over cluster centres, then the Flat buckets
# ---------------------------------------------------------------------------


def tree_parents(reps: np.ndarray, F: int) -> np.ndarray:
    """Level-2 centres: parent p is the plain mean of the representatives of buckets [p*F, min((p+1)*F, NB)).

    The pages give no rule for building the tree; grouping F consecutive bucket ids under one parent, with the
    parent's centre the mean of its children's centres, is the plainest reading (a clusterer that emits its
    buckets in cluster order gives exactly this layout)."""
    reps = np.asarray(reps, dtype=np.float64)
    nb = reps.shape[0]
    return np.stack([reps[p * F: min((p + 1) * F, nb)].mean(axis=0) for p in range(-(-nb // F))])


def tree_select_row(q_I_b: np.ndarray, w_b: np.ndarray, reps: np.ndarray, members: np.ndarray, F: int, M2: int,
                    M: int, q_pos: int, sink: int, window: int):
    """One query of the two-level tree search: (sorted positions, M-th candidate bucket score, M2-th parent score).

    Level 2: every parent centre is scored with the indexer formula and the M2 best parents are kept (stable
    sort on descending score: ties -> lower parent id).  Level 1: the kept parents' children (ascending bucket
    id) are the candidates; they are scored the same way and the M best are kept (ties -> lower bucket id).
    The kept buckets expand to their members, with sink and window, clipped to [0, q_pos], as in Flat mode.
    """
    q_pos = int(q_pos)
    reps = np.asarray(reps, dtype=np.float64)
    nb = reps.shape[0]
    q = np.asarray(q_I_b)[None]
    w = np.asarray(w_b)[None]
    parents = tree_parents(reps, F)
    ps = bucket_scores(q, w, parents)[0]
    porder = np.argsort(-ps, kind="stable")
    n2 = min(M2, parents.shape[0])
    kept_parents = np.sort(porder[:n2])
    m2th = float(ps[porder[n2 - 1]])
    cand = np.concatenate([np.arange(p * F, min((p + 1) * F, nb)) for p in kept_parents]).astype(np.int64)
    cs = bucket_scores(q, w, reps[cand])[0]
    corder = np.argsort(-cs, kind="stable")
    n1 = min(M, cand.size)
    chosen = cand[corder[:n1]]
    mth = float(cs[corder[n1 - 1]])
    pos = np.asarray(members, dtype=np.int64)[chosen].reshape(-1)
    s_sink, s_swa = fixed_positions(q_pos, sink, window)
    sel = np.unique(np.concatenate([s_sink, pos, s_swa]))
    sel = sel[(sel >= 0) & (sel <= q_pos)]
    return sel.astype(np.int64), mth, m2th


# ---------------------------------------------------------------------------
# a4: sparse attention over the MLA latent
# ---------------------------------------------------------------------------


def softmax_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """o = softmax(scale * q K^T) V per query row, two passes (max, then sums).

    q [H, d_k], keys [n, d_k], values [n, d_v].  Returns (o [H, d_v], lse [H]);
    an empty key set gives o = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    H = q.shape[0]
    if keys.shape[0] == 0:
        return np.zeros((H, values.shape[1])), np.full(H, -np.inf)
    z = scale * (q @ keys.T)  # [H, n]
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ values) / l
    lse = m[:, 0] + np.log(l[:, 0])
    return o, lse


def sparse_mla_attn(q: np.ndarray, kv_rows: np.ndarray, scale: float, d_v: int = 512):
    """Absorbed-MQA form: each gathered latent row c_s [d_qk] is the key, its first d_v dims the value."""
    kv_rows = np.asarray(kv_rows, dtype=np.float64)
    return softmax_attention(q, kv_rows, kv_rows[:, :d_v], scale)


def lse_merge(parts):
    """Online-softmax merge of partial attentions over disjoint key sets: [(o_i [H, d_v], lse_i [H])] ->
    (o, lse) of the attention over their union.

    LongCat page §"训练与 kernel：混合稀疏注意力算子（HFA）": the sparse and sliding-window operators' partial
    outputs are combined by rescaling with their log-sum-exp statistics.  With m = max_i lse_i:
    o = sum_i exp(lse_i - m) o_i / sum_i exp(lse_i - m), lse = m + log sum_i exp(lse_i - m); parts with
    lse = -inf (empty key sets) carry no weight.
    """
    os_ = [np.asarray(o, dtype=np.float64) for o, _ in parts]
    ls = np.stack([np.asarray(l, dtype=np.float64) for _, l in parts])  # [n, H]
    m = ls.max(axis=0)
    out = np.zeros_like(os_[0])
    lse = np.full(ls.shape[1], -np.inf)
    ok = np.isfinite(m)
    if ok.any():
        wts = np.where(np.isfinite(ls[:, ok]), np.exp(ls[:, ok] - m[ok]), 0.0)  # [n, H']
        den = wts.sum(axis=0)
        out[ok] = sum(wts[i][:, None] * os_[i][ok] for i in range(len(os_))) / den[:, None]
        lse[ok] = m[ok] + np.log(den)
    return out, lse


# ---------------------------------------------------------------------------
# The pages' 2-D worked example ("LSA 稀疏注意力會省顯存嗎", §三 and §四)
# ---------------------------------------------------------------------------

WORKED_Q = np.array([1.0, 0.0])
WORKED_KEYS = np.array([[1.0, 0.0], [0.8, 0.2], [0.6, 0.4], [0.4, 0.6],       # bucket A
                        [0.0, 1.0], [-0.2, 0.8], [-0.4, 0.6], [-0.6, 0.4]])   # bucket B
WORKED_VALUES = np.array([[10.0 * (i + 1), 0.0] for i in range(8)])
WORKED_MEMBERS = np.array([[0, 1, 2, 3], [4, 5, 6, 7]])
WORKED_SCALE = 1.0 / math.sqrt(2.0)


def worked_example(q: np.ndarray, positions: np.ndarray) -> np.ndarray:
    """Single-head attention of the worked example over the given key positions."""
    o, _ = softmax_attention(np.asarray(q, dtype=np.float64)[None, :], WORKED_KEYS[positions],
                             WORKED_VALUES[positions], WORKED_SCALE)
    return o[0]
