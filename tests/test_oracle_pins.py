"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test is chosen so that a plausible slip in the oracle (a dropped ReLU, a
wrong sign, a transposed operand, a wrong tie order, a missed tail) fails one.
No test here re-types the oracle's own formula.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import lsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


def _golden():
    out = {}
    for line in open(GOLDEN, encoding="utf-8"):
        if line.startswith("#") or not line.strip():
            continue
        name, val, tol, *_ = line.split()
        out[name] = (float(val), float(tol))
    return out


# --------------------------------------------------------------------------
# Worked example ("LSA 稀疏注意力會省顯存嗎", §三 / §四)
# --------------------------------------------------------------------------


def test_worked_example_full_and_bucket_a():
    g = _golden()
    full = O.worked_example(O.WORKED_Q, np.arange(8))
    a_only = O.worked_example(O.WORKED_Q, np.arange(4))
    assert abs(full[0] - g["full_read_x"][0]) < g["full_read_x"][1]
    assert abs(a_only[0] - g["bucket_a_x"][0]) < g["bucket_a_x"][1]
    assert abs(full[1]) <= g["second_coord"][1] and abs(a_only[1]) <= g["second_coord"][1]


def test_worked_example_bytes():
    """Byte accounting of §三: what is read shrinks, what is stored does not."""
    g = _golden()
    per_entry = (2 + 2) * 2  # K and V, two numbers each, 2 B per number
    assert 8 * per_entry == g["kv_bytes_full"][0]
    assert 4 * per_entry == g["kv_bytes_bucket_a"][0]
    reps = O.pool_keys(O.WORKED_KEYS, O.WORKED_MEMBERS)
    assert reps.size * 2 + O.WORKED_MEMBERS.size * 4 == g["directory_bytes"][0]


def test_worked_example_bucket_choice():
    """Flat selection on the example: reps are the member means; q=(1,0) keeps A, q=(0,1) keeps B.

    (Derived here, not printed: the page asks the reader to try bucket B for q=(0,1).)
    """
    reps = O.pool_keys(O.WORKED_KEYS, O.WORKED_MEMBERS)
    np.testing.assert_allclose(reps, [[0.7, 0.3], [-0.3, 0.7]], atol=1e-15)
    for q, want in (([1.0, 0.0], [0, 1, 2, 3]), ([0.0, 1.0], [4, 5, 6, 7])):
        bs = O.bucket_scores(np.array(q)[None, None, :], np.ones((1, 1)), reps)
        sel, _, _ = O.bucket_select_row(bs[0], q_pos=7, M=1, sink=0, window=0, members=O.WORKED_MEMBERS)
        assert sel.tolist() == want
    # derived (not page-printed): q=(0,1), bucket B only vs full read
    assert abs(O.worked_example([0.0, 1.0], np.arange(4, 8))[0] - 63.2422) < 1e-3
    assert abs(O.worked_example([0.0, 1.0], np.arange(8))[0] - 47.5628) < 1e-3


# --------------------------------------------------------------------------
# Exact input decoding
# --------------------------------------------------------------------------


def test_bf16_decode_all_codes():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = O.bf16_to_f64(bits)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_to_f64(codes)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert O.e4m3_to_f64(np.array([0x7E], np.uint8))[0] == 448.0


# --------------------------------------------------------------------------
# a1 indexer score (LongCat page, §DSA 基线, equation I_{t,s})
# --------------------------------------------------------------------------


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_score_single_head_unit_weight_is_relu_dot():
    rng = np.random.default_rng(1)
    q = _rand(rng, 1, 1, 8)
    k = _rand(rng, 20, 8)
    got = O.index_score(q, np.ones((1, 1)), k, np.array([19]))[0]
    for s in range(20):
        d = sum(float(q[0, 0, i]) * float(k[s, i]) for i in range(8))
        assert abs(got[s] - max(0.0, d)) < 1e-12


def test_score_relu_odd_part_identity():
    """ReLU(x) - ReLU(-x) = x  =>  I(q) - I(-q) = sum_j w_j q_j . k (catches a missing ReLU or sign)."""
    rng = np.random.default_rng(2)
    B, H, d, L = 3, 5, 16, 40
    q, w, k = _rand(rng, B, H, d), rng.uniform(size=(B, H)), _rand(rng, L, d)
    qp = np.full(B, L - 1)
    diff = O.index_score(q, w, k, qp) - O.index_score(-q, w, k, qp)
    lin = np.einsum("bh,bhd,sd->bs", w, q, k)
    np.testing.assert_allclose(diff, lin, rtol=1e-12, atol=1e-11)


def test_score_invariants():
    rng = np.random.default_rng(3)
    B, H, d, L = 2, 6, 12, 33
    q, w, k = _rand(rng, B, H, d), rng.uniform(size=(B, H)), _rand(rng, L, d)
    qp = np.full(B, L - 1)
    base = O.index_score(q, w, k, qp)
    assert (base >= 0).all()
    # linear in w
    w2 = rng.uniform(size=(B, H))
    np.testing.assert_allclose(O.index_score(q, w + 2 * w2, k, qp),
                               base + 2 * O.index_score(q, w2, k, qp), rtol=1e-12)
    # positively homogeneous in q and in k (the FP8 key scale commutes with ReLU)
    np.testing.assert_allclose(O.index_score(3.5 * q, w, k, qp), 3.5 * base, rtol=1e-12)
    np.testing.assert_allclose(O.index_score(q, w, 0.25 * k, qp), 0.25 * base, rtol=1e-12)
    # invariant under permuting (q_j, w_j) pairs
    perm = rng.permutation(H)
    np.testing.assert_allclose(O.index_score(q[:, perm], w[:, perm], k, qp), base, rtol=1e-12)
    # every q_j . k <= 0  =>  I = 0
    kneg = -np.abs(k)
    assert (O.index_score(np.abs(q), w, kneg, qp) == 0).all()
    # heads of one query do not leak into another (B axis is not mixed)
    np.testing.assert_allclose(O.index_score(q[1:], w[1:], k, qp[1:]), base[1:], rtol=1e-12)


def test_score_causal_mask():
    rng = np.random.default_rng(4)
    q, w, k = _rand(rng, 3, 2, 4), rng.uniform(size=(3, 2)), _rand(rng, 10, 4)
    qp = np.array([0, 4, 9])
    s = O.index_score(q, w, k, qp)
    for b in range(3):
        assert np.isfinite(s[b, : qp[b] + 1]).all()
        assert np.isneginf(s[b, qp[b] + 1:]).all()


# --------------------------------------------------------------------------
# a2 top-K + SI union (LongCat page, §DSA 基线 arg topK; §SI 预算分解)
# --------------------------------------------------------------------------


def _brute_topk(scores, q_pos, K, sink, window):
    """Rank by counting: candidate s beats t iff score_s > score_t or (equal and s < t)."""
    fixed = set(range(0, min(sink, q_pos + 1))) | set(range(max(0, q_pos - window + 1), q_pos + 1) if window else [])
    cand = [s for s in range(q_pos + 1) if s not in fixed]
    take = []
    for s in cand:
        rank = sum(1 for t in cand if scores[t] > scores[s] or (scores[t] == scores[s] and t < s))
        if rank < K:
            take.append(s)
    return sorted(fixed | set(take))


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_small(seed):
    rng = np.random.default_rng(10 + seed)
    L = int(rng.integers(1, 65))
    # coarse values force many exact ties
    scores = rng.integers(0, 6, size=L).astype(np.float64)
    for q_pos in sorted({L - 1, int(rng.integers(0, L))}):
        for K in (1, 3, 8, 64):
            for sink, window in ((0, 0), (2, 3), (4, 0), (0, 5)):
                got, _, _ = O.topk_row(scores, q_pos, K, sink, window)
                assert got.tolist() == _brute_topk(scores, q_pos, K, sink, window)


def test_topk_set_size_identity():
    rng = np.random.default_rng(20)
    scores = rng.standard_normal(500)
    for q_pos, K, sink, window in ((499, 64, 4, 128), (10, 64, 4, 128), (300, 2048, 4, 16), (0, 5, 4, 4), (3, 2, 16, 0)):
        sel, _, ncand = O.topk_row(scores, q_pos, K, sink, window)
        s_sink, s_swa = O.fixed_positions(q_pos, sink, window)
        nfixed = len(set(s_sink.tolist()) | set(s_swa.tolist()))
        assert sel.size == min(K, ncand) + nfixed
        assert (np.diff(sel) > 0).all() and sel.min() >= 0 and sel.max() <= q_pos


def test_topk_fixed_positions_excluded_from_candidates():
    """S_sparse ranks only s outside S_sink u S_swa: huge scores there do not use up K."""
    scores = np.zeros(100)
    scores[:4] = 1e9
    scores[-10:] = 1e9
    scores[50] = 5.0
    sel, _, _ = O.topk_row(scores, 99, 1, 4, 10)
    assert 50 in sel.tolist() and sel.size == 4 + 10 + 1


def test_topk_equals_full_descending_sort():
    rng = np.random.default_rng(21)
    scores = rng.standard_normal(3000)
    sel, kth, _ = O.topk_row(scores, 2999, 100, 0, 0)
    want = sorted(sorted(range(3000), key=lambda s: -scores[s])[:100])
    assert sel.tolist() == want
    assert kth == sorted(scores)[-100]


# --------------------------------------------------------------------------
# a0 / a3 representatives, bucket and micro-block selection
# --------------------------------------------------------------------------


def test_pool_keys_microblock_means():
    k = np.arange(4 * 11 * 3, dtype=np.float64).reshape(44, 3)
    reps = O.pool_keys(k[:43], block=4)  # 43 rows -> 10 complete blocks
    assert reps.shape == (10, 3)
    for n in range(10):
        assert np.array_equal(reps[n], (k[4 * n] + k[4 * n + 1] + k[4 * n + 2] + k[4 * n + 3]) / 4)


def test_bucket_size_one_is_token_topk():
    """One position per bucket => Flat selection = token top-K (sink = window = 0)."""
    rng = np.random.default_rng(30)
    B, H, d, L = 2, 4, 8, 200
    q, w, k = _rand(rng, B, H, d), rng.uniform(size=(B, H)), _rand(rng, L, d)
    qp = np.full(B, L - 1)
    tok = O.index_score(q, w, k, qp)
    members = np.arange(L).reshape(L, 1)
    reps = O.pool_keys(k, members)
    bs = O.bucket_scores(q, w, reps)
    for b in range(B):
        s1, _, _ = O.topk_row(tok[b], L - 1, 37, 0, 0)
        s2, _, _ = O.bucket_select_row(bs[b], L - 1, 37, 0, 0, members=members)
        assert s1.tolist() == s2.tolist()
        s3, _, _ = O.bucket_select_row(bs[b], L - 1, 37, 0, 0, block=1)
        assert s1.tolist() == s3.tolist()


@pytest.mark.parametrize("tail", [0, 1, 2, 3])
def test_microblock_tail_rule(tail):
    """Visible tokens of the incomplete micro-block are read directly, whatever their scores."""
    L = 4 * 30 + tail
    bscore = np.linspace(1.0, 2.0, 30)  # block 29 scores highest, 0 lowest
    sel, _, nrank = O.bucket_select_row(bscore, L - 1, M=2, sink=0, window=0, block=4)
    assert nrank == 30
    want = list(range(4 * 28, 4 * 30)) + list(range(4 * 30, 4 * 30 + tail))
    assert sel.tolist() == want


def test_microblock_only_complete_visible_blocks_ranked():
    bscore = np.arange(10, dtype=np.float64)  # later blocks score higher
    sel, _, nrank = O.bucket_select_row(bscore, q_pos=21, M=1, sink=0, window=0, block=4)
    # q_pos = 21 -> 22 visible tokens -> 5 complete blocks (0..4), tail {20, 21}
    assert nrank == 5 and sel.tolist() == [16, 17, 18, 19, 20, 21]


def test_bucket_union_dedup_and_ties():
    members = np.array([[0, 5], [1, 6], [2, 7], [3, 8]])
    bscore = np.array([1.0, 2.0, 2.0, 0.5])  # tie between buckets 1 and 2 -> lower id wins
    sel, mth, _ = O.bucket_select_row(bscore, 8, M=1, sink=2, window=2, members=members)
    assert sel.tolist() == [0, 1, 6, 7, 8] and mth == 2.0


# --------------------------------------------------------------------------
# a4 attention
# --------------------------------------------------------------------------


def test_attention_k_equals_l_is_dense_sdpa():
    """K = L (no sink/window): the selected set is every position, so the sparse pass is dense attention."""
    rng = np.random.default_rng(40)
    H, L, dqk, dv = 4, 57, 24, 16
    q, kv = _rand(rng, H, dqk), _rand(rng, L, dqk)
    sel, _, _ = O.topk_row(rng.standard_normal(L), L - 1, L, 0, 0)
    assert sel.tolist() == list(range(L))
    o, lse = O.sparse_mla_attn(q, kv[sel], 1 / math.sqrt(dqk), dv)
    tq = torch.from_numpy(q)[None, :, None, :]
    tk = torch.from_numpy(kv)[None, None].expand(1, H, L, dqk)
    tv = torch.from_numpy(kv[:, :dv])[None, None].expand(1, H, L, dv)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=1 / math.sqrt(dqk))
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-12)
    from scipy.special import logsumexp
    np.testing.assert_allclose(lse, logsumexp(q @ kv.T / math.sqrt(dqk), axis=1), rtol=1e-12)


def test_attention_brute_force_every_subset_small():
    rng = np.random.default_rng(41)
    H, L, d = 2, 6, 5
    q, kv = _rand(rng, H, d), _rand(rng, L, d)
    for r in range(1, L + 1):
        for sub in itertools.combinations(range(L), r):
            o, lse = O.sparse_mla_attn(q, kv[list(sub)], 0.7, 3)
            for h in range(H):
                z = [0.7 * sum(q[h, i] * kv[s, i] for i in range(d)) for s in sub]
                e = [math.exp(x) for x in z]
                tot = sum(e)
                for c in range(3):
                    assert abs(o[h, c] - sum(e[i] * kv[s, c] for i, s in enumerate(sub)) / tot) < 1e-9
                assert abs(lse[h] - math.log(tot)) < 1e-9


def test_attention_constant_value_and_empty_set():
    rng = np.random.default_rng(42)
    q = _rand(rng, 3, 6)
    kv = _rand(rng, 9, 6)
    kv[:, :4] = np.array([1.5, -2.0, 0.25, 7.0])  # every value row identical
    o, _ = O.sparse_mla_attn(q, kv, 0.4, 4)
    np.testing.assert_allclose(o, np.tile([1.5, -2.0, 0.25, 7.0], (3, 1)), rtol=1e-13)
    o0, lse0 = O.sparse_mla_attn(q, kv[:0], 0.4, 4)
    assert (o0 == 0).all() and np.isneginf(lse0).all()


def test_attention_shift_invariance_of_logits():
    """Adding a constant to every logit of a head leaves softmax unchanged (max-subtraction is exact math)."""
    rng = np.random.default_rng(43)
    q, kv = _rand(rng, 2, 5), _rand(rng, 7, 5)
    o1, lse1 = O.softmax_attention(q, kv, kv[:, :3], 1.0)
    big = np.concatenate([kv, np.ones((7, 1))], axis=1)
    qb = np.concatenate([q, np.full((2, 1), 1000.0)], axis=1)
    o2, lse2 = O.softmax_attention(qb, big, kv[:, :3], 1.0)
    np.testing.assert_allclose(o1, o2, rtol=1e-10)
    np.testing.assert_allclose(lse2 - lse1, 1000.0, rtol=1e-12)


# --------------------------------------------------------------------------------------------
# HI two-stage selection (LongCat page, section on hierarchical indexing)
# --------------------------------------------------------------------------------------------


def _hi_inputs(seed, L, H=4, d=16):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(H, d)), rng.uniform(0.1, 1.0, size=H) * rng.choice([-1.0, 1.0], size=H), \
        rng.normal(size=(L, d))


@pytest.mark.parametrize("L,q_pos", [(300, 299), (300, 170), (257, 256)])
def test_hi_equals_flat_when_every_page_is_recalled(L, q_pos):
    """M * P >= L: stage one recalls every visible token, so HI is the flat token top-K."""
    q, w, k = _hi_inputs(1, L)
    sel, kth, _, recalled = O.hi_select_row(q, w, k, q_pos, P=32, Bsub=8, M=64, K=20, sink=2, window=8)
    assert np.array_equal(recalled, np.arange(q_pos + 1))
    flat = O.index_score(q[None], w[None], k, np.array([q_pos]))[0]
    want, want_kth, _ = O.topk_row(flat, q_pos, 20, 2, 8)
    assert np.array_equal(sel, want) and kth == want_kth


def test_hi_pages_of_one_subblock_are_the_microblock_ranking():
    """P == Bsub: a page is one sub-block, so stage one is the micro-block ranking (tail rule included)."""
    q, w, k = _hi_inputs(2, 203)
    q_pos = 202
    _, _, mth, recalled = O.hi_select_row(q, w, k, q_pos, P=4, Bsub=4, M=7, K=5, sink=0, window=0)
    reps = O.pool_keys(k, block=4)
    bs = O.bucket_scores(q[None], w[None], reps)[0]
    want, want_mth, _ = O.bucket_select_row(bs, q_pos, 7, 0, 0, block=4)
    assert np.array_equal(recalled, want) and mth == want_mth


def test_hi_brute_force_tiny():
    """Loops over the definition, written independently of the oracle's array code."""
    L, P, Bs, M, K, sink, window, q_pos = 50, 8, 4, 2, 5, 1, 3, 45
    q, w, k = _hi_inputs(3, L, H=3, d=5)

    def tok(s):
        return sum(w[j] * max(0.0, sum(q[j][d] * k[s][d] for d in range(5))) for j in range(3))

    def mean_key(n):
        return [sum(k[n * Bs + i][d] for i in range(Bs)) / Bs for d in range(5)]

    page_score = {}
    for p in range(q_pos // P + 1):
        tot = 0.0
        for n in range(p * P // Bs, (p + 1) * P // Bs):
            if n * Bs + Bs - 1 <= q_pos:  # entirely visible complete sub-block
                km = mean_key(n)
                tot += sum(w[j] * max(0.0, sum(q[j][d] * km[d] for d in range(5))) for j in range(3))
        page_score[p] = tot
    pages = sorted(page_score, key=lambda p: (-page_score[p], p))[:M]
    recalled = {p * P + i for p in pages for i in range(P)} | set(range((q_pos + 1) // Bs * Bs, q_pos + 1))
    recalled = sorted(s for s in recalled if s <= q_pos)
    fixed = set(range(min(sink, q_pos + 1))) | set(range(q_pos - window + 1, q_pos + 1))
    cand = [s for s in recalled if s not in fixed]
    take = sorted(cand, key=lambda s: (-tok(s), s))[:K]
    want = sorted(fixed | set(take))
    sel, _, _, rec = O.hi_select_row(q, w, k, q_pos, P, Bs, M, K, sink, window)
    assert rec.tolist() == recalled
    assert sel.tolist() == want


def test_hi_is_causal():
    """Keys after the query position change neither stage."""
    q, w, k = _hi_inputs(4, 400)
    q_pos = 233
    a = O.hi_select_row(q, w, k, q_pos, P=16, Bsub=8, M=5, K=12, sink=2, window=4)
    k2 = k.copy()
    k2[q_pos + 1:] = np.random.default_rng(9).normal(size=k2[q_pos + 1:].shape) * 10
    b = O.hi_select_row(q, w, k2, q_pos, P=16, Bsub=8, M=5, K=12, sink=2, window=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[3], b[3]) and a[2] == b[2]
    assert a[3].max() <= q_pos


# --------------------------------------------------------------------------------------------
# HFA: LSE merge of partial attentions
# --------------------------------------------------------------------------------------------


@pytest.mark.parametrize("cuts", [[5], [1, 7], [0, 3, 3, 12]])
def test_lse_merge_equals_attention_over_the_union(cuts):
    """Merging the attentions of a partition (empty parts included) is the attention over the whole set."""
    rng = np.random.default_rng(11)
    q, kv = rng.normal(size=(6, 24)), rng.normal(size=(12, 24))
    bounds = [0] + cuts + [12]
    parts = [O.softmax_attention(q, kv[a:b], kv[a:b, :10], 0.3) for a, b in zip(bounds[:-1], bounds[1:])]
    o, lse = O.lse_merge(parts)
    ref_o, ref_lse = O.softmax_attention(q, kv, kv[:, :10], 0.3)
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_lse_merge_of_empty_parts_is_empty():
    o, lse = O.lse_merge([(np.zeros((3, 4)), np.full(3, -np.inf))] * 2)
    assert np.all(o == 0) and np.all(lse == -np.inf)


# --------------------------------------------------------------------------------------------
# MSA group-wise block selection
# --------------------------------------------------------------------------------------------


def test_msa_one_group_is_block_topk_of_max_pooled_scores():
    """G = 1: the block ranking of max-pooled flat token scores, by a loop-level brute force."""
    rng = np.random.default_rng(21)
    q, w, k = rng.normal(size=(4, 8)), rng.uniform(0.1, 1, size=4), rng.normal(size=(200, 8))
    q_pos, block, KB = 171, 16, 3
    (pos, kth), = O.msa_select_row(q, w, k, q_pos, G=1, block=block, KB=KB)

    def tok(s):
        return sum(w[j] * max(0.0, float(q[j] @ k[s])) for j in range(4))

    lb = q_pos // block
    bs = {c: max(tok(s) for s in range(c * block, c * block + block)) for c in range(lb)}
    keep = sorted(bs, key=lambda c: (-bs[c], c))[:KB]
    want = sorted({c * block + i for c in keep for i in range(block)} | set(range(lb * block, q_pos + 1)))
    assert pos.tolist() == want and kth == pytest.approx(bs[keep[-1]], rel=1e-12)


def test_msa_groups_use_their_own_index_heads():
    """Group g's selection depends only on index heads of group g (the others are scrambled freely)."""
    rng = np.random.default_rng(22)
    q, w, k = rng.normal(size=(8, 8)), rng.uniform(0.1, 1, size=8), rng.normal(size=(300, 8))
    a = O.msa_select_row(q, w, k, 299, G=4, block=16, KB=4)
    q2, w2 = q.copy(), w.copy()
    q2[2:], w2[2:] = rng.normal(size=(6, 8)), rng.uniform(0.1, 1, size=6)  # heads of groups 1..3 only
    b = O.msa_select_row(q2, w2, k, 299, G=4, block=16, KB=4)
    assert np.array_equal(a[0][0], b[0][0]) and a[0][1] == b[0][1]
    single = O.msa_select_row(q[0:2], w[0:2], k, 299, G=1, block=16, KB=4)[0]
    assert np.array_equal(a[0][0], single[0])


def test_msa_local_block_only_near_the_start():
    """No complete block before the query: only the local block's visible tokens."""
    rng = np.random.default_rng(23)
    q, w, k = rng.normal(size=(2, 4)), rng.uniform(size=2), rng.normal(size=(40, 4))
    (pos, kth), = O.msa_select_row(q, w, k, 9, G=1, block=16, KB=2)
    assert pos.tolist() == list(range(10)) and kth == -np.inf


def test_msa_block_ties_go_to_the_lower_block_and_max_not_sum():
    """One head, w = 1, q = (1,), blocks of 2: a token's score is max(0, k), a block's the max of its tokens'.

    Tokens 0..7 hold k = (3, 0 | 1, 1 | 3, -5 | 0, 0), blocks 0..3 score 3, 1, 3, 0; the query sits at 9 (local
    block 4).  KB = 1 keeps block 0 (tied with block 2: the lower block wins); KB = 2 keeps blocks 0 and 2.  With
    block 1 raised to (2, 2) its max (2) is still below 3 while its ReLU sum (4) would beat blocks 0 and 2 (3
    each): the max, not a sum, decides."""
    q, w = np.array([[1.0]]), np.array([1.0])
    k = np.array([[3.0], [0.0], [1.0], [1.0], [3.0], [-5.0], [0.0], [0.0], [2.0], [7.0]])
    (pos1, kth1), = O.msa_select_row(q, w, k, 9, G=1, block=2, KB=1)
    assert pos1.tolist() == [0, 1, 8, 9] and kth1 == 3.0
    (pos2, kth2), = O.msa_select_row(q, w, k, 9, G=1, block=2, KB=2)
    assert pos2.tolist() == [0, 1, 4, 5, 8, 9] and kth2 == 3.0
    k2 = k.copy()
    k2[2:4] = 2.0
    (pos3, _), = O.msa_select_row(q, w, k2, 9, G=1, block=2, KB=2)
    assert pos3.tolist() == [0, 1, 4, 5, 8, 9]


# --------------------------------------------------------------------------
# D-LSA Tree: two-level search
# --------------------------------------------------------------------------


def test_tree_parents_are_child_means_with_ragged_last():
    """Parent p = mean of buckets [pF, min((p+1)F, NB)): NB = 5, F = 2 -> means of (0,1), (2,3) and (4) alone."""
    reps = np.array([[1.0, 0.0], [3.0, 2.0], [5.0, -1.0], [7.0, 1.0], [-4.0, 9.0]])
    par = O.tree_parents(reps, 2)
    assert par.tolist() == [[2.0, 1.0], [6.0, 0.0], [-4.0, 9.0]]


def _tree_case(seed=3, NB=37, bsz=5, d=8, H=3):
    rng = np.random.default_rng(seed)
    L = NB * bsz
    members = rng.permutation(L).reshape(NB, bsz)
    reps = rng.standard_normal((NB, d))
    q = rng.standard_normal((H, d))
    w = rng.uniform(0.0, 1.0, H)
    return L, members, reps, q, w


def test_tree_full_beam_is_flat():
    """Keeping every parent makes every bucket a candidate: the search is the Flat search."""
    L, members, reps, q, w = _tree_case()
    flat_scores = O.bucket_scores(q[None], w[None], reps)[0]
    for F in (1, 4, 6, 37):
        NP = -(-37 // F)
        for M in (1, 5, 11):
            sel, mth, _ = O.tree_select_row(q, w, reps, members, F, NP, M, L - 1, 2, 3)
            want, want_mth, _ = O.bucket_select_row(flat_scores, L - 1, M, 2, 3, members=members)
            assert np.array_equal(sel, want) and mth == want_mth, (F, M)


def test_tree_one_child_per_parent_is_flat():
    """F = 1: the parents are the buckets, the M2 >= M best of them hold the M best buckets."""
    L, members, reps, q, w = _tree_case(seed=5)
    flat_scores = O.bucket_scores(q[None], w[None], reps)[0]
    for M, M2 in ((3, 3), (3, 10), (7, 8)):
        sel, _, _ = O.tree_select_row(q, w, reps, members, 1, M2, M, L - 1, 0, 0)
        want, _, _ = O.bucket_select_row(flat_scores, L - 1, M, 0, 0, members=members)
        assert np.array_equal(sel, want), (M, M2)


def test_tree_parent_mean_hides_best_child():
    """A bucket whose centre is average can hide a strong member (the LSA page warns of exactly this); here a
    parent's mean hides its best child, so the narrow beam misses what Flat keeps.

    q = (1, 0), one head, w = 1.  Buckets 0, 1 (parent 0): centres (10, 0), (-10, 0) -> parent (0, 0), score 0.
    Buckets 2, 3 (parent 1): centres (1, 0), (2, 0) -> parent (1.5, 0), score 1.5.  M2 = 1 keeps parent 1; of its
    children bucket 3 (score 2) beats bucket 2 (score 1).  Flat keeps bucket 0 (score 10)."""
    reps = np.array([[10.0, 0.0], [-10.0, 0.0], [1.0, 0.0], [2.0, 0.0]])
    members = np.array([[0, 1], [2, 3], [4, 5], [6, 7]])
    q, w = np.array([[1.0, 0.0]]), np.array([1.0])
    sel, mth, m2th = O.tree_select_row(q, w, reps, members, 2, 1, 1, 7, 0, 0)
    assert sel.tolist() == [6, 7] and mth == 2.0 and m2th == 1.5
    sel2, _, _ = O.tree_select_row(q, w, reps, members, 2, 2, 1, 7, 0, 0)
    assert sel2.tolist() == [0, 1]
    # ties at level 1 go to the lower bucket id: equal children under the kept parent
    reps_t = np.array([[10.0, 0.0], [-10.0, 0.0], [2.0, 0.0], [2.0, 0.0]])
    sel3, _, _ = O.tree_select_row(q, w, reps_t, members, 2, 1, 1, 7, 0, 0)
    assert sel3.tolist() == [4, 5]


def test_tree_union_clip_and_short_candidate_list():
    """Fewer candidates than M: all are kept; members past q_pos are dropped; sink and window join."""
    reps = np.array([[1.0], [2.0], [3.0], [4.0], [5.0]])
    members = np.array([[0, 9], [1, 8], [2, 7], [3, 6], [4, 5]])
    q, w = np.array([[1.0]]), np.array([1.0])
    # F = 2: parents (1.5), (3.5), (5); M2 = 1 keeps parent 2 (bucket 4 alone); M = 3 > 1 candidate
    sel, mth, m2th = O.tree_select_row(q, w, reps, members, 2, 1, 3, 6, 1, 2)
    assert m2th == 5.0 and mth == 5.0
    assert sel.tolist() == [0, 4, 5, 6]
