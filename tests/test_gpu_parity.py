"""GPU parity of every call of the C ABI against the fp64 oracle (small and mid-size cases).

Sizes span several tiles and ragged tails while the oracle still finishes in seconds.  Full-size
workloads are in test_gpu_configs.py.
"""

import math

import numpy as np
import pytest
import torch

import lsa_synth as S
import sparse_long_context_lightning_b200 as lsa
from oracle import lsa_oracle as O

from gpu_common import (ATTN_REL, Decode, attn_rel_err, check_index_sets, f64, run_oracle_attention)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _scores_close(got: torch.Tensor, ref: np.ndarray, q_pos: np.ndarray):
    g = got.double().cpu().numpy()
    L = ref.shape[1]
    for b in range(ref.shape[0]):
        vis = np.arange(L) <= q_pos[b]
        assert np.isneginf(g[b, ~vis]).all()
        r = ref[b, vis]
        err = np.abs(g[b, vis] - r)
        # fp32 accumulation of exact products: error well under 1e-5 of the row's score scale
        assert err.max() <= 1e-5 * max(np.abs(r).max(), 1e-30), (b, err.max(), np.abs(r).max())


# --------------------------------------------------------------------------------------------
# a1 indexer
# --------------------------------------------------------------------------------------------


@pytest.mark.parametrize("name,fp8", [("tiny", False), ("decode128k", False), ("decode128k", True)])
def test_index_score_decode(name, fp8):
    d = Decode(S.WORKLOADS[name], fp8=fp8)
    L = d.wl.L
    scores = torch.empty(d.B, L, device=DEV)
    if fp8:
        lsa.lsa_index_score(d.q8, d.w, d.k8, d.q_pos, scores, q_scale=d.q_scale, k_scale=d.k_scale)
    else:
        lsa.lsa_index_score(d.q_I, d.w, d.k_I, d.q_pos, scores)
    torch.cuda.synchronize()
    _scores_close(scores, d.oracle_scores(), d.q_pos.cpu().numpy())


@pytest.mark.parametrize("fp8", [False, True])
def test_index_score_causal_ragged(fp8):
    """Causal rows over a ragged L: masked tails, partially visible tiles, odd B."""
    wl = S.Workload("causal", L=8192 + 77, B=37, H_I=64, d_I=128, K=64, H=16, causal_start=3000)
    qp = torch.tensor([3000 + 137 * b for b in range(37)], dtype=torch.int64)
    qp[0], qp[1], qp[2] = 0, 1, 8192 + 76
    d = Decode(wl, fp8=fp8, q_pos=qp)
    sc = torch.full((d.B, wl.L + 7), 7.0, device=DEV)  # ld = L + 7 (a multiple of 4)
    if fp8:
        lsa.lsa_index_score(d.q8, d.w, d.k8, d.q_pos, sc, q_scale=d.q_scale, k_scale=d.k_scale)
    else:
        lsa.lsa_index_score(d.q_I, d.w, d.k_I, d.q_pos, sc)
    torch.cuda.synchronize()
    _scores_close(sc[:, : wl.L], d.oracle_scores(), qp.numpy())
    assert (sc[:, wl.L:] == 7.0).all(), "entries past L must not be touched"


@pytest.mark.parametrize("H_I,d_I", [(4, 32), (16, 64), (64, 128), (1, 128)])
def test_index_score_shapes(H_I, d_I):
    wl = S.Workload("shape", L=5000, B=5, H_I=H_I, d_I=d_I, K=16, H=16)
    d = Decode(wl)
    scores = torch.empty(d.B, 5000, device=DEV)
    lsa.lsa_index_score(d.q_I, d.w, d.k_I, d.q_pos, scores)
    torch.cuda.synchronize()
    _scores_close(scores, d.oracle_scores(), d.q_pos.cpu().numpy())


# --------------------------------------------------------------------------------------------
# a2 top-K + sink / window union, on given fp32 scores (exact, including tie order)
# --------------------------------------------------------------------------------------------


def _topk_case(scores_np, q_pos, K, sink, window):
    B, L = scores_np.shape
    ld = (L + 3) // 4 * 4
    sc = torch.full((B, ld), float("nan"), device=DEV)
    sc[:, :L] = torch.from_numpy(scores_np.astype(np.float32)).to(DEV)
    kmax = K + sink + window
    idx = torch.full((B, kmax + 5), 12345, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    qp = torch.as_tensor(q_pos, dtype=torch.int64).to(DEV)
    lsa.lsa_topk_select(sc, L, K, sink, window, qp, idx, cnt)
    torch.cuda.synchronize()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    s32 = scores_np.astype(np.float32).astype(np.float64)
    for b in range(B):
        want, _, _ = O.topk_row(s32[b], int(q_pos[b]), K, sink, window)
        got = idx_h[b, : cnt_h[b]]
        assert cnt_h[b] == want.size, (b, cnt_h[b], want.size)
        assert np.array_equal(got, want), (b, np.setxor1d(got, want)[:10])
        assert np.all(idx_h[b, cnt_h[b]: kmax] == -1)
        assert np.all(idx_h[b, kmax:] == 12345), "wrote past K+sink+window"


@pytest.mark.parametrize("L", [1, 7, 100, 4096, 4099, 65537, 131072, 200003])
@pytest.mark.parametrize("K,sink,window", [(1, 0, 0), (16, 4, 0), (256, 0, 128), (2048, 4, 128)])
def test_topk_exact_random(L, K, sink, window):
    rng = np.random.default_rng(L * 7 + K)
    B = 3
    scores = rng.standard_normal((B, L)) * 50 + 100
    q_pos = [L - 1, int(rng.integers(0, L)), min(L - 1, K + sink + window + 3)]
    _topk_case(scores, q_pos, K, sink, window)


@pytest.mark.parametrize("L", [333, 4096, 131072])
def test_topk_exact_heavy_ties(L):
    rng = np.random.default_rng(L)
    B = 4
    scores = np.empty((B, L))
    scores[0] = rng.integers(0, 5, L)                 # few distinct values
    scores[1] = 3.0                                   # all equal
    scores[2] = np.where(rng.uniform(size=L) < 0.5, 0.0, rng.uniform(size=L))  # many exact zeros
    scores[3] = rng.standard_normal(L)
    scores[3, rng.integers(0, L, 50)] = np.inf        # +inf entries outrank everything
    for K, sink, window in ((1, 0, 0), (37, 2, 5), (min(L // 2, 2048), 4, 128)):
        _topk_case(scores, [L - 1] * B, K, sink, window)


@pytest.mark.parametrize("L", [131072, 200003, 600000])
@pytest.mark.parametrize("K", [64, 2048])
def test_topk_exact_stride_blind_spots(L, K):
    """Rows whose values at a regular stride (L / 1024 apart, the spacing of a fixed sample of the row) look nothing
    like the rest: the largest scores all off that stride; that stride holding a single value; holding only -inf;
    holding the largest values.  The kernel's level-0 bins come from such a sample, so its selection must not
    depend on the sample being representative."""
    rng = np.random.default_rng(L + K)
    on = (np.arange(1024, dtype=np.int64) * L) // 1024  # the stride positions
    off = np.setdiff1d(np.arange(L), on)
    scores = np.empty((4, L))
    scores[0] = rng.standard_normal(L)
    top = rng.choice(off, K + 100, replace=False)
    scores[0, top] = 10.0 ** rng.uniform(3, 6, top.size)  # the top K and more, none on the stride
    scores[1] = rng.standard_normal(L) * 30
    scores[1, on] = 5.0
    scores[2] = rng.standard_normal(L)
    scores[2, on] = -np.inf
    scores[3] = rng.standard_normal(L)
    scores[3, on] = 1e4 + rng.standard_normal(on.size)
    _topk_case(scores, [L - 1] * 4, K, 0, 0)


@pytest.mark.parametrize("K", [300, 2048])
def test_topk_exact_clustered_top(K):
    """The largest scores packed into contiguous runs (one run of K, runs of 70 every 5000 positions, runs of 60):
    a stretch of the row then holds more selected keys than a warp's list of them can hold, and the write must
    fall back to walking the chunk; the run lengths straddle that list size."""
    L = 131072
    rng = np.random.default_rng(K)
    scores = rng.standard_normal((4, L))
    scores[0, 1000:1000 + K] = 100.0 + rng.standard_normal(K)
    for start in range(7, L - 70, 5000):
        scores[1, start:start + 70] = 50.0 + rng.standard_normal(70)
        scores[2, start:start + 60] = 50.0 + rng.standard_normal(60)
    scores[3] = np.repeat(rng.standard_normal(L // 512), 512)  # runs of 512 equal values
    _topk_case(scores, [L - 1] * 4, K, 4, 128)


def test_topk_many_rows_prefill_like():
    rng = np.random.default_rng(5)
    B, L = 300, 20000
    scores = rng.standard_normal((B, L)).astype(np.float32)
    q_pos = sorted(rng.integers(0, L, B).tolist())
    q_pos[0] = 0
    _topk_case(scores, q_pos, 2048, 4, 128)


# --------------------------------------------------------------------------------------------
# a0 representatives
# --------------------------------------------------------------------------------------------


@pytest.mark.parametrize("fp8", [False, True])
def test_pool_keys(fp8):
    L, d_I = 40003, 128
    k = S.normal_bf16(S.ST_KI, (L, d_I), DEV)
    members = S.permutation(S.ST_BUCKET, L, "cpu")[: (L // 64) * 64].view(-1, 64).to(torch.int32)
    if fp8:
        k8, ks = S.quantize_e4m3_rows(k)
        kin, kscale = k8, ks
        kf = f64(ks)[:, None] * O.e4m3_to_f64(k8.cpu().numpy())
    else:
        kin, kscale = k, None
        kf = f64(k)
    cen = torch.empty(members.shape[0], d_I, device=DEV)
    lsa.lsa_pool_keys(kin, cen, 64, members=members.to(DEV), k_scale=kscale)
    blk = torch.empty(L // 4, d_I, device=DEV)
    lsa.lsa_pool_keys(kin, blk, 4, k_scale=kscale)
    torch.cuda.synchronize()
    ref = O.pool_keys(kf, members.numpy())
    np.testing.assert_allclose(f64(cen), ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())
    refb = O.pool_keys(kf, block=4)
    np.testing.assert_allclose(f64(blk), refb, rtol=1e-6, atol=1e-7)


# --------------------------------------------------------------------------------------------
# a3 bucket / micro-block selection
# --------------------------------------------------------------------------------------------


def _bucket_case(L, B, M, bsz, sink, window, flat, tie_check=True, path="full"):
    """path: "full" workspace (tensor-core scoring of the split representatives where the shape allows),
    "min" workspace (CUDA-core scoring), or "split" (lsa_bucket_select_split from a cached split)."""
    wl = S.Workload("bk", L=L, B=B, H_I=64, d_I=128, K=M * bsz, H=16, sink=sink, window=window,
                    mode="flat" if flat else "microblock", bsz=bsz, M=M)
    q_I, w = S.index_queries(wl)
    k = S.normal_bf16(S.ST_KI, (L, 128), DEV)
    if flat:
        members = S.bucket_members(wl).to(DEV)
        nb = members.shape[0]
    else:
        members = None
        nb = L // bsz
    cen = torch.empty(nb, 128, device=DEV)
    lsa.lsa_pool_keys(k, cen, bsz, members=members)
    qp = torch.full((B,), L - 1, dtype=torch.int64)
    if not flat:
        qp[1:] = torch.tensor([L - 1 - 5 * i for i in range(1, B)])
    kmax = M * bsz + (bsz - 1) + sink + window
    idx = torch.full((B, kmax), 777, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    if path == "split":
        split = torch.empty(3, nb, 128, dtype=torch.bfloat16, device=DEV)
        lsa.lsa_split_representatives(cen, split)
        ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_BUCKET_MIN, B, nb, M))
        lsa.lsa_bucket_select_split(q_I.to(DEV), w.to(DEV), split, members, bsz, M, sink, window, L, qp.to(DEV), idx,
                                    cnt, ws)
    else:
        op = lsa.LSA_OP_BUCKET if path == "full" else lsa.LSA_OP_BUCKET_MIN
        ws = lsa.workspace(lsa.lsa_workspace_size(op, B, nb, M))
        lsa.lsa_bucket_select(q_I.to(DEV), w.to(DEV), cen, members, bsz, M, sink, window, L, qp.to(DEV), idx, cnt, ws)
    torch.cuda.synchronize()
    kf = f64(k)
    mem_np = members.cpu().numpy() if flat else None
    reps = O.pool_keys(kf, mem_np) if flat else O.pool_keys(kf, block=bsz)
    bs = O.bucket_scores(f64(q_I), f64(w), reps)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    ties = 0
    for b in range(B):
        want, mth, _ = O.bucket_select_row(bs[b], int(qp[b]), M, sink, window, members=mem_np,
                                           block=None if flat else bsz)
        got = idx_h[b, : cnt_h[b]]
        assert np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        if not np.array_equal(got, want):
            diff = np.setxor1d(got, want)
            owner = {}
            if flat:
                for c, row in enumerate(mem_np):
                    for s in row:
                        owner[int(s)] = c
            for s in diff.tolist():
                c = owner[s] if flat else s // bsz
                assert tie_check and abs(bs[b, c] - mth) <= 1e-5 * abs(mth), (b, s, bs[b, c], mth)
            ties += diff.size
    return ties


@pytest.mark.parametrize("tail", [0, 1, 2, 3])
def test_microblock_select(tail):
    _bucket_case(L=4 * 16384 + tail, B=4, M=512, bsz=4, sink=4, window=128, flat=False)


@pytest.mark.parametrize("path", ["full", "min", "split"])
def test_flat_bucket_select(path):
    _bucket_case(L=64 * 10000, B=8, M=32, bsz=64, sink=4, window=512, flat=True, path=path)


@pytest.mark.parametrize("path", ["min", "split"])
def test_microblock_select_paths(path):
    _bucket_case(L=4 * 16384 + 3, B=4, M=512, bsz=4, sink=4, window=128, flat=False, path=path)


def _tree_run(L, B, bsz, F, M2, M, sink, window, q_pos=None, split=False):
    """lsa_tree_select (split: lsa_tree_select_split, children on the tensor cores from the centres' cached bf16
    split) against the oracle's two-level search on the fp64 pooled keys.  Returns the GPU rows."""
    wl = S.Workload("tr", L=L, B=B, H_I=64, d_I=128, K=M * bsz, H=16, sink=sink, window=window, mode="flat",
                    bsz=bsz, M=M)
    q_I, w = S.index_queries(wl)
    k = S.normal_bf16(S.ST_KI, (L, 128), DEV)
    members = S.bucket_members(wl).to(DEV)
    nb = members.shape[0]
    cen = torch.empty(nb, 128, device=DEV)
    lsa.lsa_pool_keys(k, cen, bsz, members=members)
    NP = -(-nb // F)
    par = torch.empty(NP, 128, device=DEV)
    lsa.lsa_tree_parents(cen, F, par)
    qp = torch.full((B,), L - 1, dtype=torch.int64) if q_pos is None else torch.as_tensor(q_pos, dtype=torch.int64)
    kmax = M * bsz + sink + window
    idx = torch.full((B, kmax), 777, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_tree_workspace_size(B, NP, F, M2, M))
    if split:
        sp = torch.empty(3, nb, 128, dtype=torch.bfloat16, device=DEV)
        lsa.lsa_split_representatives(cen, sp)
        lsa.lsa_tree_select_split(q_I.to(DEV), w.to(DEV), sp, par, F, members, M2, M, sink, window, L, qp.to(DEV),
                                  idx, cnt, ws)
    else:
        lsa.lsa_tree_select(q_I.to(DEV), w.to(DEV), cen, par, F, members, M2, M, sink, window, L, qp.to(DEV), idx,
                            cnt, ws)
    torch.cuda.synchronize()
    lsa.lsa_device_status()
    # the parents themselves: fp32 means of the fp32 centres
    np.testing.assert_allclose(f64(par), O.tree_parents(f64(cen), F), rtol=1e-5, atol=1e-5)
    mem_np = members.cpu().numpy()
    reps = O.pool_keys(f64(k), mem_np)
    parents = O.tree_parents(reps, F)
    qf, wf = f64(q_I), f64(w)
    bs = O.bucket_scores(qf, wf, reps)
    ps = O.bucket_scores(qf, wf, parents)
    owner = np.empty(L, np.int64)
    owner[mem_np.reshape(-1)] = np.repeat(np.arange(nb), bsz)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        want, mth, m2th = O.tree_select_row(qf[b], wf[b], reps, mem_np, F, M2, M, int(qp[b]), sink, window)
        got = idx_h[b, : cnt_h[b]]
        assert np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        if np.array_equal(got, want):
            continue
        # only where a bucket ties the M-th candidate, or its parent ties the M2-th parent, within fp32 rounding
        for c in np.unique(owner[np.setxor1d(got, want)]):
            near_child = abs(bs[b, c] - mth) <= 1e-5 * abs(mth)
            near_parent = abs(ps[b, c // F] - m2th) <= 1e-5 * abs(m2th)
            assert near_child or near_parent, (b, c, bs[b, c], mth, ps[b, c // F], m2th)
    return idx_h, cnt_h


@pytest.mark.parametrize("F,M2,M", [(64, 16, 32), (10, 1000, 32), (1, 40, 32), (100, 1, 100)])
def test_tree_select(F, M2, M):
    """Two-level search over 10000 Flat buckets of 64 (ragged last parent for F = 64; F = 10 with M2 = NP is
    the full beam; F = 1 ranks the buckets themselves; F = 100, M2 = 1 has exactly M candidates)."""
    L, B = 64 * 10000, 6
    _tree_run(L, B, 64, F, M2, M, 4, 512, q_pos=[L - 1, L - 1, L // 2, 70000, L - 1, 4000])


@pytest.mark.parametrize("M2,M", [(16, 32), (7, 20), (156, 32)])
def test_tree_select_split(M2, M):
    """Children on the tensor cores (F = 64): 10000 buckets (a ragged last parent of 16), an odd number of kept
    parents (the last pair half empty) and a full beam over all 157 parents but one."""
    L, B = 64 * 10000, 6
    _tree_run(L, B, 64, 64, M2, M, 4, 512, q_pos=[L - 1, L - 1, L // 2, 70000, L - 1, 4000], split=True)


def test_tree_split_matches_gather_path():
    """The tensor-core children scores equal the CUDA-core ones up to fp32 summation order: same rows, except ties."""
    L, B = 64 * 6000 + 64 * 3, 4
    a_idx, a_cnt = _tree_run(L, B, 64, 64, 24, 32, 4, 128)
    b_idx, b_cnt = _tree_run(L, B, 64, 64, 24, 32, 4, 128, split=True)
    for b in range(B):
        d = np.setxor1d(a_idx[b, : a_cnt[b]], b_idx[b, : b_cnt[b]])
        assert d.size <= 2 * 64, (b, d.size)  # at most one tied bucket swapped


def test_tree_full_beam_matches_flat():
    """M2 >= NP: the tree search keeps what lsa_bucket_select (CUDA-core scoring) keeps."""
    L, B, bsz, M = 64 * 4000, 4, 64, 16
    idx_t, cnt_t = _tree_run(L, B, bsz, 16, 250, M, 4, 128)
    wl = S.Workload("tr", L=L, B=B, H_I=64, d_I=128, K=M * bsz, H=16, sink=4, window=128, mode="flat", bsz=bsz, M=M)
    q_I, w = S.index_queries(wl)
    k = S.normal_bf16(S.ST_KI, (L, 128), DEV)
    members = S.bucket_members(wl).to(DEV)
    cen = torch.empty(members.shape[0], 128, device=DEV)
    lsa.lsa_pool_keys(k, cen, bsz, members=members)
    idx = torch.full((B, M * bsz + 4 + 128), 777, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_BUCKET_MIN, B, members.shape[0], M))
    qp = torch.full((B,), L - 1, dtype=torch.int64, device=DEV)
    lsa.lsa_bucket_select(q_I.to(DEV), w.to(DEV), cen, members, bsz, M, 4, 128, L, qp, idx, cnt, ws)
    torch.cuda.synchronize()
    assert np.array_equal(cnt.cpu().numpy(), cnt_t)
    assert np.array_equal(idx.cpu().numpy(), idx_t)


def test_split_representatives_exact():
    """The three bf16 parts sum exactly (in fp64) to the fp32 representative, across magnitudes and signs."""
    g = torch.Generator().manual_seed(5)
    mant = torch.rand(4096, 128, generator=g) * 2 - 1
    expo = torch.randint(-40, 40, (4096, 128), generator=g).float()
    cen = (mant * torch.pow(2.0, expo)).float()
    # up to the largest bf16 (about 3.39e38); fp32 values beyond it overflow the first part
    cen[0, :8] = torch.tensor([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1.17549435e-38, 2.0 ** -100])
    cen_d = cen.to(DEV)
    split = torch.empty(3, 4096, 128, dtype=torch.bfloat16, device=DEV)
    lsa.lsa_split_representatives(cen_d, split)
    parts = split.float().double().cpu()
    assert torch.equal(parts.sum(0), cen.double())
    # each part is the bf16 rounding of what the earlier parts leave
    assert torch.equal(split[0].float().cpu(), cen.bfloat16().float())


def test_microblock_small_rows():
    """M larger than the number of complete visible blocks: every block is kept."""
    _bucket_case(L=4 * 100 + 3, B=3, M=512, bsz=4, sink=4, window=16, flat=False)


# --------------------------------------------------------------------------------------------
# a4 sparse attention on given index sets
# --------------------------------------------------------------------------------------------


@pytest.mark.parametrize("H", [16, 128])
def test_sparse_attn_ragged_counts(H):
    L = 20000
    B = 7
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, H, 576), DEV)
    counts = [0, 1, 17, 64, 2048, 2180, 999]
    kmax = 2180 + 3
    rng = np.random.default_rng(H)
    idx = torch.full((B, kmax), -1, dtype=torch.int32)
    for b, c in enumerate(counts):
        idx[b, :c] = torch.from_numpy(np.sort(rng.choice(L, size=c, replace=False)).astype(np.int32))
    idx, cnt = idx.to(DEV), torch.tensor(counts, dtype=torch.int32, device=DEV)
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, L, kmax, H))
    scale = 1 / math.sqrt(576)
    lsa.lsa_sparse_attn(q, kv, idx, cnt, scale, out, lse, ws)
    torch.cuda.synchronize()
    for b, c in enumerate(counts):
        sel = idx[b, :c].cpu().numpy()
        ref, ref_lse = run_oracle_attention(q[b], kv, sel, scale)
        if c == 0:
            assert (out[b] == 0).all() and torch.isneginf(lse[b]).all()
            continue
        assert attn_rel_err(out[b], ref) <= ATTN_REL
        assert np.abs(f64(lse[b]) - ref_lse).max() <= 1e-3


# --------------------------------------------------------------------------------------------
# the whole path: tiny workload, and the decode batch at L = 128K
# --------------------------------------------------------------------------------------------


def _pipeline(name, fp8=False):
    wl = S.WORKLOADS[name]
    d = Decode(wl, fp8=fp8)
    L, B = wl.L, d.B
    scores = torch.empty(B, L, device=DEV)
    if fp8:
        lsa.lsa_index_score(d.q8, d.w, d.k8, d.q_pos, scores, q_scale=d.q_scale, k_scale=d.k_scale)
    else:
        lsa.lsa_index_score(d.q_I, d.w, d.k_I, d.q_pos, scores)
    kmax = wl.K + wl.sink + wl.window
    idx = torch.empty(B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_select(scores, L, wl.K, wl.sink, wl.window, d.q_pos, idx, cnt)
    q = S.attn_queries(wl, DEV)[:B]
    kv = S.latent_cache(wl, DEV)
    out = torch.empty(B, wl.H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, wl.H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, L, kmax, wl.H))
    lsa.lsa_sparse_attn(q, kv, idx, cnt, wl.scale, out, lse, ws)
    torch.cuda.synchronize()
    return d, idx.cpu().numpy(), cnt.cpu().numpy(), q, kv, out, lse


@pytest.mark.parametrize("name", ["tiny", "decode128k"])
def test_pipeline_bf16(name):
    d, idx, cnt, q, kv, out, lse = _pipeline(name)
    wl = d.wl
    ref_scores = d.oracle_scores()
    ties = 0
    for b in range(d.B):
        want, kth, _ = O.topk_row(ref_scores[b], int(d.q_pos[b]), wl.K, wl.sink, wl.window)
        ties += check_index_sets(idx[b], int(cnt[b]), want, ref_scores[b], kth, wl.K + wl.sink + wl.window)
        ref, ref_lse = run_oracle_attention(q[b], kv, idx[b, : cnt[b]], wl.scale)
        assert attn_rel_err(out[b], ref) <= ATTN_REL
        assert np.abs(f64(lse[b]) - ref_lse).max() <= 1e-3
    print(f"{name}: tie positions differing = {ties}")


def test_pipeline_fp8_recall():
    """FP8 index scan + exact bf16 re-rank of the top-2K: recall of the bf16 oracle's top-K >= 0.99 (mean).

    Also checks that the FP8 scan alone is exact for its own inputs: its top-2K equals the oracle's
    ranking on the e4m3-decoded values up to ties.
    """
    wl = S.WORKLOADS["decode128k"]
    d = Decode(wl, fp8=True)
    L, B = wl.L, d.B
    scores = torch.empty(B, L, device=DEV)
    lsa.lsa_index_score(d.q8, d.w, d.k8, d.q_pos, scores, q_scale=d.q_scale, k_scale=d.k_scale)
    K2 = 2 * wl.K
    cand = torch.empty(B, K2 + wl.sink + wl.window, dtype=torch.int32, device=DEV)
    ccnt = torch.empty(B, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_select(scores, L, K2, wl.sink, wl.window, d.q_pos, cand, ccnt)
    kmax = wl.K + wl.sink + wl.window
    idx = torch.empty(B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_REFINE, B, cand.shape[1], wl.K))
    lsa.lsa_topk_refine(d.q_I, d.w, d.k_I, cand, ccnt, wl.K, wl.sink, wl.window, d.q_pos, idx, cnt, ws)
    torch.cuda.synchronize()
    ref_fp8 = d.oracle_scores()          # oracle on the e4m3-decoded inputs
    ref_bf16 = d.oracle_scores_bf16()    # oracle on the bf16 inputs
    cand_h, ccnt_h = cand.cpu().numpy(), ccnt.cpu().numpy()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    rec, raw = [], []
    for b in range(B):
        want8, kth8, _ = O.topk_row(ref_fp8[b], int(d.q_pos[b]), K2, wl.sink, wl.window)
        check_index_sets(cand_h[b], int(ccnt_h[b]), want8, ref_fp8[b], kth8, cand.shape[1])
        want, kth, _ = O.topk_row(ref_bf16[b], int(d.q_pos[b]), wl.K, wl.sink, wl.window)
        got = idx_h[b, : cnt_h[b]]
        assert cnt_h[b] == want.size and np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        # recall on the dynamic part (sink and window, always kept, left out; none in this workload)
        fixed = np.union1d(*O.fixed_positions(int(d.q_pos[b]), wl.sink, wl.window))
        wd = np.setdiff1d(want, fixed)
        rec.append(np.intersect1d(np.setdiff1d(got, fixed), wd).size / max(wd.size, 1))
        w1, _, _ = O.topk_row(ref_fp8[b], int(d.q_pos[b]), wl.K, wl.sink, wl.window)
        raw.append(np.intersect1d(np.setdiff1d(w1, fixed), wd).size / max(wd.size, 1))
    print(f"fp8 scan + bf16 re-rank dynamic recall mean {np.mean(rec):.4f} min {np.min(rec):.4f}; "
          f"fp8 scan alone (top-K) recall mean {np.mean(raw):.4f}")
    assert np.mean(rec) >= 0.99


def test_topk_refine_exact_on_given_candidates():
    """Re-rank equals the bf16 oracle's top-K restricted to the candidate set (up to ties)."""
    wl = S.Workload("rf", L=50000, B=6, H_I=64, d_I=128, K=300, H=16, sink=4, window=64)
    d = Decode(wl)
    rng = np.random.default_rng(9)
    K2 = 700
    qp = d.q_pos.cpu().numpy()
    cand = torch.full((wl.B, K2 + 4 + 64), -1, dtype=torch.int32)
    counts = []
    for b in range(wl.B):
        nd = [K2, 10, 0, 299, 300, K2][b]
        dyn = np.sort(rng.choice(np.arange(4, int(qp[b]) - 63), size=nd, replace=False))
        row = np.concatenate([np.arange(4), dyn, np.arange(int(qp[b]) - 63, int(qp[b]) + 1)])
        cand[b, : row.size] = torch.from_numpy(row.astype(np.int32))
        counts.append(row.size)
    cand, ccnt = cand.to(DEV), torch.tensor(counts, dtype=torch.int32, device=DEV)
    kmax = wl.K + 4 + 64
    idx = torch.empty(wl.B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(wl.B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_REFINE, wl.B, cand.shape[1], wl.K))
    lsa.lsa_topk_refine(d.q_I, d.w, d.k_I, cand, ccnt, wl.K, 4, 64, d.q_pos, idx, cnt, ws)
    torch.cuda.synchronize()
    ref = d.oracle_scores()
    for b in range(wl.B):
        row = cand[b, : counts[b]].cpu().numpy()
        dyn = row[4: counts[b] - 64]
        order = np.argsort(-ref[b, dyn], kind="stable")
        take = np.sort(dyn[order[: min(wl.K, dyn.size)]])
        kth = ref[b, take].min() if take.size else 0.0
        want = np.concatenate([np.arange(4), take, np.arange(int(qp[b]) - 63, int(qp[b]) + 1)])
        check_index_sets(idx[b].cpu().numpy(), int(cnt[b]), want, ref[b], kth, kmax)


def _attn_case(q, kv, idx, cnt, scale, check_rows):
    B, H = q.shape[0], q.shape[1]
    kmax = idx.shape[1]
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, kv.shape[0], kmax, H))
    lsa.lsa_sparse_attn(q, kv, idx, cnt, scale, out, lse, ws)
    lsa.lsa_device_status()
    counts = cnt.cpu().tolist()
    for b in check_rows:
        sel = idx[b, : counts[b]].cpu().numpy()
        ref, ref_lse = run_oracle_attention(q[b], kv, sel, scale)
        if counts[b] == 0:
            assert (out[b] == 0).all() and torch.isneginf(lse[b]).all()
            continue
        assert attn_rel_err(out[b], ref) <= ATTN_REL, b
        assert np.abs(f64(lse[b]) - ref_lse).max() <= 1e-3, b


def test_sparse_attn_decode_units():
    """The decode batch shape (16 queries, rows of up to 2048): units of up to 8 tiles of 32 rows, ragged
    counts (full, one short of a tile, a single row, none) and every query checked."""
    L, B, H = 40000, 16, 128
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, H, 576), DEV)
    counts = [2048, 2047, 2017, 1, 0, 256, 255, 33, 32, 31, 1500, 2048, 2048, 1999, 64, 2000]
    kmax = 2048
    rng = np.random.default_rng(16)
    idx = torch.full((B, kmax), -1, dtype=torch.int32)
    for b, c in enumerate(counts):
        idx[b, :c] = torch.from_numpy(np.sort(rng.choice(L, size=c, replace=False)).astype(np.int32))
    _attn_case(q, kv, idx.to(DEV), torch.tensor(counts, dtype=torch.int32, device=DEV), 1 / math.sqrt(576),
               range(B))


def test_sparse_attn_rescales_within_a_unit():
    """Logits that grow along each unit's rows by several 2^8 steps for some heads and shrink for others: the
    running softmax reference moves tile by tile for part of a warp's heads (the lazy rescale of O), and the
    second value half must replay those rescales exactly."""
    L, B, H = 32768, 16, 128
    g = torch.Generator().manual_seed(7)
    u = torch.randn(576, generator=g, dtype=torch.float64)
    u /= u.norm()
    # t(s) ramps 0 -> 500 over each eighth of the cache, so a unit (an eighth of a query's sorted rows) sees it
    # grow by ~60 per tile: z grows by ~3.7 (q_h . u) in log2 units per tile
    s = torch.arange(L, dtype=torch.float64)
    t = 500.0 * ((8.0 * s / L) % 1.0)
    noise = S.normal_bf16(S.ST_KV, (L, 576), "cpu").double()
    kv = (t[:, None] * u[None, :] + noise).to(torch.bfloat16).to(DEV)
    q = S.normal_bf16(S.ST_Q, (B, H, 576), DEV)
    kmax = 2048
    rng = np.random.default_rng(17)
    idx = torch.stack([torch.from_numpy(np.sort(rng.choice(L, size=kmax, replace=False)).astype(np.int32))
                       for _ in range(B)])
    counts = [kmax] * B
    counts[5] = 1111
    _attn_case(q, kv, idx.to(DEV), torch.tensor(counts, dtype=torch.int32, device=DEV), 1 / math.sqrt(576),
               range(B))


def test_sparse_attn_single_split_many_queries():
    """Enough queries that every query runs as one split (no combine pass)."""
    L, B, H = 30000, 80, 128
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, H, 576), DEV)
    rng = np.random.default_rng(80)
    counts = [int(c) for c in rng.integers(1, 300, B)]
    counts[3] = 0
    kmax = 300
    idx = torch.full((B, kmax), -1, dtype=torch.int32)
    for b, c in enumerate(counts):
        idx[b, :c] = torch.from_numpy(np.sort(rng.choice(L, size=c, replace=False)).astype(np.int32))
    idx, cnt = idx.to(DEV), torch.tensor(counts, dtype=torch.int32, device=DEV)
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, L, kmax, H))
    scale = 1 / math.sqrt(576)
    lsa.lsa_sparse_attn(q, kv, idx, cnt, scale, out, lse, ws)
    torch.cuda.synchronize()
    for b in (0, 3, 17, 79):
        sel = idx[b, : counts[b]].cpu().numpy()
        ref, ref_lse = run_oracle_attention(q[b], kv, sel, scale)
        if counts[b] == 0:
            assert (out[b] == 0).all() and torch.isneginf(lse[b]).all()
            continue
        assert attn_rel_err(out[b], ref) <= ATTN_REL
        assert np.abs(f64(lse[b]) - ref_lse).max() <= 1e-3


# --------------------------------------------------------------------------------------------
# HI two-stage selection
# --------------------------------------------------------------------------------------------


def _hi_run(wl, q_pos, P, Bsub, M):
    q_I, w = S.index_queries(wl)
    k = S.index_keys(wl, q_I, DEV)
    nsub = wl.L // Bsub
    means = torch.empty(nsub, 128, device=DEV)
    lsa.lsa_pool_keys(k, means, Bsub)
    split = torch.empty(3, nsub, 128, dtype=torch.bfloat16, device=DEV)
    lsa.lsa_split_representatives(means, split)
    kmax = wl.K + wl.sink + wl.window
    idx = torch.full((wl.B, kmax), 777, dtype=torch.int32, device=DEV)
    cnt = torch.empty(wl.B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_hi_workspace_size(wl.B, wl.L, P, Bsub, M, wl.K, wl.sink, wl.window))
    qp = torch.as_tensor(q_pos, dtype=torch.int64, device=DEV)
    lsa.lsa_hi_select(q_I.to(DEV), w.to(DEV), k, split, P, Bsub, M, wl.K, wl.sink, wl.window, qp, idx, cnt, ws)
    torch.cuda.synchronize()
    return q_I, w, k, idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("L,M", [(65536 + 37, 32), (40000, 64)])
def test_hi_select(L, M):
    """Against the oracle: the same set, except tokens whose score ties the K-th within 1e-5 (a page
    ranked differently at the M-th place would put tokens of other pages in the set and fail here)."""
    P, Bsub = 128, 8
    wl = S.Workload("hi", L=L, B=4, H_I=64, d_I=128, K=512, H=16, sink=4, window=128, needles="cos06",
                    n_needles=L // 100)
    q_pos = [L - 1, L - 501, 30003, 2047]
    q_I, w, k, idx_h, cnt_h = _hi_run(wl, q_pos, P, Bsub, M)
    qf, wf, kf = f64(q_I), f64(w), f64(k)
    for b in range(wl.B):
        want, kth, mth, recalled = O.hi_select_row(qf[b], wf[b], kf, q_pos[b], P, Bsub, M, wl.K, wl.sink, wl.window)
        got = idx_h[b, : cnt_h[b]]
        assert np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        assert got.max() <= q_pos[b]
        if np.array_equal(got, want):
            continue
        tok = O.index_score(qf[b][None], wf[b][None], kf[np.setxor1d(got, want)], np.array([L]))[0]
        assert np.all(np.abs(tok - kth) <= 1e-5 * abs(kth)), (b, np.setxor1d(got, want)[:8])


def test_hi_every_page_recalled_is_the_flat_selection():
    """M * P >= L: every visible token is recalled, so the result is the flat indexer + top-K's (up to
    ties of the K-th score within 1e-5, the two paths rounding the fp32 sums differently)."""
    P, Bsub, L = 128, 8, 32768 + 200
    wl = S.Workload("hi2", L=L, B=2, H_I=64, d_I=128, K=1024, H=16, sink=4, window=128, needles="cos06",
                    n_needles=300)
    q_pos = [L - 1, 20000]
    q_I, w, k, idx_h, cnt_h = _hi_run(wl, q_pos, P, Bsub, M=(L + P - 1) // P)
    scores = torch.empty(wl.B, (L + 3) // 4 * 4, device=DEV)
    qp = torch.as_tensor(q_pos, dtype=torch.int64, device=DEV)
    lsa.lsa_index_score(q_I.to(DEV), w.to(DEV), k, qp, scores)
    kmax = wl.K + wl.sink + wl.window
    idx = torch.empty(wl.B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(wl.B, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_select(scores, L, wl.K, wl.sink, wl.window, qp, idx, cnt)
    flat_h, fcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    sc = scores.cpu().numpy()
    for b in range(wl.B):
        got, ref = idx_h[b, : cnt_h[b]], flat_h[b, : fcnt[b]]
        diff = np.setxor1d(got, ref)
        if diff.size:
            kth = np.sort(sc[b, np.setdiff1d(ref, np.union1d(np.arange(4), np.arange(q_pos[b] - 127, q_pos[b] + 1)))])[0]
            assert np.all(np.abs(sc[b, diff] - kth) <= 1e-5 * abs(kth)), (b, diff[:8])


# --------------------------------------------------------------------------------------------
# HFA: sparse and contiguous branches on two streams, merged by LSE
# --------------------------------------------------------------------------------------------


@pytest.mark.parametrize("H,sink,window", [(128, 4, 128), (128, 0, 0), (128, 16, 1024), (16, 4, 128)])
def test_hybrid_attn(H, sink, window):
    """Against the oracle's merge of the two branches (and the attention over the union it equals), and
    against the single-pass kernel on the same rows."""
    L, B, K = 40000 + 5, 5, 700
    q_pos = [L - 1, L - 1, 30000, 900, 10]
    wl = S.Workload("hfa", L=L, B=B, H_I=64, d_I=128, K=K, H=H, sink=sink, window=window, needles="cos06",
                    n_needles=400)
    d = Decode(wl, q_pos=torch.tensor(q_pos, dtype=torch.int64))
    scores = torch.empty(B, L + 3, device=DEV)
    lsa.lsa_index_score(d.q_I, d.w, d.k_I, d.q_pos, scores)
    kmax = K + sink + window
    idx = torch.empty(B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_select(scores, L, K, sink, window, d.q_pos, idx, cnt)
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, H, 576), DEV)
    scale = 1 / math.sqrt(576)
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_HYBRID_ATTN, B, L, kmax, H, sink, window))
    lsa.lsa_hybrid_attn(q, kv, idx, cnt, sink, window, d.q_pos, scale, out, lse, ws)
    out1 = torch.empty_like(out)
    lse1 = torch.empty_like(lse)
    lsa.lsa_sparse_attn(q, kv, idx, cnt, scale, out1, lse1, lsa.workspace(lsa.lsa_workspace_size(
        lsa.LSA_OP_ATTN, B, L, kmax, H)))
    torch.cuda.synchronize()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        row = idx_h[b, : cnt_h[b]]
        s_sink, s_swa = O.fixed_positions(q_pos[b], sink, window)
        fixed = np.union1d(s_sink, s_swa)
        sparse = np.setdiff1d(row, fixed)
        assert np.array_equal(np.union1d(sparse, fixed), row)
        merged = O.lse_merge([run_oracle_attention(q[b], kv, sparse, scale),
                              run_oracle_attention(q[b], kv, fixed, scale)])
        ref, ref_lse = run_oracle_attention(q[b], kv, row, scale)
        np.testing.assert_allclose(merged[0], ref, rtol=1e-9, atol=1e-12)
        assert attn_rel_err(out[b], merged[0]) <= ATTN_REL
        assert np.abs(f64(lse[b]) - merged[1]).max() <= 1e-3
        assert attn_rel_err(out[b], f64(out1[b])) <= ATTN_REL


# --------------------------------------------------------------------------------------------
# MSA: group-wise block selection and the attention over it
# --------------------------------------------------------------------------------------------


def _msa_case(L, B, G, KB, q_pos):
    wl = S.Workload("msa", L=L, B=B, H_I=64, d_I=128, K=KB * 128, H=128, needles="cos06", n_needles=L // 100)
    q_I, w = S.index_queries(wl)
    k = S.index_keys(wl, q_I, DEV)
    ld = (G * KB + 1) * 128
    idx = torch.full((B, ld), -7, dtype=torch.int32, device=DEV)
    gm = torch.zeros(B, ld, dtype=torch.uint8, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_msa_workspace_size(B, L, G, KB))
    qp = torch.as_tensor(q_pos, dtype=torch.int64, device=DEV)
    lsa.lsa_msa_select(q_I.to(DEV), w.to(DEV), k, G, KB, qp, idx, gm, cnt, ws)
    torch.cuda.synchronize()
    return q_I, w, k, qp, idx, gm, cnt


@pytest.mark.parametrize("G,KB", [(8, 16), (1, 8), (4, 5)])
def test_msa_select(G, KB):
    """Each group's set (the union row's entries with its bit) against the oracle; blocks may differ only where
    their score ties the KB-th within 1e-5."""
    L, B = 40000 + 77, 4
    q_pos = [L - 1, 20000, 127, 300]
    q_I, w, k, _, idx, gm, cnt = _msa_case(L, B, G, KB, q_pos)
    qf, wf, kf = f64(q_I), f64(w), f64(k)
    idx_h, gm_h, cnt_h = idx.cpu().numpy(), gm.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        row, m = idx_h[b, : cnt_h[b]], gm_h[b, : cnt_h[b]]
        assert np.all(np.diff(row) > 0) and row.max() == q_pos[b]
        want = O.msa_select_row(qf[b], wf[b], kf, q_pos[b], G, 128, KB)
        for g in range(G):
            got = row[(m >> g) & 1 == 1]
            ref, kth = want[g]
            if np.array_equal(got, ref):
                continue
            hg = 64 // G
            for blk in np.unique(np.setxor1d(got, ref) // 128):
                sc = O.index_score(qf[b][None, g * hg:(g + 1) * hg], wf[b][None, g * hg:(g + 1) * hg],
                                   kf[blk * 128:(blk + 1) * 128], np.array([127]))[0].max()
                assert abs(sc - kth) <= 1e-5 * abs(kth), (b, g, blk)


@pytest.mark.parametrize("G,KB,q_pos", [(8, 16, [40076, 20000, 5000]), (2, 8, [40076, 20000, 5000]),
                                         (4, 5, [40076, 20000, 5000]), (1, 8, [40076, 20000, 5000]),
                                         (8, 4, [50, 127, 300, 40076]), (2, 3, [50, 127, 300, 40076])])
def test_msa_attn(G, KB, q_pos):
    """Head h attends to its group's rows only: against the oracle attention per head over those rows.  The last
    case has queries whose only block is the partial local one (q_pos 50, 127) and one with fewer kept blocks than
    KB (q_pos 300)."""
    L, B = 40000 + 77, len(q_pos)
    _, _, _, _, idx, gm, cnt = _msa_case(L, B, G, KB, q_pos)
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, 128, 576), DEV)
    scale = 1 / math.sqrt(576)
    out = torch.empty(B, 128, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, 128, device=DEV)
    ws = lsa.workspace(lsa.lsa_msa_attn_workspace_size(B, idx.shape[1], G))
    lsa.lsa_msa_attn(q, kv, idx, gm, cnt, G, scale, out, lse, ws)
    torch.cuda.synchronize()
    idx_h, gm_h, cnt_h = idx.cpu().numpy(), gm.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        row, m = idx_h[b, : cnt_h[b]], gm_h[b, : cnt_h[b]]
        for g in range(G):
            sel = row[(m >> g) & 1 == 1]
            heads = slice(g * (128 // G), (g + 1) * (128 // G))
            ref, ref_lse = run_oracle_attention(q[b, heads], kv, sel, scale)
            assert attn_rel_err(out[b, heads], ref) <= ATTN_REL, (b, g)
            assert np.abs(f64(lse[b, heads]) - ref_lse).max() <= 1e-3
