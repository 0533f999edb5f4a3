"""Parity at the workloads' full sizes, in the launch configuration the bench uses.

The oracle checks every query of the decode workloads and a seeded sample of 256 rows (plus the first
and last) of the 8192-query causal prefill chunk.  The 10M-token Flat workload keeps an 11.5 GB latent
cache on the device; the oracle rebuilds every representative from the member keys in fp64.
"""


import numpy as np
import pytest
import torch

import lsa_synth as S
import sparse_long_context_lightning_b200 as lsa
from oracle import lsa_oracle as O

from gpu_common import ATTN_REL, Decode, attn_rel_err, f64, run_oracle_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fp8_select(d: Decode, wl: S.Workload):
    """FP8 scan -> top-2K (+sink/window) -> exact bf16 re-rank to K: the FP8-mode selection."""
    L, B = wl.L, d.B
    scores = torch.empty(B, L, device=DEV)
    lsa.lsa_index_score(d.q8, d.w, d.k8, d.q_pos, scores, q_scale=d.q_scale, k_scale=d.k_scale)
    K2 = 2 * wl.K
    cand = torch.empty(B, K2 + wl.sink + wl.window, dtype=torch.int32, device=DEV)
    ccnt = torch.empty(B, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_select(scores, L, K2, wl.sink, wl.window, d.q_pos, cand, ccnt)
    del scores
    kmax = wl.K + wl.sink + wl.window
    idx = torch.empty(B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_REFINE, B, cand.shape[1], wl.K))
    lsa.lsa_topk_refine(d.q_I, d.w, d.k_I, cand, ccnt, wl.K, wl.sink, wl.window, d.q_pos, idx, cnt, ws)
    return idx, cnt


def _attend(wl, q, kv, idx, cnt):
    B = idx.shape[0]
    out = torch.empty(B, wl.H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, wl.H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, kv.shape[0], idx.shape[1], wl.H))
    lsa.lsa_sparse_attn(q, kv, idx, cnt, wl.scale, out, lse, ws)
    return out, lse


def _recall_and_attention(d, wl, idx, cnt, q, kv, out, lse, rows, ref_bf16):
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    rec = []
    for i, b in enumerate(rows):
        want, _, _ = O.topk_row(ref_bf16[i], int(d.q_pos[b]), wl.K, wl.sink, wl.window)
        got = idx_h[b, : cnt_h[b]]
        assert cnt_h[b] == want.size and np.all(np.diff(got) > 0)
        rec.append(np.intersect1d(got, want).size / want.size)
        ref, ref_lse = run_oracle_attention(q[b], kv, got, wl.scale)
        assert attn_rel_err(out[b], ref) <= ATTN_REL
        assert np.abs(f64(lse[b]) - ref_lse).max() <= 1e-3
    return float(np.mean(rec)), float(np.min(rec))


def test_prefill_chunk_sampled_rows():
    """8192 causal queries (q_pos 122880..131071) over L = 131072, FP8 scan + re-rank, K=2048 + 4 + 128."""
    wl = S.WORKLOADS["prefill"]
    d = Decode(wl, fp8=True)
    idx, cnt = _fp8_select(d, wl)
    q = S.attn_queries(wl, DEV)
    kv = S.latent_cache(wl, DEV)
    out, lse = _attend(wl, q, kv, idx, cnt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = sorted({0, wl.B - 1, *rng.choice(np.arange(1, wl.B - 1), 256, replace=False).tolist()})
    ref = np.concatenate([d.oracle_scores_bf16(rows[i: i + 8]) for i in range(0, len(rows), 8)])
    mean, mn = _recall_and_attention(d, wl, idx, cnt, q, kv, out, lse, rows, ref)
    print(f"prefill sampled rows={len(rows)} recall mean {mean:.4f} min {mn:.4f}")
    assert mean >= 0.99


def test_decode1m_fp8():
    wl = S.WORKLOADS["decode1m"]
    d = Decode(wl, fp8=True)
    idx, cnt = _fp8_select(d, wl)
    q = S.attn_queries(wl, DEV)
    kv = S.latent_cache(wl, DEV)
    out, lse = _attend(wl, q, kv, idx, cnt)
    torch.cuda.synchronize()
    ref = d.oracle_scores_bf16()
    mean, mn = _recall_and_attention(d, wl, idx, cnt, q, kv, out, lse, list(range(wl.B)), ref)
    print(f"decode1m recall mean {mean:.4f} min {mn:.4f}")
    assert mean >= 0.99


@pytest.mark.parametrize("L", [1048576, 1048575])
def test_decode1m_microblock(L):
    """Micro-block variant: 4-token mean-pooled keys, top-512 blocks + incomplete tail + sink 4 + window 128."""
    base = S.WORKLOADS["decode1m_mb"]
    wl = S.Workload(base.name, L=L, B=base.B, H_I=64, d_I=128, K=base.K, H=128, sink=4, window=128,
                    needles="cos06", n_needles=10485, mode="microblock", bsz=4, M=512)
    d = Decode(wl)
    nb = L // 4
    cen = torch.empty(nb, 128, device=DEV)
    lsa.lsa_pool_keys(d.k_I, cen, 4)
    kmax = wl.kmax
    idx = torch.empty(wl.B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(wl.B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_BUCKET, wl.B, nb, wl.M))
    lsa.lsa_bucket_select(d.q_I, d.w, cen, None, 4, wl.M, 4, 128, L, d.q_pos, idx, cnt, ws)
    q = S.attn_queries(wl, DEV)
    kv = S.latent_cache(wl, DEV)
    out, lse = _attend(wl, q, kv, idx, cnt)
    torch.cuda.synchronize()
    kf = f64(d.k_I)
    reps = O.pool_keys(kf, block=4)
    np.testing.assert_allclose(f64(cen), reps, rtol=1e-6, atol=1e-7)
    bs = O.bucket_scores(f64(d.q_I_cpu), f64(d.w_cpu), reps)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(wl.B):
        want, mth, _ = O.bucket_select_row(bs[b], int(d.q_pos[b]), wl.M, 4, 128, block=4)
        got = idx_h[b, : cnt_h[b]]
        assert np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        for s in np.setxor1d(got, want).tolist():
            assert abs(bs[b, s // 4] - mth) <= 1e-5 * abs(mth), (b, s)
        if L % 4:
            assert set(range(4 * (L // 4), L)) <= set(got.tolist()), "tail tokens must be read"
        ref, _ = run_oracle_attention(q[b], kv, got, wl.scale)
        assert attn_rel_err(out[b], ref) <= ATTN_REL


def test_flat10m():
    """L = 10M: 156,250 Flat buckets of 64, top-32 + sink 4 + window 512, attention over an 11.5 GB cache."""
    wl = S.WORKLOADS["flat10m"]
    q_I, w = S.index_queries(wl)
    k_I = S.index_keys(wl, q_I, DEV)
    members = S.bucket_members(wl, DEV)
    nb = members.shape[0]
    cen = torch.empty(nb, 128, device=DEV)
    lsa.lsa_pool_keys(k_I, cen, wl.bsz, members=members)
    qp = wl.q_pos().to(DEV)
    kmax = wl.kmax
    idx = torch.empty(wl.B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(wl.B, dtype=torch.int32, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_BUCKET, wl.B, nb, wl.M))
    lsa.lsa_bucket_select(q_I.to(DEV), w.to(DEV), cen, members, wl.bsz, wl.M, wl.sink, wl.window, wl.L, qp, idx, cnt,
                          ws)
    q = S.attn_queries(wl, DEV)
    kv = S.latent_cache(wl, DEV)
    out, lse = _attend(wl, q, kv, idx, cnt)
    torch.cuda.synchronize()
    # oracle: representatives in fp64 from the member keys, in chunks of buckets
    mem_h = members.cpu().numpy()
    reps = np.empty((nb, 128))
    for c0 in range(0, nb, 8192):
        rows = members[c0: c0 + 8192].reshape(-1).long()
        kk = f64(k_I[rows]).reshape(-1, wl.bsz, 128)
        reps[c0: c0 + 8192] = kk.mean(axis=1)
    gcen = f64(cen)
    assert np.abs(gcen - reps).max() <= 1e-6 * max(1.0, np.abs(reps).max())
    bs = O.bucket_scores(f64(q_I), f64(w), reps)
    owner = np.empty(wl.L, dtype=np.int64)
    owner[mem_h.reshape(-1)] = np.repeat(np.arange(nb), wl.bsz)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    del kv
    for b in range(wl.B):
        want, mth, _ = O.bucket_select_row(bs[b], wl.L - 1, wl.M, wl.sink, wl.window, members=mem_h)
        got = idx_h[b, : cnt_h[b]]
        assert np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        for s in np.setxor1d(got, want).tolist():
            assert abs(bs[b, owner[s]] - mth) <= 1e-5 * abs(mth), (b, s)
        rows = S.latent_rows(wl, torch.as_tensor(got, dtype=torch.int64))
        ref, ref_lse = O.sparse_mla_attn(f64(q[b]), f64(rows), wl.scale)
        assert attn_rel_err(out[b], ref) <= ATTN_REL
        assert np.abs(f64(lse[b]) - ref_lse).max() <= 1e-3
