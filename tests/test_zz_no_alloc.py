"""lsa_bucket_select_noalloc: the selection entry point for callers that cannot allocate device memory.

Such callers (a plugin whose host framework owns every device allocation, a thread that must stay out
of the CUDA allocator) get the same selection from a scratch buffer compiled into the library.  These
tests call it through the C ABI and compare it with lsa_bucket_select, which uses caller-allocated
scratch: index sets are integer results, so they must match exactly, on two calls in a row.  This file
is collected last so that a run stopping at the first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import lsa_synth as S
import sparse_long_context_lightning_b200 as lsa
from oracle import lsa_oracle as O
from gpu_common import TIE_REL, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(L, B, M, bsz, sink, window, flat):
    wl = S.Workload("na", L=L, B=B, H_I=64, d_I=128, K=M * bsz, H=16, sink=sink, window=window,
                    mode="flat" if flat else "microblock", bsz=bsz, M=M)
    q_I, w = S.index_queries(wl)
    q_I, w = q_I.to(DEV), w.to(DEV)
    k = S.normal_bf16(S.ST_KI, (L, 128), DEV)
    members = S.bucket_members(wl).to(DEV) if flat else None
    nb = members.shape[0] if flat else L // bsz
    cen = torch.empty(nb, 128, device=DEV)
    lsa.lsa_pool_keys(k, cen, bsz, members=members)
    qp = torch.tensor([L - 1 - 3 * i for i in range(B)], dtype=torch.int64, device=DEV)
    kmax = M * bsz + (bsz - 1) + sink + window
    return q_I, w, cen, members, qp, kmax, nb


# (flat, L, B, M, bsz, sink, window).  The small cases (2048 and 4096 representatives) are shapes where the
# whole static buffer would also hold the tensor-core path's split copy of the representatives; the entry
# point must still score on the CUDA cores, as the smaller workspace does.
CASES = {
    "flat-20000": (True, 64 * 20000, 8, 32, 64, 4, 512),
    "micro-16384": (False, 4 * 16384 + 3, 4, 512, 4, 4, 128),
    "flat-2048": (True, 64 * 2048, 4, 32, 64, 4, 512),
    "micro-4096": (False, 4 * 4096 + 2, 3, 64, 4, 4, 128),
}


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_allocating_entry_point(case):
    flat, L, B, M, bsz, sink, window = CASES[case]
    q_I, w, cen, members, qp, kmax, nb = _case(L, B, M, bsz, sink, window, flat)
    ref_idx = torch.empty(B, kmax, dtype=torch.int32, device=DEV)
    ref_cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    # the static scratch has the smaller workspace's layout: CUDA-core scoring, as here
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_BUCKET_MIN, B, nb, M))
    lsa.lsa_bucket_select(q_I, w, cen, members, bsz, M, sink, window, L, qp, ref_idx, ref_cnt, ws)
    for _ in range(2):  # two calls in a row share the static scratch
        idx = torch.full((B, kmax), 99, dtype=torch.int32, device=DEV)
        cnt = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        lsa.lsa_bucket_select_noalloc(q_I, w, cen, members, bsz, M, sink, window, L, qp, idx, cnt)
        torch.cuda.synchronize()
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(idx, ref_idx)


def test_noalloc_rejects_requests_beyond_the_static_buffer():
    """156250 Flat buckets need 625 KB of scratch per query: 14 queries exceed the 8 MiB buffer."""
    B, NB, M = 14, 156250, 32
    q_I = torch.zeros(B, 64, 128, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(B, 64, device=DEV)
    cen = torch.zeros(NB, 128, device=DEV)
    members = torch.zeros(NB, 64, dtype=torch.int32, device=DEV)
    qp = torch.zeros(B, dtype=torch.int64, device=DEV)
    idx = torch.zeros(B, M * 64 + 63 + 4 + 512, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(B, dtype=torch.int32, device=DEV)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_bucket_select_noalloc(q_I, w, cen, members, 64, M, 4, 512, NB * 64, qp, idx, cnt)
    assert e.value.status == -3  # LSA_ERR_WORKSPACE
    assert b"static buffer" in lsa.load_library().lsa_last_error()


@pytest.mark.parametrize("case", ["flat-2048", "micro-4096"])
def test_noalloc_small_tables_match_the_oracle(case):
    """With few representatives the result is also the oracle's selection (ties at the M-th score aside)."""
    flat, L, B, M, bsz, sink, window = CASES[case]
    q_I, w, cen, members, qp, kmax, nb = _case(L, B, M, bsz, sink, window, flat)
    idx = torch.full((B, kmax), 99, dtype=torch.int32, device=DEV)
    cnt = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_bucket_select_noalloc(q_I, w, cen, members, bsz, M, sink, window, L, qp, idx, cnt)
    torch.cuda.synchronize()
    k = S.normal_bf16(S.ST_KI, (L, 128), "cpu")
    mem_np = members.cpu().numpy() if flat else None
    reps = O.pool_keys(f64(k), mem_np) if flat else O.pool_keys(f64(k), block=bsz)
    bs = O.bucket_scores(f64(q_I.cpu()), f64(w.cpu()), reps)
    owner = {}
    if flat:
        for c, row in enumerate(mem_np):
            for x in row:
                owner[int(x)] = c
    idx_h, cnt_h, qp_h = idx.cpu().numpy(), cnt.cpu().numpy(), qp.cpu().numpy()
    for b in range(B):
        want, mth, _ = O.bucket_select_row(bs[b], int(qp_h[b]), M, sink, window, members=mem_np,
                                           block=None if flat else bsz)
        got = idx_h[b, : cnt_h[b]]
        assert np.all(np.diff(got) > 0) and np.all(idx_h[b, cnt_h[b]:] == -1)
        for x in np.setxor1d(got, want).tolist():
            c = owner[x] if flat else x // bsz
            assert abs(bs[b, c] - mth) <= TIE_REL * abs(mth), (b, x, bs[b, c], mth)


def test_noalloc_second_call_allocates_nothing():
    """After a first call on the device (which may load the module and with it the static buffer), a
    further call leaves the device's free memory unchanged."""
    flat, L, B, M, bsz, sink, window = CASES["flat-2048"]
    q_I, w, cen, members, qp, kmax, nb = _case(L, B, M, bsz, sink, window, flat)
    idx = torch.empty(B, kmax, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, dtype=torch.int32, device=DEV)
    lsa.lsa_bucket_select_noalloc(q_I, w, cen, members, bsz, M, sink, window, L, qp, idx, cnt)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    lsa.lsa_bucket_select_noalloc(q_I, w, cen, members, bsz, M, sink, window, L, qp, idx, cnt)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
