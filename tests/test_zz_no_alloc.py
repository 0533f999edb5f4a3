"""lsa_bucket_select_noalloc: the selection entry point for callers that cannot allocate device memory.

Such callers (a plugin whose host framework owns every device allocation, a thread that must stay out
of the CUDA allocator) get the same selection from a scratch buffer compiled into the library.  These
tests call it through the C ABI and compare it with lsa_bucket_select, which uses caller-allocated
scratch: index sets are integer results, so they must match exactly, on two calls in a row.  This file
is collected last so that a run stopping at the first failure has already run every other test.
"""

import pytest
import torch

import lsa_synth as S
import sparse_long_context_lightning_b200 as lsa

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


@pytest.mark.parametrize("flat", [True, False])
def test_noalloc_matches_allocating_entry_point(flat):
    if flat:
        L, B, M, bsz, sink, window = 64 * 20000, 8, 32, 64, 4, 512
    else:
        L, B, M, bsz, sink, window = 4 * 16384 + 3, 4, 512, 4, 4, 128
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
