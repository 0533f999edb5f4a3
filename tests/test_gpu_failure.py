"""Failure reporting on the GPU, exercised without faulting it.

- A bounded device-side wait that runs out: ``lsa_selftest_wait`` waits on an mbarrier that nothing completes,
  with a 1 ms limit, records the give-up and returns; ``lsa_device_status`` must report LSA_ERR_TIMEOUT once,
  then LSA_OK, and the context must stay usable.
- A selected index outside [0, L): every attention kernel clamps it (the access stays in bounds) and flags it;
  ``lsa_device_status`` must report LSA_ERR_DEVICE_CHECK once, then LSA_OK.
"""

import math

import numpy as np
import pytest
import torch

import lsa_synth as S
import sparse_long_context_lightning_b200 as lsa

pytestmark = pytest.mark.gpu

DEV = "cuda"
LSA_ERR_DEVICE_CHECK, LSA_ERR_TIMEOUT = -5, -6


def test_bounded_wait_gives_up_and_is_reported():
    lsa.lsa_device_status()  # clean start
    lsa.lsa_selftest_wait(1_000_000)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_device_status()
    assert e.value.status == LSA_ERR_TIMEOUT
    assert b"k_selftest_wait" in lsa.load_library().lsa_last_error()
    lsa.lsa_device_status()  # the flag was cleared
    x = torch.arange(1024, device=DEV, dtype=torch.float32)
    assert float(x.sum()) == 1024 * 1023 / 2  # the context still works


def test_selftest_rejects_bad_limits():
    for bad in (0, 2_000_000_000):
        with pytest.raises(lsa.LsaError) as e:
            lsa.lsa_selftest_wait(bad)
        assert e.value.status == -1


@pytest.mark.parametrize("B,H,kmax", [(4, 128, 100), (80, 128, 300), (2, 16, 100)])
def test_out_of_range_index_is_clamped_and_reported(B, H, kmax):
    """B=4: the decode (two-pass) kernel; 80 queries of 300 rows: the value-half kernel (more units than one
    wave of the two-pass kernel); H=16: the CUDA-core kernel."""
    L = 5000
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, H, 576), DEV)
    rng = np.random.default_rng(5)
    idx = torch.stack([torch.from_numpy(np.sort(rng.choice(L, size=kmax, replace=False)).astype(np.int32))
                       for _ in range(B)])
    cnt = torch.full((B,), kmax, dtype=torch.int32)
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, H, device=DEV)
    ws = lsa.workspace(lsa.lsa_workspace_size(lsa.LSA_OP_ATTN, B, L, kmax, H))
    scale = 1 / math.sqrt(576)
    lsa.lsa_device_status()
    good = idx.to(DEV)
    lsa.lsa_sparse_attn(q, kv, good, cnt.to(DEV), scale, out, lse, ws)
    lsa.lsa_device_status()  # valid indices: no flag
    bad = idx.clone()
    bad[B - 1, 7] = L + 5
    bad[0, kmax - 1] = -3
    lsa.lsa_sparse_attn(q, kv, bad.to(DEV), cnt.to(DEV), scale, out, lse, ws)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_device_status()
    assert e.value.status == LSA_ERR_DEVICE_CHECK
    lsa.lsa_device_status()
    # entries past count are never read, whatever they hold
    pad = idx.clone()
    cnt2 = torch.full((B,), kmax - 10, dtype=torch.int32)
    pad[:, kmax - 10:] = -1
    lsa.lsa_sparse_attn(q, kv, pad.to(DEV), cnt2.to(DEV), scale, out, lse, ws)
    lsa.lsa_device_status()


def test_msa_rows_that_are_not_whole_blocks_are_reported():
    """The 8-group MSA attention runs each kept block as one tile of 128 consecutive tokens; a union row whose
    block holds other tokens is computed all the same (every access stays in bounds) and flagged."""
    B, G, KB, L = 1, 8, 2, 4096
    ld = (G * KB + 1) * 128
    idx = torch.full((B, ld), -1, dtype=torch.int32)
    gm = torch.zeros((B, ld), dtype=torch.uint8)
    # two whole blocks for every group, the second one with its tokens reversed (still in [0, L))
    idx[0, :128] = torch.arange(256, 384, dtype=torch.int32)
    idx[0, 128:256] = torch.arange(1023, 895, -1, dtype=torch.int32)
    gm[0, :256] = 0xFF
    cnt = torch.tensor([256], dtype=torch.int32)
    kv = S.normal_bf16(S.ST_KV, (L, 576), DEV)
    q = S.normal_bf16(S.ST_Q, (B, 128, 576), DEV)
    out = torch.empty(B, 128, 512, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, 128, device=DEV)
    lsa.lsa_device_status()  # clean start
    lsa.lsa_msa_attn(q, kv, idx.to(DEV), gm.to(DEV), cnt.to(DEV), G, 1 / math.sqrt(576), out, lse,
                     lsa.workspace(lsa.lsa_msa_attn_workspace_size(B, ld, G)))
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_device_status()
    assert e.value.status == LSA_ERR_DEVICE_CHECK
    assert b"k_msa_attn_rows" in lsa.load_library().lsa_last_error()
    lsa.lsa_device_status()  # the flag was cleared
