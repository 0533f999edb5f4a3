"""The seeded input generator: counter words, row regeneration, permutations."""

import torch

import lsa_synth as S


def test_counter_words_match_python_int_definition():
    idx = torch.tensor([0, 1, 2, 7, 12345678901, 5_759_999_999], dtype=torch.int64)
    for stream in (1, 5, 8):
        got = S.counter_words(stream, idx).tolist()
        base = S.stream_key(stream)
        want = [S._s64(S.mix64_int(base + (int(i) + 1) * S._GAMMA)) for i in idx]
        assert got == want


def test_rows_regenerate_full_tensor():
    full = S.normal_bf16(S.ST_KV, (300, 576))
    rows = torch.tensor([0, 17, 299, 5])
    assert torch.equal(S.latent_rows(S.Workload("x", 300, 1, 1, 1, 1, 1), rows).view(torch.int16),
                       full[rows].view(torch.int16))


def test_normal_and_uniform_moments():
    x = S.normal_bf16(3, (1 << 20,)).double()
    assert abs(x.mean().item()) < 5e-3 and abs(x.std().item() - 1.0) < 5e-3
    u = S.uniform_f32(2, (1 << 20,)).double()
    assert u.min() >= 0 and u.max() < 1 and abs(u.mean().item() - 0.5) < 2e-3


def test_permutation_and_members():
    p = S.permutation(8, 1000)
    assert torch.equal(torch.sort(p).values, torch.arange(1000))
    wl = S.Workload("f", 640, 1, 1, 4, 1, 1, mode="flat", bsz=64, M=2)
    m = S.bucket_members(wl)
    assert m.shape == (10, 64) and torch.equal(torch.sort(m.view(-1).long()).values, torch.arange(640))


def test_needles_have_cos06_to_their_query():
    wl = S.WORKLOADS["decode128k"]
    q_I, _ = S.index_queries(wl)
    pos, rows = S.needle_rows(wl, q_I)
    assert pos.numel() == 1310 and len(set(pos.tolist())) == 1310
    u = q_I.double().mean(dim=1)
    u = u / u.norm(dim=1, keepdim=True)
    b = torch.arange(pos.numel()) % wl.B
    cos = (rows.double() * u[b]).sum(1) / rows.double().norm(dim=1)
    assert (cos - 0.6).abs().max() < 0.01
