"""The C ABI without a GPU: the library loads, exports every declared entry point, and rejects bad
arguments before it launches anything."""

import ctypes
import os
import re

import pytest

import sparse_long_context_lightning_b200 as lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "lsa.h"), encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(lsa.LIB_PATH):
        from sparse_long_context_lightning_b200 import build
        build.build()
    return lsa.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"lsa_index_score", "lsa_topk_select", "lsa_bucket_select", "lsa_sparse_attn", "lsa_pool_keys"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(lsa.SIGNATURES), "binding is missing a declared entry point"


def test_status_strings(lib):
    assert lib.lsa_strerror(0) == b"ok"
    for st in range(-6, 0):
        assert lib.lsa_strerror(st) not in (b"", b"unknown status")
    assert lib.lsa_strerror(7) == b"unknown status"
    assert lib.lsa_version().startswith(b"lsa-b200")


def test_workspace_sizes(lib):
    assert lib.lsa_workspace_size(lsa.LSA_OP_TOPK, 16, 131072, 2048, 0, 0, 0) == 0
    nb = lib.lsa_workspace_size(lsa.LSA_OP_BUCKET_MIN, 8, 156250, 32, 0, 0, 0)
    assert nb >= 8 * 156250 * 4 + 8 * 32 * 4 + 8 * 4 and nb % 256 == 0
    # the full workspace adds the representatives' three-part bf16 split (3 x 156250 x 128 x 2 bytes)
    full = lib.lsa_workspace_size(lsa.LSA_OP_BUCKET, 8, 156250, 32, 0, 0, 0)
    assert full >= nb + 3 * 156250 * 128 * 2 and full % 256 == 0
    assert lib.lsa_workspace_size(99, 1, 1, 1, 1, 0, 0) == ctypes.c_size_t(-1).value
    assert lib.lsa_workspace_size(lsa.LSA_OP_ATTN, -1, 1, 1, 1, 0, 0) == ctypes.c_size_t(-1).value


def test_argument_checks_launch_nothing(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: every call below fails validation first
    # K = 0
    assert lib.lsa_topk_select(fake, 4096, 1, 4096, 0, 0, 0, fake, fake, 4096, fake, None) == -1
    # idx_ld too small for K + sink + window
    assert lib.lsa_topk_select(fake, 4096, 1, 4096, 256, 4, 128, fake, fake, 300, fake, None) == -1
    # ld < L
    assert lib.lsa_topk_select(fake, 100, 1, 4096, 16, 0, 0, fake, fake, 16, fake, None) == -1
    # unsupported latent width
    assert lib.lsa_sparse_attn(fake, fake, 10, fake, 8, fake, 1, 16, 512, 512, 1.0, fake, None, None, 0, None) == -2
    # unsupported head count
    assert lib.lsa_sparse_attn(fake, fake, 10, fake, 8, fake, 1, 12, 576, 512, 1.0, fake, None, None, 0, None) == -2
    # bf16 index mode with a scale pointer
    assert lib.lsa_index_score(fake, fake, fake, fake, None, 0, 1, 4, 32, 64, fake, fake, 64, None) == -1
    # FP8 mode without scales
    assert lib.lsa_index_score(fake, None, fake, fake, None, 1, 1, 4, 32, 64, fake, fake, 64, None) == -1
    # unsupported d_I
    assert lib.lsa_index_score(fake, None, fake, fake, None, 0, 1, 4, 48, 64, fake, fake, 64, None) == -2
    # bucket select: workspace missing
    assert lib.lsa_bucket_select(fake, None, fake, 0, 1, 4, 32, fake, 16, None, 4, 2, 0, 0, 64, fake, fake, 16, fake,
                                 None, 0, None) == -3
    # bucket select: FP8 representatives are not supported
    assert lib.lsa_bucket_select(fake, fake, fake, 1, 1, 4, 32, fake, 16, None, 4, 2, 0, 0, 64, fake, fake, 16, fake,
                                 fake, 1 << 20, None) == -2
    # pool keys: more micro-blocks than L / bsz
    assert lib.lsa_pool_keys(fake, 0, None, 64, 32, None, 4, 17, fake, None) == -1
    # empty batches are a no-op
    assert lib.lsa_topk_select(fake, 4096, 0, 4096, 8, 0, 0, fake, fake, 8, fake, None) == 0
    assert lib.lsa_sparse_attn(fake, fake, 10, fake, 8, fake, 0, 16, 576, 512, 1.0, fake, None, None, 0, None) == 0


def test_selection_workspace_sizes(lib):
    """Host-side size arithmetic of the tree, MSA and HI scratch (no device involved)."""
    bad = ctypes.c_size_t(-1).value
    # tree: at least the parent scores, both candidate rows and the parents' bf16 split
    t = lib.lsa_tree_workspace_size(8, 2442, 64, 64, 32)
    assert t % 256 == 0 and t >= 8 * 2444 * 4 + 2 * 8 * 4096 * 4 + 3 * 2442 * 128 * 2
    assert lib.lsa_tree_workspace_size(8, 2442, 0, 64, 32) == bad
    assert lib.lsa_tree_workspace_size(-1, 2442, 64, 64, 32) == bad
    # MSA selection: block scores for every (query, group)
    m = lib.lsa_msa_workspace_size(16, 131072, 8, 16)
    assert m % 256 == 0 and m >= 16 * 8 * 1024 * 4
    # MSA attention: G = 2, 4, 8 read the union row directly (no scratch); G = 1 compacts the rows for the
    # 128-head attention
    for G in (2, 4, 8):
        assert lib.lsa_msa_attn_workspace_size(16, 129 * 128, G) == 0
    a1 = lib.lsa_msa_attn_workspace_size(16, 129 * 128, 1)
    assert a1 % 256 == 0 and a1 >= 16 * 129 * 128 * 4
    assert lib.lsa_msa_attn_workspace_size(16, 128, 0) == bad
    assert lib.lsa_hi_workspace_size(4, 1 << 20, 128, 8, 1024, 2048, 4, 128) > 0


def test_selection_argument_checks_launch_nothing(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: every call below fails validation first
    # tree: NP must be ceil(NB / F)
    assert lib.lsa_tree_select(fake, fake, 1, 64, 128, fake, 1000, fake, 99, 10, fake, 64, 8, 4, 0, 0, 64000, fake,
                               fake, 256, fake, fake, 1 << 20, None) == -1
    # tree: M2 above 1024
    assert lib.lsa_tree_select(fake, fake, 1, 64, 128, fake, 1000, fake, 100, 10, fake, 64, 2000, 4, 0, 0, 64000,
                               fake, fake, 256, fake, fake, 1 << 20, None) == -1
    # tree: unsupported d_I
    assert lib.lsa_tree_select(fake, fake, 1, 64, 48, fake, 1000, fake, 100, 10, fake, 64, 8, 4, 0, 0, 64000, fake,
                               fake, 256, fake, fake, 1 << 20, None) == -2
    # tree: workspace missing
    assert lib.lsa_tree_select(fake, fake, 1, 64, 128, fake, 1000, fake, 100, 10, fake, 64, 8, 4, 0, 0, 64000, fake,
                               fake, 256, fake, None, 0, None) == -3
    # tree parents: F = 0
    assert lib.lsa_tree_parents(fake, 1000, 128, 0, fake, None) == -1
    # MSA selection: G = 3, and idx_ld too small for G*KB + 1 blocks
    assert lib.lsa_msa_select(fake, fake, fake, 1, 64, 128, 4096, 3, 4, fake, fake, fake, 1 << 16, fake, fake,
                              1 << 20, None) == -2
    assert lib.lsa_msa_select(fake, fake, fake, 1, 64, 128, 4096, 8, 4, fake, fake, fake, 128, fake, fake, 1 << 20,
                              None) == -1
    # MSA attention: G = 3; workspace missing
    assert lib.lsa_msa_attn(fake, fake, 4096, fake, fake, 1024, fake, 1, 128, 576, 512, 3, 1.0, fake, None, fake,
                            1 << 20, None) == -2
    assert lib.lsa_msa_attn(fake, fake, 4096, fake, fake, 1024, fake, 1, 128, 576, 512, 1, 1.0, fake, None, None, 0,
                            None) == -3  # G = 1 compacts the rows through the workspace (G = 2, 4, 8 need none)
    # empty batches are a no-op
    assert lib.lsa_tree_select(fake, fake, 0, 64, 128, fake, 1000, fake, 100, 10, fake, 64, 8, 4, 0, 0, 64000, fake,
                               fake, 256, fake, None, 0, None) == 0
