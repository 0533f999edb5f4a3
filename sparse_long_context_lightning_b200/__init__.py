"""Token-level sparse attention for one long-context layer on B200 (sm_100a).

Python binding of ``liblsa.so`` (C ABI declared in ``include/lsa.h``).  The functions below only
marshal arguments (device pointers, sizes, the current CUDA stream) into the C calls: every step of
the path runs in the library's CUDA kernels.  Importing this package does not load the library;
the first call does, and raises ``LsaError`` if the built library is missing.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblsa.so")

LSA_OK = 0
LSA_BF16 = 0
LSA_FP8_E4M3 = 1
LSA_OP_TOPK, LSA_OP_BUCKET, LSA_OP_ATTN, LSA_OP_REFINE, LSA_OP_BUCKET_MIN, LSA_OP_HYBRID_ATTN = 1, 2, 3, 4, 5, 6

_STATUS = {0: "LSA_OK", -1: "LSA_ERR_INVALID_ARG", -2: "LSA_ERR_UNSUPPORTED", -3: "LSA_ERR_WORKSPACE",
           -4: "LSA_ERR_CUDA", -5: "LSA_ERR_DEVICE_CHECK", -6: "LSA_ERR_TIMEOUT"}

# exported symbol -> (restype, argtypes)
_P, _I64, _I32, _F32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "lsa_index_score": (_I32, [_P, _P, _P, _P, _P, _I32, _I64, _I32, _I32, _I64, _P, _P, _I64, _P]),
    "lsa_topk_select": (_I32, [_P, _I64, _I64, _I64, _I32, _I32, _I32, _P, _P, _I64, _P, _P]),
    "lsa_topk_refine": (_I32, [_P, _P, _P, _I64, _I32, _I32, _I64, _P, _I64, _P, _I32, _I32, _I32, _P, _P, _I64, _P,
                               _P, _SZ, _P]),
    "lsa_pool_keys": (_I32, [_P, _I32, _P, _I64, _I32, _P, _I32, _I64, _P, _P]),
    "lsa_bucket_select": (_I32, [_P, _P, _P, _I32, _I64, _I32, _I32, _P, _I64, _P, _I32, _I32, _I32, _I32, _I64,
                                 _P, _P, _I64, _P, _P, _SZ, _P]),
    "lsa_bucket_select_noalloc": (_I32, [_P, _P, _P, _I32, _I64, _I32, _I32, _P, _I64, _P, _I32, _I32, _I32, _I32,
                                         _I64, _P, _P, _I64, _P, _P]),
    "lsa_split_representatives": (_I32, [_P, _I64, _I32, _P, _P]),
    "lsa_bucket_select_split": (_I32, [_P, _P, _I64, _I32, _I32, _P, _I64, _P, _I32, _I32, _I32, _I32, _I64, _P, _P,
                                       _I64, _P, _P, _SZ, _P]),
    "lsa_hi_select": (_I32, [_P, _P, _P, _I64, _I32, _I32, _I64, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P, _P, _I64,
                             _P, _P, _SZ, _P]),
    "lsa_hi_workspace_size": (_SZ, [_I64, _I64, _I32, _I32, _I32, _I32, _I32, _I32]),
    "lsa_hybrid_attn": (_I32, [_P, _P, _I64, _P, _I64, _P, _I64, _I32, _I32, _I32, _I32, _I32, _P, _F32, _P, _P, _P,
                               _SZ, _P]),
    "lsa_tree_parents": (_I32, [_P, _I64, _I32, _I32, _P, _P]),
    "lsa_tree_workspace_size": (_SZ, [_I64, _I64, _I32, _I32, _I32]),
    "lsa_tree_select": (_I32, [_P, _P, _I64, _I32, _I32, _P, _I64, _P, _I64, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                               _I64, _P, _P, _I64, _P, _P, _SZ, _P]),
    "lsa_tree_select_split": (_I32, [_P, _P, _I64, _I32, _I32, _P, _I64, _P, _I64, _I32, _P, _I32, _I32, _I32, _I32,
                                     _I32, _I64, _P, _P, _I64, _P, _P, _SZ, _P]),
    "lsa_msa_select": (_I32, [_P, _P, _P, _I64, _I32, _I32, _I64, _I32, _I32, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "lsa_msa_workspace_size": (_SZ, [_I64, _I64, _I32, _I32]),
    "lsa_msa_attn_workspace_size": (_SZ, [_I64, _I64, _I32]),
    "lsa_msa_attn": (_I32, [_P, _P, _I64, _P, _P, _I64, _P, _I64, _I32, _I32, _I32, _I32, _F32, _P, _P, _P, _SZ, _P]),
    "lsa_sparse_attn": (_I32, [_P, _P, _I64, _P, _I64, _P, _I64, _I32, _I32, _I32, _F32, _P, _P, _P, _SZ, _P]),
    "lsa_workspace_size": (_SZ, [_I32, _I64, _I64, _I32, _I32, _I32, _I32]),
    "lsa_device_status": (_I32, [_P]),
    "lsa_selftest_wait": (_I32, [ctypes.c_uint64, _P]),
    "lsa_strerror": (ctypes.c_char_p, [_I32]),
    "lsa_last_error": (ctypes.c_char_p, []),
    "lsa_version": (ctypes.c_char_p, []),
}


class LsaError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)} {detail}".strip())
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblsa.so (once).  Raises LsaError when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise LsaError("load_library", -4, f"{path} is missing: run `python -m sparse_long_context_lightning_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, st: int):
    if st != LSA_OK:
        lib = load_library()
        raise LsaError(fn, st, lib.lsa_last_error().decode() if st in (-4, -5, -6) else "")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return LSA_FP8_E4M3
    raise LsaError("dtype", -2, f"index tensors must be bf16 or e4m3 codes, got {t.dtype}")


def lsa_workspace_size(op: int, B: int, L: int, K: int, H: int = 0, sink: int = 0, window: int = 0) -> int:
    return int(load_library().lsa_workspace_size(op, B, L, K, H, sink, window))


def lsa_index_score(q_idx, w, k_idx, q_pos, scores, q_scale=None, k_scale=None, stream=None):
    """scores[b, s] = sum_j w[b,j] ReLU(q_idx[b,j] . k_idx[s]) (s <= q_pos[b]), else -inf."""
    B, H_I, d_I = q_idx.shape
    L = k_idx.shape[0]
    st = load_library().lsa_index_score(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale),
                                        _dtype_code(q_idx), B, H_I, d_I, L, _ptr(q_pos), _ptr(scores),
                                        scores.stride(0), _stream(stream))
    _check("lsa_index_score", st)


def lsa_topk_select(scores, L, K, sink, window, q_pos, idx, count, stream=None):
    """Top-K of each score row over [0, q_pos] minus sink/window, unioned with sink and window."""
    st = load_library().lsa_topk_select(_ptr(scores), scores.stride(0), scores.shape[0], L, K, sink, window,
                                        _ptr(q_pos), _ptr(idx), idx.stride(0), _ptr(count), _stream(stream))
    _check("lsa_topk_select", st)


def lsa_topk_refine(q_idx, w, k_idx, cand, cand_count, K, sink, window, q_pos, idx, count, ws, stream=None):
    """Re-rank the dynamic candidates of `cand` (a K' top-K row) with bf16 scores; keep the top K."""
    B, H_I, d_I = q_idx.shape
    st = load_library().lsa_topk_refine(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, H_I, d_I, k_idx.shape[0], _ptr(cand),
                                        cand.stride(0), _ptr(cand_count), K, sink, window, _ptr(q_pos), _ptr(idx),
                                        idx.stride(0), _ptr(count), _ptr(ws),
                                        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_topk_refine", st)


def lsa_pool_keys(k_idx, centroids, bsz, members=None, k_scale=None, stream=None):
    """centroids[c] = mean of the bsz member index keys (explicit members, or contiguous blocks)."""
    L, d_I = k_idx.shape
    st = load_library().lsa_pool_keys(_ptr(k_idx), _dtype_code(k_idx), _ptr(k_scale), L, d_I, _ptr(members), bsz,
                                      centroids.shape[0], _ptr(centroids), _stream(stream))
    _check("lsa_pool_keys", st)


def lsa_bucket_select(q_idx, w, centroids, members, bsz, M, sink, window, L, q_pos, idx, count, ws, stream=None):
    """Flat buckets (members given) or micro-blocks (members None): top-M representatives, expanded."""
    B, H_I, d_I = q_idx.shape
    st = load_library().lsa_bucket_select(_ptr(q_idx), None, _ptr(w), _dtype_code(q_idx), B, H_I, d_I,
                                          _ptr(centroids), centroids.shape[0], _ptr(members), bsz, M, sink, window,
                                          L, _ptr(q_pos), _ptr(idx), idx.stride(0), _ptr(count), _ptr(ws),
                                          0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_bucket_select", st)


def lsa_split_representatives(centroids, split, stream=None):
    """split[p] (bf16 [3, NB, d_I]): centroids == split[0] + split[1] + split[2] exactly."""
    NB, d_I = centroids.shape
    st = load_library().lsa_split_representatives(_ptr(centroids), NB, d_I, _ptr(split), _stream(stream))
    _check("lsa_split_representatives", st)


def lsa_bucket_select_split(q_idx, w, split, members, bsz, M, sink, window, L, q_pos, idx, count, ws, stream=None):
    """lsa_bucket_select from the representatives' cached bf16 split (lsa_split_representatives)."""
    B, H_I, d_I = q_idx.shape
    st = load_library().lsa_bucket_select_split(_ptr(q_idx), _ptr(w), B, H_I, d_I, _ptr(split), split.shape[1],
                                                _ptr(members), bsz, M, sink, window, L, _ptr(q_pos), _ptr(idx),
                                                idx.stride(0), _ptr(count), _ptr(ws),
                                                0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_bucket_select_split", st)


def lsa_device_status(stream=None):
    """Synchronise the stream and raise if a kernel gave up a bounded wait (LSA_ERR_TIMEOUT) or failed a
    device-side index check (LSA_ERR_DEVICE_CHECK) since the last check."""
    _check("lsa_device_status", load_library().lsa_device_status(_stream(stream)))


def lsa_selftest_wait(limit_ns, stream=None):
    """Launch a kernel whose bounded wait on an mbarrier nothing completes runs out after limit_ns."""
    _check("lsa_selftest_wait", load_library().lsa_selftest_wait(int(limit_ns), _stream(stream)))


def lsa_tree_parents(centroids, F, parents, stream=None):
    """Level-2 centres of the tree search: parent p = mean of the centres of buckets [pF, min((p+1)F, NB))."""
    NB, d_I = centroids.shape
    st = load_library().lsa_tree_parents(_ptr(centroids), NB, d_I, F, _ptr(parents), _stream(stream))
    _check("lsa_tree_parents", st)


def lsa_tree_workspace_size(B, NP, F, M2, M):
    return load_library().lsa_tree_workspace_size(B, NP, F, M2, M)


def lsa_tree_select(q_idx, w, centroids, parents, F, members, M2, M, sink, window, L, q_pos, idx, count, ws,
                    stream=None):
    """Two-level tree search: top-M2 parents, then the top-M of their children, expanded as Flat buckets."""
    B, H_I, d_I = q_idx.shape
    NB, bsz = members.shape
    st = load_library().lsa_tree_select(_ptr(q_idx), _ptr(w), B, H_I, d_I, _ptr(centroids), NB, _ptr(parents),
                                        parents.shape[0], F, _ptr(members), bsz, M2, M, sink, window, L,
                                        _ptr(q_pos), _ptr(idx), idx.stride(0), _ptr(count), _ptr(ws),
                                        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_tree_select", st)


def lsa_tree_select_split(q_idx, w, split, parents, F, members, M2, M, sink, window, L, q_pos, idx, count, ws,
                          stream=None):
    """lsa_tree_select with the children scored on the tensor cores from the centres' cached bf16 split."""
    B, H_I, d_I = q_idx.shape
    NB, bsz = members.shape
    st = load_library().lsa_tree_select_split(_ptr(q_idx), _ptr(w), B, H_I, d_I, _ptr(split), NB, _ptr(parents),
                                              parents.shape[0], F, _ptr(members), bsz, M2, M, sink, window, L,
                                              _ptr(q_pos), _ptr(idx), idx.stride(0), _ptr(count), _ptr(ws),
                                              0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_tree_select_split", st)


def lsa_hi_workspace_size(B, L, P, Bsub, M, K, sink, window):
    return load_library().lsa_hi_workspace_size(B, L, P, Bsub, M, K, sink, window)


def lsa_hi_select(q_idx, w, k_idx, sub_split, P, Bsub, M, K, sink, window, q_pos, idx, count, ws, stream=None):
    """Two-stage selection: top-M pages from the sub-block means' split, then token top-K on their tokens."""
    B, H_I, d_I = q_idx.shape
    L = k_idx.shape[0]
    st = load_library().lsa_hi_select(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, H_I, d_I, L, _ptr(sub_split), P, Bsub, M,
                                      K, sink, window, _ptr(q_pos), _ptr(idx), idx.stride(0), _ptr(count), _ptr(ws),
                                      0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_hi_select", st)


def lsa_bucket_select_noalloc(q_idx, w, centroids, members, bsz, M, sink, window, L, q_pos, idx, count,
                              stream=None):
    """lsa_bucket_select with the library's static 8 MiB scratch (for callers that cannot allocate)."""
    B, H_I, d_I = q_idx.shape
    st = load_library().lsa_bucket_select_noalloc(_ptr(q_idx), None, _ptr(w), _dtype_code(q_idx), B, H_I, d_I,
                                                  _ptr(centroids), centroids.shape[0], _ptr(members), bsz, M, sink,
                                                  window, L, _ptr(q_pos), _ptr(idx), idx.stride(0), _ptr(count),
                                                  _stream(stream))
    _check("lsa_bucket_select_noalloc", st)


def lsa_sparse_attn(q, kv, idx, count, scale, out, lse=None, ws=None, stream=None):
    """out[b,h] = softmax_{s in S_b}(scale q[b,h].kv[s]) kv[s,:512] over the selected latent rows."""
    B, H, d_qk = q.shape
    d_v = out.shape[-1]
    st = load_library().lsa_sparse_attn(_ptr(q), _ptr(kv), kv.shape[0], _ptr(idx), idx.stride(0), _ptr(count), B, H,
                                        d_qk, d_v, float(scale), _ptr(out), _ptr(lse), _ptr(ws),
                                        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_sparse_attn", st)


def lsa_hybrid_attn(q, kv, idx, count, sink, window, q_pos, scale, out, lse=None, ws=None, stream=None):
    """lsa_sparse_attn over sink | sparse | window rows, the fixed part on a second stream, merged by LSE."""
    B, H, d_qk = q.shape
    d_v = out.shape[-1]
    st = load_library().lsa_hybrid_attn(_ptr(q), _ptr(kv), kv.shape[0], _ptr(idx), idx.stride(0), _ptr(count), B, H,
                                        d_qk, d_v, sink, window, _ptr(q_pos), float(scale), _ptr(out), _ptr(lse),
                                        _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                        _stream(stream))
    _check("lsa_hybrid_attn", st)


def lsa_msa_workspace_size(B, L, G, KB):
    return load_library().lsa_msa_workspace_size(B, L, G, KB)


def lsa_msa_select(q_idx, w, k_idx, G, KB, q_pos, idx, gmask, count, ws, stream=None):
    """Group-wise block selection: per group of index heads, top-KB 128-token blocks by max-pooled score."""
    B, H_I, d_I = q_idx.shape
    st = load_library().lsa_msa_select(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, H_I, d_I, k_idx.shape[0], G, KB,
                                       _ptr(q_pos), _ptr(idx), _ptr(gmask), idx.stride(0), _ptr(count), _ptr(ws),
                                       0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_msa_select", st)


def lsa_msa_attn_workspace_size(B, idx_ld, G):
    return load_library().lsa_msa_attn_workspace_size(B, idx_ld, G)


def lsa_msa_attn(q, kv, idx, gmask, count, G, scale, out, lse=None, ws=None, stream=None):
    """Attention over a group-wise selection: head h attends to the rows its group kept."""
    B, H, d_qk = q.shape
    d_v = out.shape[-1]
    st = load_library().lsa_msa_attn(_ptr(q), _ptr(kv), kv.shape[0], _ptr(idx), _ptr(gmask), idx.stride(0),
                                     _ptr(count), B, H, d_qk, d_v, G, float(scale), _ptr(out), _ptr(lse), _ptr(ws),
                                     0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("lsa_msa_attn", st)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Caller-owned scratch buffer (256-byte aligned by the CUDA caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
