// C ABI of the library: argument validation, scratch layout, dispatch to the kernels.
#include <cstdio>
#include <cstring>

#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {

static thread_local char g_last_error[256] = "";

void set_last_error(const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg ? msg : "");
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LSA_OK;
  set_last_error(cudaGetErrorString(e));
  return LSA_ERR_CUDA;
}

int launch_score_simt(const void* q, const float* q_scale, const float* w, const void* k, const float* k_scale,
                      int dtype, int64_t B, int H_I, int d_I, int64_t L, const int64_t* q_pos, float* scores,
                      int64_t ld, cudaStream_t s);
int launch_topk_mode(const float* scores, int64_t ld, int64_t B, int64_t L, int K, int sink, int window,
                     const int64_t* q_pos, int mode, int div, int32_t* idx, int64_t idx_ld, int32_t* count,
                     int64_t kmax, cudaStream_t s);
size_t refine_ws_bytes(int64_t B, int64_t cand_ld, int K);
int launch_refine(const void* q, const float* w, const void* k, int64_t B, int H_I, int d_I, int64_t L,
                  const int32_t* cand, int64_t cand_ld, const int32_t* cand_count, int K, int sink, int window,
                  const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, int64_t kmax, void* ws,
                  cudaStream_t s);
int launch_attn_simt(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                     const int32_t* count, int64_t B, int H, float scale, void* out, float* lse, cudaStream_t s);

// Scratch layout of lsa_bucket_select: bucket scores [B, ld_nb] fp32 | kept [B, M] int32 | kept_count [B] int32
// | (tensor-core scoring) the representatives' exact three-part bf16 split [3, NB, 128] bf16.  Without the last
// part (a smaller workspace) the representatives are scored on the CUDA cores.
static void bucket_ws_layout(int64_t B, int64_t NB, int M, size_t* off_kept, size_t* off_cnt, size_t* off_split,
                             size_t* total_min, size_t* total, int64_t* ld_nb) {
  *ld_nb = (NB + 3) / 4 * 4;
  size_t o = align_up(static_cast<size_t>(B) * static_cast<size_t>(*ld_nb) * 4, 256);
  *off_kept = o;
  o = align_up(o + static_cast<size_t>(B) * static_cast<size_t>(M) * 4, 256);
  *off_cnt = o;
  o = align_up(o + static_cast<size_t>(B) * 4, 256);
  *total_min = o;
  *off_split = o;
  *total = align_up(o + static_cast<size_t>(NB) * 128 * 2 * 3, 256);
}

// the workspace without the split part (CUDA-core scoring)
size_t bucket_ws_min_bytes(int64_t B, int64_t NB, int M) {
  size_t a, b, c, mn, tot;
  int64_t ld;
  bucket_ws_layout(B, NB, M, &a, &b, &c, &mn, &tot, &ld);
  return mn;
}

// Scratch layout of lsa_hi_select: sub-block scores [B, ld_sub] fp32 | page scores [B, ld_pg] fp32 |
// kept pages [B, M] int32 | kept count [B] | candidate rows [B, cand_ld] int32 | candidate count [B] |
// the re-rank's own scratch.
struct HiLayout {
  int64_t nsub, npages, ld_sub, ld_pg, cand_ld;
  size_t o_page, o_kept, o_kcnt, o_cand, o_ccnt, o_ref, total;
};
static HiLayout hi_ws_layout(int64_t B, int64_t L, int P, int Bsub, int M, int K, int sink, int window) {
  HiLayout h;
  h.nsub = L / Bsub;
  h.npages = cdiv(L, P);
  h.ld_sub = (h.nsub + 3) / 4 * 4;
  h.ld_pg = (h.npages + 3) / 4 * 4;
  h.cand_ld = static_cast<int64_t>(M) * P + (Bsub - 1) + sink + window;
  size_t o = align_up(static_cast<size_t>(B) * h.ld_sub * 4, 256);
  h.o_page = o;
  o = align_up(o + static_cast<size_t>(B) * h.ld_pg * 4, 256);
  h.o_kept = o;
  o = align_up(o + static_cast<size_t>(B) * M * 4, 256);
  h.o_kcnt = o;
  o = align_up(o + static_cast<size_t>(B) * 4, 256);
  h.o_cand = o;
  o = align_up(o + static_cast<size_t>(B) * h.cand_ld * 4, 256);
  h.o_ccnt = o;
  o = align_up(o + static_cast<size_t>(B) * 4, 256);
  h.o_ref = o;
  h.total = o + refine_ws_bytes(B, h.cand_ld, K);
  return h;
}

// Scratch layout of lsa_msa_select: block scores [B G, ld_nb] fp32 | per-(query, group) positions [B G] int64 |
// kept blocks [B G, KB] int32 | kept count [B G] int32.
struct MsaLayout {
  int64_t nb, ld_nb;
  size_t o_qp, o_kept, o_kcnt, total;
};
static MsaLayout msa_ws_layout(int64_t B, int64_t L, int G, int KB) {
  MsaLayout m;
  m.nb = cdiv(L, 128);
  m.ld_nb = (m.nb + 3) / 4 * 4;
  size_t o = align_up(static_cast<size_t>(B) * G * m.ld_nb * 4, 256);
  m.o_qp = o;
  o = align_up(o + static_cast<size_t>(B) * G * 8, 256);
  m.o_kept = o;
  o = align_up(o + static_cast<size_t>(B) * G * KB * 4, 256);
  m.o_kcnt = o;
  m.total = align_up(o + static_cast<size_t>(B) * G * 4, 256);
  return m;
}

// Scratch layout of lsa_tree_select: parent scores [B, ldp] fp32 | kept parents [B, M2] | count [B] |
// candidate scores [B, ldc] fp32 | candidate buckets [B, ldc] int32 | selected slots [B, M] | count [B] |
// kept buckets [B, M] | count [B] | the parents' split [3, NP, 128] bf16.
struct TreeLayout {
  int64_t ldp, n_cand, ldc;
  size_t o_kp, o_kpc, o_cs, o_cid, o_pos, o_posc, o_kb, o_kbc, o_split, total;
};
static TreeLayout tree_ws_layout(int64_t B, int64_t NP, int F, int M2, int M) {
  TreeLayout t;
  t.ldp = (NP + 3) / 4 * 4;
  t.n_cand = static_cast<int64_t>(M2) * F;
  t.ldc = (t.n_cand + 3) / 4 * 4;
  const size_t b = static_cast<size_t>(B);
  size_t o = align_up(b * t.ldp * 4, 256);
  t.o_kp = o;
  o = align_up(o + b * M2 * 4, 256);
  t.o_kpc = o;
  o = align_up(o + b * 4, 256);
  t.o_cs = o;
  o = align_up(o + b * t.ldc * 4, 256);
  t.o_cid = o;
  o = align_up(o + b * t.ldc * 4, 256);
  t.o_pos = o;
  o = align_up(o + b * M * 4, 256);
  t.o_posc = o;
  o = align_up(o + b * 4, 256);
  t.o_kb = o;
  o = align_up(o + b * M * 4, 256);
  t.o_kbc = o;
  o = align_up(o + b * 4, 256);
  t.o_split = o;  // the parents' exact three-part bf16 split (tensor-core scoring of level 2)
  t.total = align_up(o + static_cast<size_t>(NP) * 128 * 2 * 3, 256);
  return t;
}

// Self-test of the give-up path: one thread waits on an mbarrier that nothing completes, with a short limit.
__device__ int g_selftest_timeout;
__global__ void k_selftest_wait(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  sm100::mbar_init(&bar, 1);
  sm100::fence_mbar_init();
  // phase 0 of `bar` never completes: the bounded wait runs out after limit_ns
  if (!sm100::mbar_wait(&bar, 0, limit_ns)) atomicExch(&g_selftest_timeout, 1);
}

static int take_selftest_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_selftest_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_selftest_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace lsa

using namespace lsa;

extern "C" {

const char* lsa_version(void) { return "lsa-b200 0.2"; }

int lsa_selftest_wait(uint64_t limit_ns, void* stream) {
  LSA_CHECK_ARG(limit_ns >= 1 && limit_ns <= 1000000000ull);
  k_selftest_wait<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  LSA_CUDA_TRY(cudaGetLastError());
  return LSA_OK;
}

int lsa_device_status(void* stream) {
  const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e);
  int a2_check = 0, at_check = 0, ma_check = 0;
  const int ix = take_index_timeout(), at = take_attn_timeout(&at_check), rs = take_rescore_timeout();
  const int a2 = take_attn2_flags(&a2_check), stw = take_selftest_timeout(), sm_check = take_attn_simt_check();
  const int tt = take_tree_tc_timeout(), ma = take_msa_attn_flags(&ma_check);
  if (ix < 0 || at < 0 || rs < 0 || a2 < 0 || stw < 0 || sm_check < 0 || tt < 0 || ma < 0)
    return cuda_status(cudaGetLastError());
  if (ix || at || rs || a2 || stw || tt || ma) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "bounded wait gave up in:%s%s%s%s%s%s%s", ix ? " k_index_score_tc" : "",
                  at ? " k_sparse_attn_tc" : "", rs ? " k_rescore_tc" : "", a2 ? " k_sparse_attn_2p" : "",
                  stw ? " k_selftest_wait" : "", tt ? " k_tree_child_tc" : "", ma ? " k_msa_attn_rows" : "");
    set_last_error(msg);
    return LSA_ERR_TIMEOUT;
  }
  if (a2_check || at_check || sm_check || ma_check) {
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "device check failed (a selected index outside [0, L), the row clamped; or MSA rows that are not whole "
                  "blocks) in:%s%s%s%s",
                  a2_check ? " k_sparse_attn_2p" : "", at_check ? " k_sparse_attn_tc" : "",
                  sm_check ? " k_attn_simt" : "", ma_check ? " k_msa_attn_rows" : "");
    set_last_error(msg);
    return LSA_ERR_DEVICE_CHECK;
  }
  return LSA_OK;
}

const char* lsa_last_error(void) { return g_last_error; }

const char* lsa_strerror(int status) {
  switch (status) {
    case LSA_OK: return "ok";
    case LSA_ERR_INVALID_ARG: return "invalid argument";
    case LSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LSA_ERR_CUDA: return "CUDA error (see lsa_last_error)";
    case LSA_ERR_DEVICE_CHECK: return "device-side check failed";
    case LSA_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

size_t lsa_workspace_size(int op, int64_t B, int64_t L, int K, int H, int sink, int window) {
  (void)sink;
  (void)window;
  if (B < 0 || L < 0 || K < 0 || H < 0) return static_cast<size_t>(-1);
  switch (op) {
    case LSA_OP_TOPK: return 0;
    case LSA_OP_BUCKET: {
      size_t ok, oc, osp, mn, tot;
      int64_t ldn;
      bucket_ws_layout(B, L, K, &ok, &oc, &osp, &mn, &tot, &ldn);
      return tot;
    }
    case LSA_OP_BUCKET_MIN: return bucket_ws_min_bytes(B, L, K);
    case LSA_OP_ATTN: return sparse_attn_ws_bytes(B, K, H);
    case LSA_OP_HYBRID_ATTN: return hybrid_attn_ws_bytes(B, K, H, sink, window);
    case LSA_OP_REFINE: return refine_ws_bytes(B, L, K);
    default: return static_cast<size_t>(-1);
  }
}

int lsa_index_score(const void* q_idx, const float* q_scale, const float* w, const void* k_idx, const float* k_scale,
                    int dtype, int64_t B, int H_I, int d_I, int64_t L, const int64_t* q_pos, float* scores,
                    int64_t ld, void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 0 && H_I >= 1 && H_I <= 64 && ld >= L && (ld % 4) == 0);
  LSA_CHECK_ARG(dtype == LSA_BF16 || dtype == LSA_FP8_E4M3);
  if (B == 0 || L == 0) return LSA_OK;
  LSA_CHECK_ARG(q_idx && w && k_idx && q_pos && scores);
  LSA_CHECK_ARG(aligned16(q_idx) && aligned16(k_idx) && aligned16(scores));
  LSA_CHECK_ARG(B <= 65535 * 16);
  if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
  if (H_I * d_I > 8192) return LSA_ERR_UNSUPPORTED;
  if (dtype == LSA_BF16) {
    LSA_CHECK_ARG(q_scale == nullptr && k_scale == nullptr);
  } else {
    LSA_CHECK_ARG(q_scale != nullptr && k_scale != nullptr);
  }
  return launch_index_score(q_idx, q_scale, w, k_idx, k_scale, dtype, B, H_I, d_I, L, q_pos, scores, ld,
                            static_cast<cudaStream_t>(stream));
}

int lsa_topk_select(const float* scores, int64_t ld, int64_t B, int64_t L, int K, int sink, int window,
                    const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 0 && L < (int64_t(1) << 31) && K >= 1 && sink >= 0 && window >= 0);
  LSA_CHECK_ARG(ld >= L && (ld % 4) == 0);
  const int64_t kmax_full = static_cast<int64_t>(K) + sink + window;
  LSA_CHECK_ARG(idx_ld >= kmax_full);
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(B <= 65535);
  LSA_CHECK_ARG(scores && q_pos && idx && count && aligned16(scores));
  if (L == 0) return LSA_ERR_INVALID_ARG;
  return launch_topk_mode(scores, ld, B, L, K, sink, window, q_pos, 0, 1, idx, idx_ld, count, kmax_full,
                          static_cast<cudaStream_t>(stream));
}

int lsa_topk_refine(const void* q_idx, const float* w, const void* k_idx, int64_t B, int H_I, int d_I, int64_t L,
                    const int32_t* cand, int64_t cand_ld, const int32_t* cand_count, int K, int sink, int window,
                    const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, void* ws, size_t ws_bytes,
                    void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 1 && L < (int64_t(1) << 31) && K >= 1 && sink >= 0 && window >= 0);
  LSA_CHECK_ARG(H_I >= 1 && H_I <= 64 && cand_ld >= 1 && cand_ld < (int64_t(1) << 31));
  const int64_t kmax_full = static_cast<int64_t>(K) + sink + window;
  LSA_CHECK_ARG(idx_ld >= kmax_full);
  if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(B <= 65535);
  LSA_CHECK_ARG(q_idx && w && k_idx && cand && cand_count && q_pos && idx && count);
  LSA_CHECK_ARG(aligned16(q_idx) && aligned16(k_idx));
  if (ws == nullptr || !aligned256(ws) || ws_bytes < refine_ws_bytes(B, cand_ld, K)) return LSA_ERR_WORKSPACE;
  return launch_refine(q_idx, w, k_idx, B, H_I, d_I, L, cand, cand_ld, cand_count, K, sink, window, q_pos, idx, idx_ld,
                       count, kmax_full, ws, static_cast<cudaStream_t>(stream));
}

int lsa_pool_keys(const void* k_idx, int dtype, const float* k_scale, int64_t L, int d_I, const int32_t* members,
                  int bsz, int64_t NB, float* centroids, void* stream) {
  LSA_CHECK_ARG(L >= 0 && NB >= 0 && bsz >= 1 && bsz <= 1024 && d_I >= 4 && (d_I % 4) == 0);
  LSA_CHECK_ARG(dtype == LSA_BF16 || dtype == LSA_FP8_E4M3);
  if (members == nullptr) LSA_CHECK_ARG(NB <= L / bsz);
  if (NB == 0) return LSA_OK;
  LSA_CHECK_ARG(k_idx && centroids && aligned16(centroids));
  if (dtype == LSA_FP8_E4M3) LSA_CHECK_ARG(k_scale != nullptr);
  return launch_pool_keys(k_idx, dtype, k_scale, L, d_I, members, bsz, NB, centroids,
                          static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace lsa {
// The selection of lsa_bucket_select / lsa_bucket_select_split: representatives as fp32 `centroids` or as
// their cached bf16 split (`split_given`, then centroids == nullptr).
static int bucket_select_impl(const void* q_idx, const float* q_scale, const float* w, int dtype, int64_t B, int H_I,
                              int d_I, const float* centroids, const void* split_given, int64_t NB,
                              const int32_t* members, int bsz, int M, int sink, int window, int64_t L,
                              const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, void* ws,
                              size_t ws_bytes, void* stream) {
  LSA_CHECK_ARG(B >= 0 && NB >= 1 && NB < (int64_t(1) << 31) && bsz >= 1 && M >= 1 && M <= 1024);
  LSA_CHECK_ARG(sink >= 0 && window >= 0 && L >= 1 && H_I >= 1 && H_I <= 64);
  LSA_CHECK_ARG(static_cast<int64_t>(M) * bsz + bsz + sink + window <= 8192);
  // the incomplete tail block exists only in micro-block mode
  const int64_t kmax_full = static_cast<int64_t>(M) * bsz + (members ? 0 : bsz - 1) + sink + window;
  LSA_CHECK_ARG(idx_ld >= kmax_full);
  if (dtype != LSA_BF16 || q_scale != nullptr) return LSA_ERR_UNSUPPORTED;
  if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
  // the shapes the tensor-core scoring tiles
  const bool tc_shape = d_I == 128 && (H_I == 32 || H_I == 64) && NB >= 128 && NB < (int64_t(1) << 29);
  if (split_given && !tc_shape) return LSA_ERR_UNSUPPORTED;
  if (members == nullptr) LSA_CHECK_ARG(NB <= L / bsz);
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(B <= 65535);
  LSA_CHECK_ARG(q_idx && w && (centroids || split_given) && q_pos && idx && count && aligned16(q_idx));
  LSA_CHECK_ARG(centroids ? aligned16(centroids) : aligned16(split_given));
  size_t off_kept, off_cnt, off_split, total_min, total;
  int64_t ldn;
  bucket_ws_layout(B, NB, M, &off_kept, &off_cnt, &off_split, &total_min, &total, &ldn);
  if (ws == nullptr || !aligned256(ws) || ws_bytes < total_min) return LSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* bscores = reinterpret_cast<float*>(base);
  int32_t* kept = reinterpret_cast<int32_t*>(base + off_kept);
  int32_t* kcnt = reinterpret_cast<int32_t*>(base + off_cnt);
  int st;
  if (split_given) {
    st = launch_centroid_score_tc(q_idx, w, split_given, B, H_I, NB, bscores, ldn, s);
  } else if (tc_shape && ws_bytes >= total) {
    // tensor cores when the workspace holds the split
    void* split = base + off_split;
    st = launch_split_bf16x3(centroids, NB * 128, split, s);
    if (st == LSA_OK) st = launch_centroid_score_tc(q_idx, w, split, B, H_I, NB, bscores, ldn, s);
  } else {
    st = launch_centroid_score(q_idx, w, centroids, B, H_I, d_I, NB, bscores, ldn, s);
  }
  if (st != LSA_OK) return st;
  // top-M buckets: all NB ranked (explicit members) or the complete visible micro-blocks
  st = launch_topk_mode(bscores, ldn, B, NB, M, 0, 0, q_pos, members ? 1 : 2, bsz, kept, M, kcnt, M, s);
  if (st != LSA_OK) return st;
  // rows are -1 padded up to idx_ld
  return launch_bucket_expand(kept, M, kcnt, members, bsz, sink, window, members ? 0 : bsz, q_pos, B, idx, idx_ld,
                              count, idx_ld, s);
}
}  // namespace lsa

extern "C" {

int lsa_bucket_select(const void* q_idx, const float* q_scale, const float* w, int dtype, int64_t B, int H_I,
                      int d_I, const float* centroids, int64_t NB, const int32_t* members, int bsz, int M, int sink,
                      int window, int64_t L, const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count,
                      void* ws, size_t ws_bytes, void* stream) {
  if (centroids == nullptr && B > 0) return LSA_ERR_INVALID_ARG;
  return bucket_select_impl(q_idx, q_scale, w, dtype, B, H_I, d_I, centroids, nullptr, NB, members, bsz, M, sink,
                            window, L, q_pos, idx, idx_ld, count, ws, ws_bytes, stream);
}

int lsa_bucket_select_split(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const void* split,
                            int64_t NB, const int32_t* members, int bsz, int M, int sink, int window, int64_t L,
                            const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, void* ws,
                            size_t ws_bytes, void* stream) {
  if (split == nullptr && B > 0) return LSA_ERR_INVALID_ARG;
  return bucket_select_impl(q_idx, nullptr, w, LSA_BF16, B, H_I, d_I, nullptr, split, NB, members, bsz, M, sink,
                            window, L, q_pos, idx, idx_ld, count, ws, ws_bytes, stream);
}

int lsa_split_representatives(const float* centroids, int64_t NB, int d_I, void* split, void* stream) {
  LSA_CHECK_ARG(NB >= 0 && d_I >= 4 && (d_I % 4) == 0);
  if (NB == 0) return LSA_OK;
  LSA_CHECK_ARG(centroids && split && aligned16(centroids) && aligned16(split));
  return launch_split_bf16x3(centroids, NB * d_I, split, static_cast<cudaStream_t>(stream));
}

int lsa_hybrid_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                    const int32_t* count, int64_t B, int H, int d_qk, int d_v, int sink, int window,
                    const int64_t* q_pos, float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                    void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 1 && idx_ld >= 0 && idx_ld <= 65536 && sink >= 0 && window >= 0);
  LSA_CHECK_ARG(static_cast<int64_t>(sink) + window <= 65536);
  if (d_qk != 576 || d_v != 512) return LSA_ERR_UNSUPPORTED;
  if (H != 16 && H != 32 && H != 64 && H != 128) return LSA_ERR_UNSUPPORTED;
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(q && kv && idx && count && q_pos && out);
  LSA_CHECK_ARG(aligned16(q) && aligned16(kv) && aligned16(out));
  LSA_CHECK_ARG(B <= 65535);
  return launch_hybrid_attn(q, kv, L, idx, idx_ld, count, B, H, sink, window, q_pos, scale, out, lse, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream));
}

size_t lsa_msa_workspace_size(int64_t B, int64_t L, int G, int KB) {
  if (B < 0 || L < 1 || G < 1 || KB < 1) return static_cast<size_t>(-1);
  return msa_ws_layout(B, L, G, KB).total;
}

int lsa_msa_select(const void* q_idx, const float* w, const void* k_idx, int64_t B, int H_I, int d_I, int64_t L,
                   int G, int KB, const int64_t* q_pos, int32_t* idx, uint8_t* gmask, int64_t idx_ld,
                   int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 1 && L < (int64_t(1) << 31) && KB >= 1 && G >= 1);
  if (d_I != 128 || H_I != 64 || (G != 1 && G != 2 && G != 4 && G != 8) || L < 128) return LSA_ERR_UNSUPPORTED;
  LSA_CHECK_ARG(static_cast<int64_t>(G) * KB + 1 <= 1024);
  LSA_CHECK_ARG(idx_ld >= (static_cast<int64_t>(G) * KB + 1) * 128);
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(B <= 65535 / G);
  LSA_CHECK_ARG(q_idx && w && k_idx && q_pos && idx && gmask && count && aligned16(q_idx) && aligned16(k_idx));
  const MsaLayout m = msa_ws_layout(B, L, G, KB);
  if (ws == nullptr || !aligned256(ws) || ws_bytes < m.total) return LSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* bs = reinterpret_cast<float*>(base);
  int64_t* qp1 = reinterpret_cast<int64_t*>(base + m.o_qp);
  int32_t* kept = reinterpret_cast<int32_t*>(base + m.o_kept);
  int32_t* kcnt = reinterpret_cast<int32_t*>(base + m.o_kcnt);
  // block scores per (query, group), fused into the indexer's epilogue; then per (query, group) the top-KB of
  // the blocks before the local one (MODE_BLOCKS ranks c < (pos + 1) / 128 with pos = q_pos - 1)
  int st = launch_block_max_tc(q_idx, w, k_idx, B, L, G, q_pos, bs, m.ld_nb, s);
  if (st == LSA_OK) st = launch_shift_qpos(q_pos, B, G, -1, qp1, s);
  if (st == LSA_OK) st = launch_topk_mode(bs, m.ld_nb, B * G, m.nb, KB, 0, 0, qp1, 2, 128, kept, KB, kcnt, KB, s);
  if (st == LSA_OK) st = launch_msa_expand(kept, KB, kcnt, G, 128, q_pos, B, idx, gmask, idx_ld, count, s);
  return st;
}

int lsa_tree_parents(const float* centroids, int64_t NB, int d_I, int F, float* parents, void* stream) {
  LSA_CHECK_ARG(NB >= 0 && d_I >= 1 && d_I <= 128 && F >= 1);
  if (NB == 0) return LSA_OK;
  LSA_CHECK_ARG(centroids && parents);
  return launch_tree_parents(centroids, NB, d_I, F, parents, static_cast<cudaStream_t>(stream));
}

size_t lsa_tree_workspace_size(int64_t B, int64_t NP, int F, int M2, int M) {
  if (B < 0 || NP < 0 || F < 1 || M2 < 1 || M < 1) return static_cast<size_t>(-1);
  return tree_ws_layout(B, NP, F, M2, M).total;
}

}  // extern "C"

namespace lsa {
// The tree search of lsa_tree_select / lsa_tree_select_split: children scored from the fp32 centres on the CUDA
// cores, or (split_given) from the centres' cached exact bf16 split on the tensor cores.
static int tree_select_impl(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const float* centroids,
                            const void* split_given, int64_t NB, const float* parents, int64_t NP, int F,
                            const int32_t* members, int bsz, int M2, int M, int sink, int window, int64_t L,
                            const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, void* ws,
                            size_t ws_bytes, void* stream) {
  LSA_CHECK_ARG(B >= 0 && NB >= 1 && NB < (int64_t(1) << 31) && F >= 1 && NP == cdiv(NB, F) && bsz >= 1);
  LSA_CHECK_ARG(M2 >= 1 && M2 <= 1024 && M >= 1 && M <= 1024 && static_cast<int64_t>(M2) * F < (int64_t(1) << 30));
  LSA_CHECK_ARG(sink >= 0 && window >= 0 && L >= 1 && H_I >= 1 && H_I <= 64);
  LSA_CHECK_ARG(static_cast<int64_t>(M) * bsz + sink + window <= 8192);
  LSA_CHECK_ARG(idx_ld >= static_cast<int64_t>(M) * bsz + sink + window);
  if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
  if (split_given && (F != 64 || H_I != 64 || d_I != 128 || NB >= (int64_t(1) << 29))) return LSA_ERR_UNSUPPORTED;
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(B <= 65535);
  LSA_CHECK_ARG(q_idx && w && (centroids || split_given) && parents && members && q_pos && idx && count);
  LSA_CHECK_ARG(aligned16(q_idx) && aligned16(parents) && (split_given ? aligned16(split_given) : aligned16(centroids)));
  const TreeLayout t = tree_ws_layout(B, NP, F, M2, M);
  if (ws == nullptr || !aligned256(ws) || ws_bytes < t.total) return LSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* pscore = reinterpret_cast<float*>(base);
  int32_t* kp = reinterpret_cast<int32_t*>(base + t.o_kp);
  int32_t* kpc = reinterpret_cast<int32_t*>(base + t.o_kpc);
  float* cscore = reinterpret_cast<float*>(base + t.o_cs);
  int32_t* cid = reinterpret_cast<int32_t*>(base + t.o_cid);
  int32_t* kpos = reinterpret_cast<int32_t*>(base + t.o_pos);
  int32_t* kposc = reinterpret_cast<int32_t*>(base + t.o_posc);
  int32_t* kb = reinterpret_cast<int32_t*>(base + t.o_kb);
  int32_t* kbc = reinterpret_cast<int32_t*>(base + t.o_kbc);
  // level 2: every parent centre scored -- on the tensor cores from the parents' exact bf16 split where the
  // shape tiles (fp32-accurate, as the Flat path), else on the CUDA cores -- and the M2 best kept
  int st;
  if (d_I == 128 && (H_I == 32 || H_I == 64) && NP >= 128 && NP < (int64_t(1) << 29)) {
    void* split = base + t.o_split;
    st = launch_split_bf16x3(parents, NP * 128, split, s);
    if (st == LSA_OK) st = launch_centroid_score_tc(q_idx, w, split, B, H_I, NP, pscore, t.ldp, s);
  } else {
    st = launch_centroid_score(q_idx, w, parents, B, H_I, d_I, NP, pscore, t.ldp, s);
  }
  if (st == LSA_OK) st = launch_topk_mode(pscore, t.ldp, B, NP, M2, 0, 0, q_pos, 1, 1, kp, M2, kpc, M2, s);
  // level 1: the kept parents' children (64 consecutive centre rows per parent on the tensor cores, else a gather
  // on the CUDA cores); the M best candidate slots
  if (st == LSA_OK) {
    if (split_given)
      st = launch_tree_child_score_tc(q_idx, w, B, split_given, NB, kp, M2, kpc, t.n_cand, cscore, cid, t.ldc, s);
    else
      st = launch_tree_child_score(q_idx, w, B, H_I, d_I, centroids, NB, F, kp, M2, kpc, t.n_cand, cscore, cid,
                                   t.ldc, s);
  }
  if (st == LSA_OK) st = launch_topk_mode(cscore, t.ldc, B, t.n_cand, M, 0, 0, q_pos, 1, 1, kpos, M, kposc, M, s);
  if (st == LSA_OK) st = launch_tree_map(kpos, M, kposc, cid, t.ldc, t.n_cand, B, kb, M, kbc, s);
  // the kept buckets' members, sink and window (Flat expansion)
  if (st == LSA_OK)
    st = launch_bucket_expand(kb, M, kbc, members, bsz, sink, window, 0, q_pos, B, idx, idx_ld, count, idx_ld, s);
  return st;
}
}  // namespace lsa

extern "C" {

int lsa_tree_select(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const float* centroids,
                    int64_t NB, const float* parents, int64_t NP, int F, const int32_t* members, int bsz, int M2,
                    int M, int sink, int window, int64_t L, const int64_t* q_pos, int32_t* idx, int64_t idx_ld,
                    int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  if (centroids == nullptr && B > 0) return LSA_ERR_INVALID_ARG;
  return tree_select_impl(q_idx, w, B, H_I, d_I, centroids, nullptr, NB, parents, NP, F, members, bsz, M2, M, sink,
                          window, L, q_pos, idx, idx_ld, count, ws, ws_bytes, stream);
}

int lsa_tree_select_split(const void* q_idx, const float* w, int64_t B, int H_I, int d_I, const void* split,
                          int64_t NB, const float* parents, int64_t NP, int F, const int32_t* members, int bsz,
                          int M2, int M, int sink, int window, int64_t L, const int64_t* q_pos, int32_t* idx,
                          int64_t idx_ld, int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  if (split == nullptr && B > 0) return LSA_ERR_INVALID_ARG;
  return tree_select_impl(q_idx, w, B, H_I, d_I, nullptr, split, NB, parents, NP, F, members, bsz, M2, M, sink,
                          window, L, q_pos, idx, idx_ld, count, ws, ws_bytes, stream);
}

// Scratch of lsa_msa_attn: G = 1 compacts the rows (all of the union, the one group's) and runs the 128-head
// attention on them: rows [B, idx_ld] | counts [B] | the attention's scratch.  G = 2, 4, 8 need none.
struct MsaAttnLayout {
  size_t o_cnt, o_att, total;
};
static MsaAttnLayout msa_attn_layout(int64_t B, int64_t idx_ld, int G) {
  MsaAttnLayout m;
  if (G > 1) {
    m.o_cnt = m.o_att = m.total = 0;
    return m;
  }
  m.o_cnt = align_up(static_cast<size_t>(B) * idx_ld * 4, 256);
  m.o_att = m.o_cnt + align_up(static_cast<size_t>(B) * 4, 256);
  m.total = m.o_att + sparse_attn_ws_bytes(B, idx_ld, 128);
  return m;
}

size_t lsa_msa_attn_workspace_size(int64_t B, int64_t idx_ld, int G) {
  if (B < 0 || idx_ld < 0 || G < 1) return static_cast<size_t>(-1);
  return msa_attn_layout(B, idx_ld, G).total;
}

int lsa_msa_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, const uint8_t* gmask, int64_t idx_ld,
                 const int32_t* count, int64_t B, int H, int d_qk, int d_v, int G, float scale, void* out, float* lse,
                 void* ws, size_t ws_bytes, void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 1 && idx_ld >= 0 && idx_ld <= 65536);
  if (d_qk != 576 || d_v != 512 || H != 128 || (G != 1 && G != 2 && G != 4 && G != 8)) return LSA_ERR_UNSUPPORTED;
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(q && kv && idx && gmask && count && out);
  LSA_CHECK_ARG(aligned16(q) && aligned16(kv) && aligned16(out) && B * G <= 65535);
  const MsaAttnLayout m = msa_attn_layout(B, idx_ld, G);
  if (m.total > 0 && (ws == nullptr || !aligned256(ws) || ws_bytes < m.total)) return LSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (G > 1) {
    // one CTA per (query, 16-head slice), each block its group kept on the MMA's M side, the group's blocks read
    // from the union row's masks
    return launch_msa_attn_rows(q, kv, L, idx, gmask, idx_ld, count, B, G, scale, out, lse, s);
  }
  // G = 1: the rows compacted, then the 128-head tensor-core attention
  unsigned char* base = static_cast<unsigned char*>(ws);
  int32_t* grows = reinterpret_cast<int32_t*>(base);
  int32_t* gcnt = reinterpret_cast<int32_t*>(base + m.o_cnt);
  int st = launch_msa_group_rows(idx, gmask, idx_ld, count, B, G, grows, gcnt, s);
  if (st == LSA_OK)
    st = launch_sparse_attn(q, kv, L, grows, idx_ld, gcnt, B, 128, scale, out, lse, base + m.o_att, ws_bytes - m.o_att, s);
  return st;
}

size_t lsa_hi_workspace_size(int64_t B, int64_t L, int P, int Bsub, int M, int K, int sink, int window) {
  if (B < 0 || L < 1 || P < 1 || Bsub < 1 || P % Bsub != 0 || M < 1 || K < 1 || sink < 0 || window < 0)
    return static_cast<size_t>(-1);
  return hi_ws_layout(B, L, P, Bsub, M, K, sink, window).total;
}

int lsa_hi_select(const void* q_idx, const float* w, const void* k_idx, int64_t B, int H_I, int d_I, int64_t L,
                  const void* sub_split, int P, int Bsub, int M, int K, int sink, int window, const int64_t* q_pos,
                  int32_t* idx, int64_t idx_ld, int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 1 && L < (int64_t(1) << 31) && K >= 1 && sink >= 0 && window >= 0);
  LSA_CHECK_ARG(Bsub >= 1 && P >= Bsub && P % Bsub == 0 && P <= 65536 && M >= 1 && M <= 1024);
  LSA_CHECK_ARG(static_cast<int64_t>(M) * P + Bsub + sink + window < (int64_t(1) << 31));
  LSA_CHECK_ARG(idx_ld >= static_cast<int64_t>(K) + sink + window);
  // the sub-block scoring is the tensor-core representative scoring
  if (d_I != 128 || (H_I != 32 && H_I != 64) || L / Bsub < 128 || L / Bsub >= (int64_t(1) << 29))
    return LSA_ERR_UNSUPPORTED;
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(B <= 65535);
  LSA_CHECK_ARG(q_idx && w && k_idx && sub_split && q_pos && idx && count);
  LSA_CHECK_ARG(aligned16(q_idx) && aligned16(k_idx) && aligned16(sub_split));
  const HiLayout h = hi_ws_layout(B, L, P, Bsub, M, K, sink, window);
  if (ws == nullptr || !aligned256(ws) || ws_bytes < h.total) return LSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* sub = reinterpret_cast<float*>(base);
  float* page = reinterpret_cast<float*>(base + h.o_page);
  int32_t* kept = reinterpret_cast<int32_t*>(base + h.o_kept);
  int32_t* kcnt = reinterpret_cast<int32_t*>(base + h.o_kcnt);
  int32_t* cand = reinterpret_cast<int32_t*>(base + h.o_cand);
  int32_t* ccnt = reinterpret_cast<int32_t*>(base + h.o_ccnt);
  // stage one: sub-block scores, page sums, the top-M pages (every page ranked; pages past q_pos are -inf)
  int st = launch_centroid_score_tc(q_idx, w, sub_split, B, H_I, h.nsub, sub, h.ld_sub, s);
  if (st == LSA_OK) st = launch_page_sum(sub, h.ld_sub, h.nsub, P, Bsub, h.npages, B, q_pos, page, h.ld_pg, s);
  if (st == LSA_OK) st = launch_topk_mode(page, h.ld_pg, B, h.npages, M, 0, 0, q_pos, 1, 1, kept, M, kcnt, M, s);
  // the recalled tokens as a candidate row, then stage two: the token score and top-K on them
  if (st == LSA_OK) st = launch_page_expand(kept, M, kcnt, P, Bsub, sink, window, q_pos, B, cand, h.cand_ld, ccnt, s);
  if (st == LSA_OK)
    st = launch_refine(q_idx, w, k_idx, B, H_I, d_I, L, cand, h.cand_ld, ccnt, K, sink, window, q_pos, idx, idx_ld,
                       count, static_cast<int64_t>(K) + sink + window, base + h.o_ref, s);
  return st;
}

int lsa_sparse_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                    const int32_t* count, int64_t B, int H, int d_qk, int d_v, float scale, void* out, float* lse,
                    void* ws, size_t ws_bytes, void* stream) {
  LSA_CHECK_ARG(B >= 0 && L >= 1 && idx_ld >= 0 && idx_ld <= 65536);
  if (d_qk != 576 || d_v != 512) return LSA_ERR_UNSUPPORTED;
  if (H != 16 && H != 32 && H != 64 && H != 128) return LSA_ERR_UNSUPPORTED;
  if (B == 0) return LSA_OK;
  LSA_CHECK_ARG(q && kv && idx && count && out);
  LSA_CHECK_ARG(aligned16(q) && aligned16(kv) && aligned16(out));
  LSA_CHECK_ARG(B <= 65535);
  return launch_sparse_attn(q, kv, L, idx, idx_ld, count, B, H, scale, out, lse, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace lsa {



}  // namespace lsa
