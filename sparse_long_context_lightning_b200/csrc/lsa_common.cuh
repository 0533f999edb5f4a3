// Shared device helpers of the sm_100a library (no host-visible API here).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cooperative_groups.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <vector>

#include "../../include/lsa.h"

namespace cg = cooperative_groups;

namespace lsa {

// ---------------------------------------------------------------------------
// host-side error plumbing
// ---------------------------------------------------------------------------
void set_last_error(const char* msg);
int cuda_status(cudaError_t e);  // LSA_OK or LSA_ERR_CUDA (+ records the message)

#define LSA_CHECK_ARG(cond)                  \
  do {                                       \
    if (!(cond)) return LSA_ERR_INVALID_ARG; \
  } while (0)

#define LSA_CUDA_TRY(expr)                           \
  do {                                               \
    cudaError_t e_ = (expr);                         \
    if (e_ != cudaSuccess) return lsa::cuda_status(e_); \
  } while (0)

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device): the attribute outlives
// the launch, so later launches skip the host call.
inline cudaError_t func_smem_once(const void* f, int bytes) {
  struct Entry {
    const void* f;
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : done)
    if (x.f == f && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back(Entry{f, dev, bytes});
  return e;
}

// Launch with programmatic stream serialization (the kernel may start while the previous kernel of the stream
// finishes; it calls pdl_wait() before its first global access) and, if cluster_x > 0, a cluster dimension.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

// bf16 bits -> fp32 (exact).
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// OCP e4m3fn code -> fp32 (exact; every e4m3 value is an fp32 value).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  const uint32_t sign = (c & 0x80u) << 24;
  const uint32_t e = (c >> 3) & 0xFu;
  const uint32_t m = c & 0x7u;
  float v;
  if (e == 0) {
    v = static_cast<float>(m) * 0.001953125f;  // m/8 * 2^-6
  } else {
    v = __uint_as_float(((e + 120u) << 23) | (m << 20));  // (1+m/8) * 2^(e-7)
  }
  if ((c & 0x7Fu) == 0x7Fu) v = __uint_as_float(0x7FC00000u);
  return __uint_as_float(__float_as_uint(v) | sign);
}

// Order-preserving map of an fp32 bit pattern to uint32: a < b (as floats, -0 < +0) <=> key(a) < key(b).
__device__ __forceinline__ uint32_t f32_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace lsa

// Launch helpers implemented per kernel file (called from lsa_api.cu).
namespace lsa {
int launch_index_score(const void* q, const float* q_scale, const float* w, const void* k,
                       const float* k_scale, int dtype, int64_t B, int H_I, int d_I, int64_t L,
                       const int64_t* q_pos, float* scores, int64_t ld, cudaStream_t s);
int launch_centroid_score(const void* q, const float* w, const float* centroids, int64_t B, int H_I,
                          int d_I, int64_t NB, float* scores, int64_t ld, cudaStream_t s);
int launch_split_bf16x3(const float* x, int64_t n, void* out, cudaStream_t s);
int launch_centroid_score_tc(const void* q, const float* w, const void* split, int64_t B, int H_I, int64_t NB,
                             float* scores, int64_t ld, cudaStream_t s);
size_t bucket_ws_min_bytes(int64_t B, int64_t NB, int M);
int launch_page_sum(const float* sub, int64_t sub_ld, int64_t nsub, int P, int Bsub, int64_t npages, int64_t B,
                    const int64_t* q_pos, float* page, int64_t page_ld, cudaStream_t s);
int launch_page_expand(const int32_t* kept, int64_t kept_ld, const int32_t* kcnt, int P, int Bsub, int sink,
                       int window, const int64_t* q_pos, int64_t B, int32_t* cand, int64_t cand_ld,
                       int32_t* ccount, cudaStream_t s);
int launch_pool_keys(const void* k, int dtype, const float* k_scale, int64_t L, int d_I,
                     const int32_t* members, int bsz, int64_t NB, float* centroids, cudaStream_t s);
int launch_bucket_expand(const int32_t* kept, int64_t kept_ld, const int32_t* kept_count,
                         const int32_t* members, int bsz, int sink, int window, int tail_block,
                         const int64_t* q_pos, int64_t B, int32_t* idx, int64_t idx_ld, int32_t* count,
                         int64_t kmax, cudaStream_t s);
int launch_hybrid_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                       const int32_t* count, int64_t B, int H, int sink, int window, const int64_t* q_pos,
                       float scale, void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t s);
size_t hybrid_attn_ws_bytes(int64_t B, int64_t idx_ld, int H, int sink, int window);
int launch_sparse_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                       const int32_t* count, int64_t B, int H, float scale, void* out, float* lse,
                       void* ws, size_t ws_bytes, cudaStream_t s);
int take_index_timeout();
int take_attn_timeout(int* check);
int take_attn_simt_check();
int take_tree_tc_timeout();
int launch_tree_child_score_tc(const void* q, const float* w, int64_t B, const void* split, int64_t NB,
                               const int32_t* kp, int64_t kp_ld, const int32_t* kpc, int64_t n_cand, float* cscore,
                               int32_t* cid, int64_t ldc, cudaStream_t s);
int take_rescore_timeout();
int launch_tree_parents(const float* reps, int64_t NB, int d_I, int F, float* parents, cudaStream_t s);
int launch_tree_child_score(const void* q, const float* w, int64_t B, int H_I, int d_I, const float* reps, int64_t NB,
                            int F, const int32_t* kp, int64_t kp_ld, const int32_t* kpc, int64_t n_cand,
                            float* cscore, int32_t* cid, int64_t ldc, cudaStream_t s);
int launch_tree_map(const int32_t* kpos, int64_t kpos_ld, const int32_t* kposc, const int32_t* cid, int64_t ldc,
                    int64_t n_cand, int64_t B, int32_t* kept, int64_t kept_ld, int32_t* kcount, cudaStream_t s);
int launch_msa_group_rows(const int32_t* idx, const uint8_t* gmask, int64_t idx_ld, const int32_t* count, int64_t B,
                          int G, int32_t* grows, int32_t* gcount, cudaStream_t s);
int launch_block_max_tc(const void* q, const float* w, const void* k, int64_t B, int64_t L, int G,
                        const int64_t* q_pos, float* scores, int64_t ld, cudaStream_t s);
int launch_msa_expand(const int32_t* kept, int64_t kept_ld, const int32_t* kcnt, int G, int block,
                      const int64_t* q_pos, int64_t B, int32_t* idx, uint8_t* gmask, int64_t idx_ld, int32_t* count,
                      cudaStream_t s);
int launch_shift_qpos(const int64_t* q_pos, int64_t B, int G, int64_t delta, int64_t* out, cudaStream_t s);
size_t sparse_attn_ws_bytes(int64_t B, int64_t kmax, int H);
int take_attn2_flags(int* check);
int take_msa_attn_flags(int* check);
int launch_msa_attn_rows(const void* q, const void* kv, int64_t L, const int32_t* idx, const uint8_t* gmask, int64_t ld,
                         const int32_t* count, int64_t B, int G, float scale, void* out, float* lse, cudaStream_t s);
}  // namespace lsa
