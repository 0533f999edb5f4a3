// Exact re-ranking of a coarse candidate set: bf16 index scores over the recalled positions, then the
// final top-K, unioned with the fixed sink / window positions.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）": a cheap first stage recalls
// candidates, the second stage runs the standard token-level indexer score (equation I_{t,s}) on the
// recalled tokens only and takes the final arg topK there.  Here the first stage is the FP8 indexer
// pass with top-K' (K' > K), and the second stage re-scores those K' positions from the bf16 index
// queries and keys, so the kept set matches the full-precision ranking.
#include "lsa_common.cuh"

namespace lsa {

int launch_topk_mode(const float* scores, int64_t ld, int64_t B, int64_t L, int K, int sink, int window,
                     const int64_t* q_pos, int mode, int div, int32_t* idx, int64_t idx_ld, int32_t* count,
                     int64_t kmax, cudaStream_t s);

namespace {

constexpr int RF_THREADS = 128;

struct Fixed {
  int nsink, wlo, whi;
};
__device__ __forceinline__ Fixed fixed_of(int64_t qp64, int sink, int window) {
  Fixed f;
  const int qp = static_cast<int>(qp64);
  f.nsink = min(sink, qp + 1);
  f.wlo = window > 0 ? max(qp - window + 1, f.nsink) : qp + 1;
  f.whi = qp + 1;
  return f;
}

// rescored[b, j] = I(q_b, k_{s_j}) for the j-th dynamic candidate s_j of query b (cand rows hold the
// sink entries first, then the dynamic candidates ascending, then the window entries).
// ndyn_m1[b] = (number of dynamic candidates) - 1, used as the candidate range of the next top-K.
template <int D>
__global__ void __launch_bounds__(RF_THREADS) k_rescore(const uint16_t* __restrict__ q, const float* __restrict__ w,
                                                        const uint16_t* __restrict__ k, int H_I, int64_t L,
                                                        const int32_t* __restrict__ cand, int64_t cand_ld,
                                                        const int32_t* __restrict__ cand_count,
                                                        const int64_t* __restrict__ q_pos, int sink, int window,
                                                        float* __restrict__ out, int64_t out_ld,
                                                        int64_t* __restrict__ ndyn_m1) {
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;
  float* ws = smem + H_I * D;
  const int b = blockIdx.y, tid = threadIdx.x;
  const int j = blockIdx.x * RF_THREADS + tid;
  const Fixed f = fixed_of(q_pos[b], sink, window);
  const int n = min(static_cast<int64_t>(cand_count[b]), cand_ld);
  int nfix = f.nsink + (f.whi - f.wlo);
  int ndyn = max(0, n - nfix);
  if (blockIdx.x == 0 && tid == 0) ndyn_m1[b] = static_cast<int64_t>(ndyn) - 1;
  for (int i = tid; i < H_I * D; i += RF_THREADS) qs[i] = bf16_bits_to_f32(q[static_cast<int64_t>(b) * H_I * D + i]);
  for (int i = tid; i < H_I; i += RF_THREADS) ws[i] = w[static_cast<int64_t>(b) * H_I + i];
  __syncthreads();
  if (j >= out_ld) return;
  float acc = -INFINITY;
  if (j < ndyn) {
    int64_t s = cand[static_cast<int64_t>(b) * cand_ld + f.nsink + j];
    s = s < 0 ? 0 : (s >= L ? L - 1 : s);
    float kr[D];
    const uint16_t* kp = k + s * D;
    #pragma unroll
    for (int d = 0; d < D; d += 8) {
      const uint4 raw = *reinterpret_cast<const uint4*>(kp + d);
      const uint32_t v4[4] = {raw.x, raw.y, raw.z, raw.w};
      #pragma unroll
      for (int t = 0; t < 4; ++t) {
        kr[d + 2 * t] = bf16_bits_to_f32(v4[t] & 0xFFFFu);
        kr[d + 2 * t + 1] = bf16_bits_to_f32(v4[t] >> 16);
      }
    }
    acc = 0.f;
    for (int h = 0; h < H_I; ++h) {
      const float* qh = qs + h * D;
      float dot = 0.f;
      #pragma unroll
      for (int d = 0; d < D; d += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(qh + d);
        dot = fmaf(qv.x, kr[d], dot);
        dot = fmaf(qv.y, kr[d + 1], dot);
        dot = fmaf(qv.z, kr[d + 2], dot);
        dot = fmaf(qv.w, kr[d + 3], dot);
      }
      acc = fmaf(ws[h], fmaxf(dot, 0.f), acc);
    }
  }
  out[static_cast<int64_t>(b) * out_ld + j] = acc;
}

// idx row = sink entries, then the kept dynamic candidates (ascending), then the window entries.
__global__ void __launch_bounds__(256) k_refine_assemble(const int32_t* __restrict__ cand, int64_t cand_ld,
                                                         const int32_t* __restrict__ cand_count,
                                                         const int32_t* __restrict__ kept, int64_t kept_ld,
                                                         const int32_t* __restrict__ kept_count,
                                                         const int64_t* __restrict__ q_pos, int sink, int window,
                                                         int32_t* __restrict__ idx, int64_t idx_ld,
                                                         int32_t* __restrict__ count, int kmax) {
  const int b = blockIdx.x, tid = threadIdx.x;
  const Fixed f = fixed_of(q_pos[b], sink, window);
  const int n = min(static_cast<int64_t>(cand_count[b]), cand_ld);
  const int nwin = f.whi - f.wlo;
  const int ndyn = max(0, n - f.nsink - nwin);
  const int nk = kept_count[b];
  const int32_t* crow = cand + static_cast<int64_t>(b) * cand_ld;
  int32_t* out = idx + static_cast<int64_t>(b) * idx_ld;
  for (int i = tid; i < f.nsink; i += 256) out[i] = crow[i];
  for (int i = tid; i < nk; i += 256) out[f.nsink + i] = crow[f.nsink + kept[static_cast<int64_t>(b) * kept_ld + i]];
  for (int i = tid; i < nwin; i += 256) out[f.nsink + nk + i] = crow[f.nsink + ndyn + i];
  const int total = f.nsink + nk + nwin;
  for (int i = total + tid; i < kmax; i += 256) out[i] = -1;
  if (tid == 0) count[b] = total;
}

void refine_ws_layout(int64_t B, int64_t cand_ld, int K, size_t* o_ndyn, size_t* o_kept, size_t* o_kcnt,
                      size_t* total, int64_t* out_ld) {
  *out_ld = (cand_ld + 3) / 4 * 4;
  size_t o = align_up(static_cast<size_t>(B) * static_cast<size_t>(*out_ld) * 4, 256);
  *o_ndyn = o;
  o = align_up(o + static_cast<size_t>(B) * 8, 256);
  *o_kept = o;
  o = align_up(o + static_cast<size_t>(B) * K * 4, 256);
  *o_kcnt = o;
  *total = align_up(o + static_cast<size_t>(B) * 4, 256);
}

}  // namespace

size_t refine_ws_bytes(int64_t B, int64_t cand_ld, int K) {
  size_t a, b, c, t;
  int64_t ld;
  refine_ws_layout(B, cand_ld, K, &a, &b, &c, &t, &ld);
  return t;
}

int launch_refine(const void* q, const float* w, const void* k, int64_t B, int H_I, int d_I, int64_t L,
                  const int32_t* cand, int64_t cand_ld, const int32_t* cand_count, int K, int sink, int window,
                  const int64_t* q_pos, int32_t* idx, int64_t idx_ld, int32_t* count, int64_t kmax, void* ws,
                  cudaStream_t s) {
  size_t o_ndyn, o_kept, o_kcnt, total;
  int64_t out_ld;
  refine_ws_layout(B, cand_ld, K, &o_ndyn, &o_kept, &o_kcnt, &total, &out_ld);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* rs = reinterpret_cast<float*>(base);
  int64_t* ndyn_m1 = reinterpret_cast<int64_t*>(base + o_ndyn);
  int32_t* kept = reinterpret_cast<int32_t*>(base + o_kept);
  int32_t* kcnt = reinterpret_cast<int32_t*>(base + o_kcnt);
  const dim3 grid(static_cast<unsigned>(cdiv(out_ld, RF_THREADS)), static_cast<unsigned>(B));
  const size_t smem = static_cast<size_t>(H_I) * d_I * 4 + static_cast<size_t>(H_I) * 4;
  const uint16_t* qq = static_cast<const uint16_t*>(q);
  const uint16_t* kk = static_cast<const uint16_t*>(k);
  switch (d_I) {
    case 32:
      k_rescore<32><<<grid, RF_THREADS, smem, s>>>(qq, w, kk, H_I, L, cand, cand_ld, cand_count, q_pos, sink, window,
                                                   rs, out_ld, ndyn_m1);
      break;
    case 64:
      k_rescore<64><<<grid, RF_THREADS, smem, s>>>(qq, w, kk, H_I, L, cand, cand_ld, cand_count, q_pos, sink, window,
                                                   rs, out_ld, ndyn_m1);
      break;
    case 128:
      LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_rescore<128>), 64 * 1024));
      k_rescore<128><<<grid, RF_THREADS, smem, s>>>(qq, w, kk, H_I, L, cand, cand_ld, cand_count, q_pos, sink,
                                                    window, rs, out_ld, ndyn_m1);
      break;
    default:
      return LSA_ERR_UNSUPPORTED;
  }
  LSA_CUDA_TRY(cudaGetLastError());
  // top-K among each row's dynamic candidates [0, ndyn): the candidate range is [0, ndyn_m1 + 1)
  int st = launch_topk_mode(rs, out_ld, B, out_ld, K, 0, 0, ndyn_m1, /*MODE_BLOCKS*/ 2, 1, kept, K, kcnt, K, s);
  if (st != LSA_OK) return st;
  k_refine_assemble<<<static_cast<unsigned>(B), 256, 0, s>>>(cand, cand_ld, cand_count, kept, K, kcnt, q_pos, sink,
                                                            window, idx, idx_ld, count, static_cast<int>(kmax));
  return cuda_status(cudaGetLastError());
}

}  // namespace lsa
