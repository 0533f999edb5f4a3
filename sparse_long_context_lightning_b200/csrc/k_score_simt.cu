// Indexer-formula scoring on CUDA cores:  out[b, s] = kscale[s] * sum_j w'[b,j] * max(0, q[b,j,:] . k[s,:]).
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线", equation I_{t,s}.  Used for fp32
// representatives (Flat buckets / micro-blocks, where the keys are fp32 means) and for index shapes the
// tensor-core kernel does not tile (small H_I*B).  One thread owns one key row in registers; the queries
// of a block are staged one at a time in shared memory as fp32 (w' = w * q_scale folds the FP8 query
// scale; the FP8 key scale is applied after the head sum, which is exact math because scale > 0
// commutes with ReLU).
#include "lsa_common.cuh"

namespace lsa {
namespace {

enum { KT_BF16 = 0, KT_E4M3 = 1, KT_F32 = 2 };

constexpr int SC_THREADS = 128;
constexpr int SC_QB = 16;  // queries per block (looped)

template <int KT, int D>
__global__ void __launch_bounds__(SC_THREADS) k_score_simt(const void* __restrict__ q, int q_fp8,
                                                           const float* __restrict__ q_scale,
                                                           const float* __restrict__ w, const void* __restrict__ k,
                                                           const float* __restrict__ k_scale, int H_I, int64_t L,
                                                           int64_t B, const int64_t* __restrict__ q_pos,
                                                           float* __restrict__ out, int64_t ld) {
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;              // [H_I][D]
  float* wsum = smem + H_I * D;  // [H_I]
  const int tid = threadIdx.x;
  const int64_t s = static_cast<int64_t>(blockIdx.x) * SC_THREADS + tid;
  float kr[D];
  float ks = 1.f;
  if (s < L) {
    if (KT == KT_BF16) {
      const uint16_t* kp = static_cast<const uint16_t*>(k) + s * D;
      #pragma unroll
      for (int d = 0; d < D; d += 8) {
        const uint4 raw = *reinterpret_cast<const uint4*>(kp + d);
        kr[d + 0] = bf16_bits_to_f32(raw.x & 0xFFFFu);
        kr[d + 1] = bf16_bits_to_f32(raw.x >> 16);
        kr[d + 2] = bf16_bits_to_f32(raw.y & 0xFFFFu);
        kr[d + 3] = bf16_bits_to_f32(raw.y >> 16);
        kr[d + 4] = bf16_bits_to_f32(raw.z & 0xFFFFu);
        kr[d + 5] = bf16_bits_to_f32(raw.z >> 16);
        kr[d + 6] = bf16_bits_to_f32(raw.w & 0xFFFFu);
        kr[d + 7] = bf16_bits_to_f32(raw.w >> 16);
      }
    } else if (KT == KT_E4M3) {
      const uint8_t* kp = static_cast<const uint8_t*>(k) + s * D;
      #pragma unroll
      for (int d = 0; d < D; d += 16) {
        const uint4 raw = *reinterpret_cast<const uint4*>(kp + d);
        const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          #pragma unroll
          for (int j = 0; j < 4; ++j) kr[d + 4 * i + j] = e4m3_to_f32((wv[i] >> (8 * j)) & 0xFFu);
        }
      }
      ks = k_scale[s];
    } else {
      const float* kp = static_cast<const float*>(k) + s * D;
      #pragma unroll
      for (int d = 0; d < D; d += 4) {
        const float4 v = *reinterpret_cast<const float4*>(kp + d);
        kr[d] = v.x;
        kr[d + 1] = v.y;
        kr[d + 2] = v.z;
        kr[d + 3] = v.w;
      }
    }
  }
  const int64_t b0 = static_cast<int64_t>(blockIdx.y) * SC_QB;
  const int64_t b1 = b0 + SC_QB < B ? b0 + SC_QB : B;
  for (int64_t b = b0; b < b1; ++b) {
    __syncthreads();
    for (int i = tid; i < H_I * D; i += SC_THREADS) {
      const int64_t gi = b * H_I * D + i;
      qs[i] = q_fp8 ? e4m3_to_f32(static_cast<const uint8_t*>(q)[gi])
                    : bf16_bits_to_f32(static_cast<const uint16_t*>(q)[gi]);
    }
    for (int j = tid; j < H_I; j += SC_THREADS) wsum[j] = w[b * H_I + j] * (q_scale ? q_scale[b * H_I + j] : 1.f);
    __syncthreads();
    if (s >= L) continue;
    float acc;
    if (q_pos != nullptr && s > q_pos[b]) {
      acc = -INFINITY;
    } else {
      acc = 0.f;
      for (int j = 0; j < H_I; ++j) {
        const float* qj = qs + j * D;
        float dot = 0.f;
        #pragma unroll
        for (int d = 0; d < D; d += 4) {
          const float4 qv = *reinterpret_cast<const float4*>(qj + d);
          dot = fmaf(qv.x, kr[d], dot);
          dot = fmaf(qv.y, kr[d + 1], dot);
          dot = fmaf(qv.z, kr[d + 2], dot);
          dot = fmaf(qv.w, kr[d + 3], dot);
        }
        acc = fmaf(wsum[j], fmaxf(dot, 0.f), acc);
      }
      acc *= ks;
    }
    out[b * ld + s] = acc;
  }
}

template <int KT>
int launch_kt(const void* q, int q_fp8, const float* q_scale, const float* w, const void* k, const float* k_scale,
              int H_I, int d_I, int64_t L, int64_t B, const int64_t* q_pos, float* out, int64_t ld, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(cdiv(L, SC_THREADS)), static_cast<unsigned>(cdiv(B, SC_QB)));
  const size_t smem = static_cast<size_t>(H_I) * d_I * 4 + static_cast<size_t>(H_I) * 4;
  switch (d_I) {
    case 32:
      LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_score_simt<KT, 32>), 64 * 1024));
      k_score_simt<KT, 32><<<grid, SC_THREADS, smem, st>>>(q, q_fp8, q_scale, w, k, k_scale, H_I, L, B, q_pos, out, ld);
      break;
    case 64:
      LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_score_simt<KT, 64>), 64 * 1024));
      k_score_simt<KT, 64><<<grid, SC_THREADS, smem, st>>>(q, q_fp8, q_scale, w, k, k_scale, H_I, L, B, q_pos, out, ld);
      break;
    case 128:
      LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_score_simt<KT, 128>), 64 * 1024));
      k_score_simt<KT, 128><<<grid, SC_THREADS, smem, st>>>(q, q_fp8, q_scale, w, k, k_scale, H_I, L, B, q_pos, out, ld);
      break;
    default:
      return LSA_ERR_UNSUPPORTED;
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace

int launch_score_simt(const void* q, const float* q_scale, const float* w, const void* k, const float* k_scale,
                      int dtype, int64_t B, int H_I, int d_I, int64_t L, const int64_t* q_pos, float* scores,
                      int64_t ld, cudaStream_t s) {
  if (B == 0 || L == 0) return LSA_OK;
  if (dtype == LSA_BF16) return launch_kt<KT_BF16>(q, 0, nullptr, w, k, nullptr, H_I, d_I, L, B, q_pos, scores, ld, s);
  return launch_kt<KT_E4M3>(q, 1, q_scale, w, k, k_scale, H_I, d_I, L, B, q_pos, scores, ld, s);
}

int launch_centroid_score(const void* q, const float* w, const float* centroids, int64_t B, int H_I, int d_I,
                          int64_t NB, float* scores, int64_t ld, cudaStream_t s) {
  // every representative is ranked: no causal mask (q_pos = nullptr)
  if (B == 0 || NB == 0) return LSA_OK;
  return launch_kt<KT_F32>(q, 0, nullptr, w, centroids, nullptr, H_I, d_I, NB, B, nullptr, scores, ld, s);
}

}  // namespace lsa
