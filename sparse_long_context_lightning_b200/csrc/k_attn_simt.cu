// Sparse absorbed-MQA attention on CUDA cores (reference-quality kernel for small head counts).
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线": u_t = Attn(h_t, {c_s | s in S_t}), the MLA
// latent c_s shared by every head, value = first 512 dims.  One CTA per (query, 16 heads); the selected
// rows are gathered 32 at a time into shared memory and reduced with an online softmax in fp32.
#include "lsa_common.cuh"

namespace lsa {
namespace {

__device__ int g_attn_simt_check;  // set when a selected index was outside [0, L) (the row was clamped)

constexpr int AS_THREADS = 256;
constexpr int AS_HG = 16;
constexpr int AS_TILE = 32;
constexpr int AS_DQK = 576;
constexpr int AS_DV = 512;
constexpr int AS_STRIDE = 578;  // bf16 elements per staged row (odd word count: conflict-free)

__global__ void __launch_bounds__(AS_THREADS) k_attn_simt(const uint16_t* __restrict__ q,
                                                          const uint16_t* __restrict__ kv, int64_t L,
                                                          const int32_t* __restrict__ idx, int64_t idx_ld,
                                                          const int32_t* __restrict__ count, int H, float scale,
                                                          uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char dsm[];
  float* qs = reinterpret_cast<float*>(dsm);                                  // [16][576]
  uint16_t* kvs = reinterpret_cast<uint16_t*>(qs + AS_HG * AS_DQK);           // [32][578]
  float* ps = reinterpret_cast<float*>(kvs + AS_TILE * AS_STRIDE);            // [16][32]
  float* mrow = ps + AS_HG * AS_TILE;                                          // [16]
  float* lrow = mrow + AS_HG;                                                  // [16]
  float* arow = lrow + AS_HG;                                                  // [16]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y;
  const int h0 = blockIdx.x * AS_HG;
  const uint16_t* qb = q + (static_cast<int64_t>(b) * H + h0) * AS_DQK;
  for (int i = tid; i < AS_HG * AS_DQK; i += AS_THREADS) qs[i] = bf16_bits_to_f32(qb[i]) * scale;
  if (tid < AS_HG) {
    mrow[tid] = -INFINITY;
    lrow[tid] = 0.f;
  }
  const int hh = tid / 16, cc = tid % 16;
  float o[AS_DV / 16];
  #pragma unroll
  for (int i = 0; i < AS_DV / 16; ++i) o[i] = 0.f;
  const int n = min(static_cast<int64_t>(count[b]), idx_ld);
  const int32_t* rowidx = idx + static_cast<int64_t>(b) * idx_ld;
  __syncthreads();
  for (int t0 = 0; t0 < n; t0 += AS_TILE) {
    const int nt = min(AS_TILE, n - t0);
    for (int i = tid; i < nt * (AS_DQK / 8); i += AS_THREADS) {
      const int r = i / (AS_DQK / 8), c = i % (AS_DQK / 8);
      int64_t s = rowidx[t0 + r];
      if (s < 0 || s >= L) atomicExch(&g_attn_simt_check, 1);  // clamped below: the access stays in bounds
      s = s < 0 ? 0 : (s >= L ? L - 1 : s);
      const uint4 v = *reinterpret_cast<const uint4*>(kv + s * AS_DQK + c * 8);
      uint32_t* dst = reinterpret_cast<uint32_t*>(kvs + r * AS_STRIDE + c * 8);
      dst[0] = v.x;
      dst[1] = v.y;
      dst[2] = v.z;
      dst[3] = v.w;
    }
    __syncthreads();
    for (int p = tid; p < AS_HG * AS_TILE; p += AS_THREADS) {
      const int h = p / AS_TILE, r = p % AS_TILE;
      float dot = -INFINITY;
      if (r < nt) {
        const float* qh = qs + h * AS_DQK;
        const uint32_t* kr = reinterpret_cast<const uint32_t*>(kvs + r * AS_STRIDE);
        float acc = 0.f;
        for (int d = 0; d < AS_DQK / 2; ++d) {
          const uint32_t pr = kr[d];
          const float2 qv = *reinterpret_cast<const float2*>(qh + 2 * d);
          acc = fmaf(qv.x, bf16_bits_to_f32(pr & 0xFFFFu), acc);
          acc = fmaf(qv.y, bf16_bits_to_f32(pr >> 16), acc);
        }
        dot = acc;
      }
      ps[h * AS_TILE + r] = dot;
    }
    __syncthreads();
    for (int h = warp; h < AS_HG; h += AS_THREADS / 32) {
      const float x = ps[h * AS_TILE + lane];
      const float mx = warp_max(x);
      const float mold = mrow[h];
      const float mnew = fmaxf(mold, mx);
      const float p = lane < nt ? __expf(x - mnew) : 0.f;
      const float sum = warp_sum(p);
      ps[h * AS_TILE + lane] = p;
      __syncwarp();
      if (lane == 0) {
        const float alpha = mold == -INFINITY ? 0.f : __expf(mold - mnew);
        arow[h] = alpha;
        lrow[h] = lrow[h] * alpha + sum;
        mrow[h] = mnew;
      }
    }
    __syncthreads();
    {
      const float alpha = arow[hh];
      #pragma unroll
      for (int i = 0; i < AS_DV / 16; ++i) o[i] *= alpha;
      for (int r = 0; r < nt; ++r) {
        const float p = ps[hh * AS_TILE + r];
        const uint16_t* vr = kvs + r * AS_STRIDE + cc;
        #pragma unroll
        for (int i = 0; i < AS_DV / 16; ++i) o[i] = fmaf(p, bf16_bits_to_f32(vr[16 * i]), o[i]);
      }
    }
    __syncthreads();
  }
  const float l = lrow[hh];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint16_t* ob = out + (static_cast<int64_t>(b) * H + h0 + hh) * AS_DV;
  #pragma unroll
  for (int i = 0; i < AS_DV / 16; ++i) {
    const __nv_bfloat16 v = __float2bfloat16_rn(o[i] * inv);
    ob[cc + 16 * i] = *reinterpret_cast<const uint16_t*>(&v);
  }
  if (lse != nullptr && cc == 0) lse[static_cast<int64_t>(b) * H + h0 + hh] = l > 0.f ? mrow[hh] + logf(l) : -INFINITY;
}

}  // namespace

int launch_attn_simt(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                     const int32_t* count, int64_t B, int H, float scale, void* out, float* lse, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  const size_t smem = AS_HG * AS_DQK * 4 + AS_TILE * AS_STRIDE * 2 + AS_HG * AS_TILE * 4 + 3 * AS_HG * 4;
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_attn_simt), static_cast<int>(smem)));
  const dim3 grid(static_cast<unsigned>(H / AS_HG), static_cast<unsigned>(B));
  k_attn_simt<<<grid, AS_THREADS, smem, s>>>(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kv), L, idx,
                                            idx_ld, count, H, scale, static_cast<uint16_t*>(out), lse);
  return cuda_status(cudaGetLastError());
}

// The index-range flag, read and cleared (1: an index outside [0, L) was clamped since the last call; -1: CUDA
// error).
int take_attn_simt_check() {
  int c = 0;
  if (cudaMemcpyFromSymbol(&c, g_attn_simt_check, sizeof(int)) != cudaSuccess) return -1;
  const int zero = 0;
  if (c != 0 && cudaMemcpyToSymbol(g_attn_simt_check, &zero, sizeof(int)) != cudaSuccess) return -1;
  return c;
}

}  // namespace lsa
