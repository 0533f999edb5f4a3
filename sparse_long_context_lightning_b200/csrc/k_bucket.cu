// Bucket / micro-block representatives and the expansion of kept buckets to token positions.
//
// "LSA 稀疏注意力會省顯存嗎", section 二 steps 2-4: each bucket keeps a representative vector and its
// member positions; Flat compares representatives, expands the kept buckets and adds sink + window.
// "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）": the representative is the
// mean of the members' index keys, computed once per sequence and cached.
// Lecture "从两本账看懂长上下文注意力", section "Qwen Sparse Attention" / "尾部计数与 query 自身": 4-token
// micro-blocks; the visible tokens of the incomplete tail block are added directly.
#include "lsa_common.cuh"

#include <algorithm>

namespace lsa {

int sm_count();

namespace {

// centroids[c, d] = sum_i k[m(c,i), d] / bsz, one thread per (bucket, 4 dims), members in order.
template <int DT>
__global__ void k_pool_keys(const void* __restrict__ kptr, const float* __restrict__ k_scale, int64_t L, int d_I,
                            const int32_t* __restrict__ members, int bsz, int64_t NB,
                            float* __restrict__ centroids) {
  const int groups = d_I / 4;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t c = t / groups;
  const int g = static_cast<int>(t % groups);
  if (c >= NB) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < bsz; ++i) {
    int64_t s = members ? static_cast<int64_t>(members[c * bsz + i]) : c * bsz + i;
    s = s < 0 ? 0 : (s >= L ? L - 1 : s);  // out-of-range members are clamped, never dereferenced
    float4 v;
    if (DT == LSA_BF16) {
      const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(kptr) + s * d_I + g * 4);
      v.x = bf16_bits_to_f32(raw.x & 0xFFFFu);
      v.y = bf16_bits_to_f32(raw.x >> 16);
      v.z = bf16_bits_to_f32(raw.y & 0xFFFFu);
      v.w = bf16_bits_to_f32(raw.y >> 16);
    } else {
      const uint32_t raw = *reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(kptr) + s * d_I + g * 4);
      const float sc = k_scale[s];
      v.x = e4m3_to_f32(raw & 0xFFu) * sc;
      v.y = e4m3_to_f32((raw >> 8) & 0xFFu) * sc;
      v.z = e4m3_to_f32((raw >> 16) & 0xFFu) * sc;
      v.w = e4m3_to_f32(raw >> 24) * sc;
    }
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const float n = static_cast<float>(bsz);
  acc.x /= n;
  acc.y /= n;
  acc.z /= n;
  acc.w /= n;
  reinterpret_cast<float4*>(centroids + c * d_I)[g] = acc;
}

constexpr int EX_THREADS = 1024;
constexpr int EX_MAX = 8192;

// One CTA per query: gather kept buckets' positions + tail + sink + window, bitonic sort, de-dup.
// E elements per thread (P = 1024 E slots, blocked: thread t holds slots [E t, E t + E)); the sorting
// network's compare-exchange stages run in registers (partner in the same thread), by warp shuffles
// (partner in the same warp) or through shared memory (two block barriers per stage) by partner distance.
template <int E>
__global__ void __launch_bounds__(EX_THREADS) k_bucket_expand(
    const int32_t* __restrict__ kept, int64_t kept_ld, const int32_t* __restrict__ kept_count,
    const int32_t* __restrict__ members, int bsz, int sink, int window, int tail_block,
    const int64_t* __restrict__ q_pos, int32_t* __restrict__ idx, int64_t idx_ld,
    int32_t* __restrict__ count, int kmax) {
  constexpr int P = EX_THREADS * E;
  __shared__ int32_t buf[P];
  __shared__ uint32_t wsum[EX_THREADS / 32];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qp = static_cast<int>(q_pos[b]);
  const int nk = min(kept_count[b], static_cast<int>(kept_ld));
  const int nmem = nk * bsz;
  const int nsink = min(sink, qp + 1);
  const int wlo = window > 0 ? max(0, qp - window + 1) : qp + 1;
  const int nwin = qp + 1 - wlo;
  const int tlo = tail_block > 0 ? ((qp + 1) / tail_block) * tail_block : qp + 1;
  const int ntail = qp + 1 - tlo;
  const int n = min(nmem + nsink + nwin + ntail, P);  // the host sizes P for the largest n
  // kept buckets, then their members: E independent loads per round trip
  int c[E], m[E];
  #pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = tid * E + e;
    c[e] = i < nmem ? kept[static_cast<int64_t>(b) * kept_ld + i / bsz] : 0;
  }
  #pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = tid * E + e;
    m[e] = (i < nmem && members) ? members[static_cast<int64_t>(c[e]) * bsz + (i % bsz)] : c[e] * bsz + (i % bsz);
  }
  int v[E];
  #pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = tid * E + e;
    int x = 0x7FFFFFFF;
    if (i < nmem) {
      x = m[e] <= qp ? m[e] : 0x7FFFFFFF;
    } else if (i < nmem + nsink) {
      x = i - nmem;
    } else if (i < nmem + nsink + nwin) {
      x = wlo + (i - nmem - nsink);
    } else if (i < n) {
      x = tlo + (i - nmem - nsink - nwin);
    }
    v[e] = x;
  }
  // bitonic sort, ascending: slot i meets slot i ^ j; the lower slot keeps the min when (i & k) == 0
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
        #pragma unroll
        for (int e = 0; e < E; ++e) {
          const int f = e ^ j;
          if (f > e) {
            const int i = tid * E + e;
            const bool asc = (i & k) == 0;
            const int x = v[e], y = v[f];
            if ((x > y) == asc) {
              v[e] = y;
              v[f] = x;
            }
          }
        }
      } else if (j < 32 * E) {
        const int tj = j / E;  // partner thread distance, < 32
        #pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const int y = __shfl_xor_sync(0xffffffffu, v[e], tj);
          const bool keep_min = ((i & j) == 0) == ((i & k) == 0);
          v[e] = keep_min ? min(v[e], y) : max(v[e], y);
        }
      } else {
        #pragma unroll
        for (int e = 0; e < E; ++e) buf[tid * E + e] = v[e];
        __syncthreads();
        #pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const int y = buf[i ^ j];
          const bool keep_min = ((i & j) == 0) == ((i & k) == 0);
          v[e] = keep_min ? min(v[e], y) : max(v[e], y);
        }
        __syncthreads();
      }
    }
  }
  // de-duplicate: a slot is kept if it is valid and differs from the slot before it
  const int prev_last = __shfl_up_sync(0xffffffffu, v[E - 1], 1);
  buf[tid] = v[E - 1];  // for lane 0: the last slot of the previous warp's last thread
  __syncthreads();
  int before = tid == 0 ? -1 : (lane == 0 ? buf[tid - 1] : prev_last);
  uint32_t mine = 0;
  #pragma unroll
  for (int e = 0; e < E; ++e) {
    mine += (v[e] != 0x7FFFFFFF) && (v[e] != before);
    before = v[e];
  }
  uint32_t incl = mine;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0, total = 0;
  for (int w = 0; w < EX_THREADS / 32; ++w) {
    const uint32_t x = wsum[w];
    wbase += w < warp ? x : 0u;
    total += x;
  }
  uint32_t o = wbase + incl - mine;
  int32_t* out = idx + static_cast<int64_t>(b) * idx_ld;
  before = tid == 0 ? -1 : (lane == 0 ? buf[tid - 1] : prev_last);
  #pragma unroll
  for (int e = 0; e < E; ++e) {
    if ((v[e] != 0x7FFFFFFF) && (v[e] != before) && o < static_cast<uint32_t>(kmax)) out[o++] = v[e];
    before = v[e];
  }
  for (int i = static_cast<int>(total) + tid; i < kmax; i += EX_THREADS) out[i] = -1;
  if (tid == 0) count[b] = static_cast<int32_t>(min(total, static_cast<uint32_t>(kmax)));
}

// out[p * n + i] (p = 0, 1, 2): bf16 parts of x[i] with x[i] = part0 + part1 + part2 exactly.  Each part is
// the round-to-nearest bf16 of what the earlier parts leave; the remainders are exact fp32 differences and
// shrink by 8 significand bits per part, so the third part holds the last 8 of fp32's 24 bits exactly.
__global__ void k_split_bf16x3(const float4* __restrict__ x, int64_t n4, uint2* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = x[i];
    const float e[4] = {v.x, v.y, v.z, v.w};
    uint32_t part[3][4];
    #pragma unroll
    for (int c = 0; c < 4; ++c) {
      float r = e[c];
      #pragma unroll
      for (int p = 0; p < 3; ++p) {
        const __nv_bfloat16 h = __float2bfloat16_rn(r);
        part[p][c] = static_cast<uint32_t>(__bfloat16_as_ushort(h));
        r -= __bfloat162float(h);
      }
    }
    #pragma unroll
    for (int p = 0; p < 3; ++p)
      out[p * n4 + i] = make_uint2(part[p][0] | (part[p][1] << 16), part[p][2] | (part[p][3] << 16));
  }
}

}  // namespace

int launch_pool_keys(const void* k, int dtype, const float* k_scale, int64_t L, int d_I, const int32_t* members,
                     int bsz, int64_t NB, float* centroids, cudaStream_t s) {
  if (NB == 0) return LSA_OK;
  const int64_t threads = NB * (d_I / 4);
  const int bs = 256;
  const int64_t grid = cdiv(threads, bs);
  if (dtype == LSA_BF16)
    k_pool_keys<LSA_BF16><<<static_cast<unsigned>(grid), bs, 0, s>>>(k, k_scale, L, d_I, members, bsz, NB, centroids);
  else
    k_pool_keys<LSA_FP8_E4M3><<<static_cast<unsigned>(grid), bs, 0, s>>>(k, k_scale, L, d_I, members, bsz, NB, centroids);
  return cuda_status(cudaGetLastError());
}

// fp32 [n] (n % 4 == 0, 16-byte aligned) -> bf16 [3, n]
int launch_split_bf16x3(const float* x, int64_t n, void* out, cudaStream_t s) {
  if (n == 0) return LSA_OK;
  const int64_t n4 = n / 4;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>(cdiv(n4, threads), static_cast<int64_t>(sm_count()) * 8);
  k_split_bf16x3<<<static_cast<unsigned>(blocks), threads, 0, s>>>(reinterpret_cast<const float4*>(x), n4,
                                                                   static_cast<uint2*>(out));
  return cuda_status(cudaGetLastError());
}

int launch_bucket_expand(const int32_t* kept, int64_t kept_ld, const int32_t* kept_count, const int32_t* members,
                         int bsz, int sink, int window, int tail_block, const int64_t* q_pos, int64_t B,
                         int32_t* idx, int64_t idx_ld, int32_t* count, int64_t kmax, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  // slots for the largest union: every kept bucket's members + sink + window + tail
  const int64_t nmax = kept_ld * bsz + sink + window + (tail_block > 0 ? tail_block - 1 : 0);
  if (nmax > EX_MAX) return LSA_ERR_INVALID_ARG;
  const dim3 grid(static_cast<unsigned>(B)), block(EX_THREADS);
  const int km = static_cast<int>(kmax);
  if (nmax <= 1024)
    k_bucket_expand<1><<<grid, block, 0, s>>>(kept, kept_ld, kept_count, members, bsz, sink, window, tail_block, q_pos,
                                              idx, idx_ld, count, km);
  else if (nmax <= 2048)
    k_bucket_expand<2><<<grid, block, 0, s>>>(kept, kept_ld, kept_count, members, bsz, sink, window, tail_block, q_pos,
                                              idx, idx_ld, count, km);
  else if (nmax <= 4096)
    k_bucket_expand<4><<<grid, block, 0, s>>>(kept, kept_ld, kept_count, members, bsz, sink, window, tail_block, q_pos,
                                              idx, idx_ld, count, km);
  else
    k_bucket_expand<8><<<grid, block, 0, s>>>(kept, kept_ld, kept_count, members, bsz, sink, window, tail_block, q_pos,
                                              idx, idx_ld, count, km);
  return cuda_status(cudaGetLastError());
}

}  // namespace lsa
