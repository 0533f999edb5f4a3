// Exact re-ranking of a coarse candidate set: bf16 index scores over the recalled positions, then the
// final top-K, unioned with the fixed sink / window positions.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）": a cheap first stage recalls
// candidates, the second stage runs the standard token-level indexer score (equation I_{t,s}) on the
// recalled tokens only and takes the final arg topK there.  Here the first stage is the FP8 indexer
// pass with top-K' (K' > K), and the second stage re-scores those K' positions from the bf16 index
// queries and keys, so the kept set matches the full-precision ranking.
#include "lsa_common.cuh"
#include "sm100.cuh"

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

// Tensor-core re-score for d_I = 128 and H_I in {32, 64}: the same I(q_b, k_s) as k_rescore, computed as
// D[cand, head] = K_cand . Q_b^T on tcgen05 (candidates = M, 128 per tile, on the TMEM lanes; heads = N;
// d_I = 128 = K, 8 MMAs of K = 16), with the ReLU / weight / head sum in the epilogue (one candidate per
// thread).  The candidates' key rows (256 B each) are gathered with 16-byte cp.async copies into the
// 128-byte-swizzled K-major layout; three stages, two TMEM accumulators.  CTA (split, b) handles the
// tiles split, split + nsplit, ... of query b.
constexpr int RT_THREADS = 288;  // warps 0-3 gather, warp 4 MMA (TMEM owner), warps 5-8 epilogue
constexpr int RT_STAGES = 3;
constexpr int RT_TILE = 128;
constexpr int RT_KB_BYTES = RT_TILE * 128;       // 16 KB: 64 dims of a tile
constexpr int RT_STAGE_BYTES = 2 * RT_KB_BYTES;  // 32 KB
constexpr int RT_Q_BYTES = 64 * 256;             // up to 64 heads x 128 dims bf16
constexpr int RT_SMEM = 1024 + RT_Q_BYTES + RT_STAGES * RT_STAGE_BYTES + 256;

__device__ int g_rescore_tc_timeout;

__global__ void __launch_bounds__(RT_THREADS, 2)
    k_rescore_tc(const uint16_t* __restrict__ q, const float* __restrict__ w, const uint16_t* __restrict__ k, int H_I,
                 int64_t L, const int32_t* __restrict__ cand, int64_t cand_ld, const int32_t* __restrict__ cand_count,
                 const int64_t* __restrict__ q_pos, int sink, int window, float* __restrict__ out, int64_t out_ld,
                 int64_t* __restrict__ ndyn_m1) {
  using namespace sm100;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = base;
  unsigned char* st_s = q_s + RT_Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(st_s + RT_STAGES * RT_STAGE_BYTES);
  uint64_t* kv_full = bars;                    // [RT_STAGES]
  uint64_t* kv_empty = kv_full + RT_STAGES;    // [RT_STAGES]
  uint64_t* acc_full = kv_empty + RT_STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* q_ready = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(q_ready + 1);
  __shared__ float w_s[64];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y, split = blockIdx.x, nsplit = gridDim.x;
  const Fixed f = fixed_of(q_pos[b], sink, window);
  const int n = min(static_cast<int64_t>(cand_count[b]), cand_ld);
  const int ndyn = max(0, n - f.nsink - (f.whi - f.wlo));
  if (split == 0 && tid == 0) ndyn_m1[b] = static_cast<int64_t>(ndyn) - 1;
  const int ntiles_all = static_cast<int>((out_ld + RT_TILE - 1) / RT_TILE);
  const int ntiles_act = (ndyn + RT_TILE - 1) / RT_TILE;
  // this CTA's active tiles: split, split + nsplit, ... below ntiles_act
  const int nmine = split < ntiles_act ? (ntiles_act - split + nsplit - 1) / nsplit : 0;
  const int32_t* crow = cand + static_cast<int64_t>(b) * cand_ld + f.nsink;
  float* orow = out + static_cast<int64_t>(b) * out_ld;

  if (tid == 0) {
    for (int i = 0; i < RT_STAGES; ++i) {
      mbar_init(&kv_full[i], 128);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(q_ready, 4);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_holder, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < 4) {
    // ---- gather: warp w copies rows 32w..32w+31 of a tile, 16 chunks of 16 B per row
    bool ok = true;
    for (int i = 0; ok && i < nmine; ++i) {
      const int t = split + i * nsplit, st = i % RT_STAGES;
      const int j = t * RT_TILE + warp * 32 + lane;
      int64_t s = j < ndyn ? crow[j] : 0;
      s = s < 0 ? 0 : (s >= L ? L - 1 : s);
      if (!mbar_spin(&kv_empty[st], ((i / RT_STAGES) & 1) ^ 1) || abort_flag) {
        ok = false;
        break;
      }
      unsigned char* dst = st_s + st * RT_STAGE_BYTES;
      #pragma unroll 4
      for (int q16 = lane; q16 < 32 * 16; q16 += 32) {
        const int rr = q16 >> 4, c = q16 & 15;  // row of the warp's 32, 16-byte chunk of the row
        const int row = warp * 32 + rr;
        const int64_t srow = __shfl_sync(0xffffffffu, s, rr);
        const int kb = c >> 3, c8 = c & 7;
        cp_async16(dst + kb * RT_KB_BYTES + row * 128 + ((c8 ^ (row & 7)) << 4), k + srow * 128 + c * 8);
      }
      cp_async_arrive_noinc(&kv_full[st]);
    }
    if (!ok && lane == 0) {
      atomicExch(&g_rescore_tc_timeout, 1);
      abort_flag = 1;
    }
  } else if (warp == 4) {
    // ---- MMA: D (128 candidates x H_I) = K_tile . Q^T, into accumulator i & 1
    if (lane == 0 && nmine > 0) {
      bool ok = mbar_spin(q_ready, 0);
      const uint32_t idesc = idesc_mma(128, H_I, 1u, 0u);
      const uint64_t qdesc = desc_sw128(smem_u32(q_s));
      for (int i = 0; ok && i < nmine; ++i) {
        const int st = i % RT_STAGES, ab = i & 1;
        if (!mbar_spin(&kv_full[st], (i / RT_STAGES) & 1) || !mbar_spin(&acc_empty[ab], ((i >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();
        tc_fence_after();
        const uint64_t kdesc = desc_sw128(smem_u32(st_s + st * RT_STAGE_BYTES));
        #pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + ab * 64, kdesc + ((kb * RT_KB_BYTES + kk * 32) >> 4),
                    qdesc + ((kb * H_I * 128 + kk * 32) >> 4), idesc, (kb | kk) != 0);
        }
        mma_commit(&kv_empty[st]);
        mma_commit(&acc_full[ab]);
      }
      if (!ok) {
        atomicExch(&g_rescore_tc_timeout, 1);
        abort_flag = 1;
      }
    }
  } else {
    // ---- epilogue warps: Q (H_I x 128, swizzled B tile) and the weights first, then one candidate per thread
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // candidate row of the tile = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int et = tid - 160;
    bool ok = true;
    if (nmine > 0) {
      for (int x = et; x < H_I * 16; x += 128) {
        const int h = x >> 4, c = x & 15, kb = c >> 3, c8 = c & 7;
        const uint4 v = *reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * H_I + h) * 128 + c * 8);
        *reinterpret_cast<uint4*>(q_s + kb * H_I * 128 + h * 128 + ((c8 ^ (h & 7)) << 4)) = v;
      }
      for (int x = et; x < H_I; x += 128) w_s[x] = w[static_cast<int64_t>(b) * H_I + x];
      fence_proxy_async_smem();  // generic stores read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
      ok = __all_sync(0xffffffffu, mbar_spin(q_ready, 0));  // the weights of every epilogue warp are visible
    }
    for (int i = 0; ok && i < nmine; ++i) {
      const int t = split + i * nsplit, ab = i & 1;
      // decided warp-wide: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_spin(&acc_full[ab], (i >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float acc = 0.f;
      for (int c0 = 0; c0 < H_I; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(trow + ab * 64 + c0, v);
        tmem_ld_wait();
        #pragma unroll
        for (int c = 0; c < 32; ++c) acc = fmaf(w_s[c0 + c], fmaxf(__uint_as_float(v[c]), 0.f), acc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      const int j = t * RT_TILE + row;
      if (j < out_ld) orow[j] = j < ndyn ? acc : -INFINITY;
    }
    if (!ok) {
      atomicExch(&g_rescore_tc_timeout, 1);
      abort_flag = 1;
    }
    // tiles of this CTA past the dynamic candidates: -inf
    for (int t = split + nmine * nsplit; t < ntiles_all; t += nsplit) {
      const int j = t * RT_TILE + row;
      if (j < out_ld) orow[j] = -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
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
  if (d_I == 128 && (H_I == 32 || H_I == 64) && B <= 65535) {
    // tensor cores; tiles of a query spread over up to ~2 waves of CTAs when the batch is small
    const int64_t tiles = cdiv(out_ld, RT_TILE);
    int64_t nsplit = (2 * 148 + B - 1) / B;
    if (nsplit > tiles) nsplit = tiles;
    if (nsplit < 1) nsplit = 1;
    LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_rescore_tc), RT_SMEM));
    k_rescore_tc<<<dim3(static_cast<unsigned>(nsplit), static_cast<unsigned>(B)), RT_THREADS, RT_SMEM, s>>>(
        qq, w, kk, H_I, L, cand, cand_ld, cand_count, q_pos, sink, window, rs, out_ld, ndyn_m1);
  } else switch (d_I) {
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

// The kernel's give-up flag, read and cleared (1: a bounded wait gave up since the last call; -1: CUDA error)
int take_rescore_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_rescore_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_rescore_tc_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace lsa
