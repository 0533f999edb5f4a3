// Per-query top-K selection (exact, never a full sort), with the sink / window union.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线": S_t = arg topK({I_{t,s}}_{s<=t}, K);
// section "机制一：流式感知索引（SI）/ 预算分解": the sink and the window are fixed, the top-K runs
// over the positions outside them, and the three sets are unioned.
//
// Design (B200): one thread-block cluster of C CTAs (C <= 16) per score row.  Each CTA owns a
// contiguous chunk of the row and, when it fits, keeps it in shared memory, so HBM is read once.
// The threshold is found by histogram refinement:
//   level 0  4096 linear value bins over [min, max] of the row's candidates,
//   level 1+ 4096-way radix digits of the order-preserving uint32 key inside the boundary bin,
// each level's per-CTA histograms summed across the cluster through distributed shared memory
// (DSMEM), until the boundary bin holds <= 1024 elements.  Those are gathered into CTA 0's shared
// memory and ranked exactly (score descending, position ascending).  A final ordered pass writes
// the selected positions in ascending order.  All cross-CTA synchronisation is the hardware
// cluster barrier: no spin-waits, no global atomics, no scratch memory.
#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;  // <= 32: per-warp arrays are reduced by one warp, lane < TK_WARPS
static_assert(TK_WARPS <= 32, "one warp reduces the per-warp partials");
constexpr int TK_BINS = 4096;
constexpr int TK_CAP = 1024;
constexpr int TK_MAXC = 16;

enum { MODE_TOKEN = 0, MODE_ALL = 1, MODE_BLOCKS = 2 };

struct TopkArgs {
  const float* scores;
  int64_t ld;
  int L;
  int K;
  int sink;
  int window;
  const int64_t* q_pos;
  int mode;  // MODE_TOKEN: visible [0,q_pos] minus sink/window; MODE_ALL: [0,L); MODE_BLOCKS: [0, min(L,(q_pos+1)/div))
  int div;
  int32_t* idx;
  int64_t idx_ld;
  int32_t* count;
  int kmax;
  int chunk;   // positions per CTA (multiple of 4)
  int cached;  // chunk kept in dynamic shared memory
};

struct TopkSmem {
  uint32_t hist[TK_BINS];
  uint32_t hred[TK_BINS];
  uint32_t coll_key[TK_CAP];
  uint32_t coll_pos[TK_CAP];
  uint32_t ncoll;
  uint32_t stot[TK_MAXC];
  float fmin[TK_MAXC];
  float fmax[TK_MAXC];
  uint32_t kmin[TK_MAXC];
  uint32_t kmax[TK_MAXC];
  uint32_t cgt[TK_MAXC];
  uint32_t ceq[TK_MAXC];
  uint32_t wa[TK_WARPS];
  uint32_t wb[TK_WARPS];
  uint32_t wc[TK_WARPS];
  float wf0[TK_WARPS];
  float wf1[TK_WARPS];
  // broadcast slots (written by the CTA that decides)
  uint32_t b_bin, b_above, b_count;
  uint32_t b_T, b_need_eq;
  uint64_t load_bar;
};

struct Row {
  const float* src;  // element s of the row is src[s - base]
  int base;
  __device__ __forceinline__ float val(int s) const { return src[s - base]; }
};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Block-wide sum of one uint32 per thread; every thread gets the total.
__device__ uint32_t block_sum_u32(uint32_t v, uint32_t* scratch) {
  v = warp_sum_u32(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  uint32_t t = lane < TK_WARPS ? scratch[lane] : 0u;
  t = warp_sum_u32(t);
  return t;
}

__global__ void __launch_bounds__(TK_THREADS, 2) k_topk_cluster(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char dyn[];
  __shared__ TopkSmem sm;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int r = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int64_t qp64 = a.q_pos[b];
  const int qp = static_cast<int>(qp64 < 0 ? -1 : (qp64 >= a.L ? a.L - 1 : qp64));
  int nsink = 0, clo = 0, chi = 0, wlo = 0, whi = 0;  // window = [wlo, whi)
  if (a.mode == MODE_TOKEN) {
    nsink = min(a.sink, qp + 1);
    clo = nsink;
    if (a.window > 0) {
      wlo = max(qp - a.window + 1, nsink);
      whi = qp + 1;
      chi = wlo;
    } else {
      wlo = whi = qp + 1;
      chi = qp + 1;
    }
  } else if (a.mode == MODE_ALL) {
    clo = 0;
    chi = a.L;
  } else {
    // q_pos is a token position here; the candidates are the complete visible blocks
    clo = 0;
    const int64_t nvis = qp64 < 0 ? 0 : (qp64 + 1) / a.div;
    chi = static_cast<int>(nvis < a.L ? nvis : a.L);
  }
  const int ncand = max(0, chi - clo);
  const int K = a.K;
  int32_t* out = a.idx + static_cast<int64_t>(b) * a.idx_ld;
  const int nwin = whi - wlo;
  const int nsel = min(K, ncand);
  const int total = nsink + nsel + nwin;

  // rank 0 writes the fixed positions, the padding and the count
  if (r == 0) {
    for (int i = tid; i < nsink; i += TK_THREADS) out[i] = i;
    for (int i = tid; i < nwin; i += TK_THREADS) out[nsink + nsel + i] = wlo + i;
    for (int i = total + tid; i < a.kmax; i += TK_THREADS) out[i] = -1;
    if (tid == 0) a.count[b] = total;
  }

  const int c0 = r * a.chunk;
  const int c1 = min(a.L, c0 + a.chunk);
  const int a0 = max(c0, clo), a1 = min(c1, chi);  // my candidates

  if (ncand <= K) {  // every candidate is selected (row-uniform branch: no cluster sync)
    for (int s = a0 + tid; s < a1; s += TK_THREADS) out[nsink + (s - clo)] = s;
    return;
  }

  // ---- stage the chunk -------------------------------------------------------------
  const float* grow = a.scores + static_cast<int64_t>(b) * a.ld;
  Row row;
  if (a.cached) {
    // one bulk asynchronous copy of the aligned part of the chunk, the last < 4 scores by plain loads
    float* cache = reinterpret_cast<float*>(dyn);
    const int lend = min(c1, chi);
    const int nvec = max(0, (lend - c0) / 4);
    if (tid == 0) {
      sm100::mbar_init(&sm.load_bar, 1);
      sm100::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
      if (nvec > 0) {
        sm100::mbar_expect_tx(&sm.load_bar, static_cast<uint32_t>(nvec) * 16u);
        sm100::bulk_load(cache, grow + c0, static_cast<uint32_t>(nvec) * 16u, &sm.load_bar);
      } else {
        sm100::mbar_arrive(&sm.load_bar);
      }
    }
    for (int s = c0 + nvec * 4 + tid; s < lend; s += TK_THREADS) cache[s - c0] = grow[s];
    // bounded wait (the copy is in bounds by construction); on give-up the row is left as the copy made it
    sm100::mbar_wait(&sm.load_bar, 0);
    row.src = cache;
    row.base = c0;
    __syncthreads();
  } else {
    row.src = grow;
    row.base = 0;
  }

  // ---- level 0 range: min / max of the candidates (non-finite values clamp into the end bins)
  {
    float lo = INFINITY, hi = -INFINITY;
    #pragma unroll 4
    for (int s = a0 + tid; s < a1; s += TK_THREADS) {
      const float x = row.val(s);
      if (isfinite(x)) {
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
    }
    lo = warp_min(lo);
    hi = warp_max(hi);
    if (lane == 0) {
      sm.wf0[warp] = lo;
      sm.wf1[warp] = hi;
    }
    __syncthreads();
    if (warp == 0) {
      lo = warp_min(lane < TK_WARPS ? sm.wf0[lane] : INFINITY);
      hi = warp_max(lane < TK_WARPS ? sm.wf1[lane] : -INFINITY);
      if (lane < C) {
        *cluster.map_shared_rank(&sm.fmin[r], lane) = lo;
        *cluster.map_shared_rank(&sm.fmax[r], lane) = hi;
      }
    }
    cluster.sync();
  }
  float gmin = INFINITY, gmax = -INFINITY;
  for (int c = 0; c < C; ++c) {
    gmin = fminf(gmin, sm.fmin[c]);
    gmax = fmaxf(gmax, sm.fmax[c]);
  }
  if (!(gmin <= gmax)) gmin = gmax = 0.f;  // no finite candidate at all
  const float inv = gmax > gmin ? static_cast<float>(TK_BINS) / (gmax - gmin) : 0.f;

  uint32_t need = static_cast<uint32_t>(K);
  uint32_t klo = 0, khi = 0xFFFFFFFFu;
  int shift = 0;
  bool resolved = false;  // threshold key known without collection (all remaining keys equal)
  uint32_t T = 0, need_eq = 0;

  for (int level = 0; level < 5; ++level) {
    // ---- histogram of this level ------------------------------------------------------
    for (int i = tid; i < TK_BINS; i += TK_THREADS) sm.hist[i] = 0;
    __syncthreads();
    #pragma unroll 4
    for (int s = a0 + tid; s < a1; s += TK_THREADS) {
      const float x = row.val(s);
      int bin;
      if (level == 0) {
        const float t = (x - gmin) * inv;
        bin = t >= static_cast<float>(TK_BINS - 1) ? TK_BINS - 1 : (t > 0.f ? static_cast<int>(t) : 0);
        if (x != x) bin = TK_BINS - 1;
      } else {
        const uint32_t k = f32_order_key(x);
        if (k < klo || k > khi) continue;
        bin = static_cast<int>((k - klo) >> shift);
      }
      atomicAdd(&sm.hist[bin], 1u);
    }
    cluster.sync();
    // ---- sum my slice of bins across the cluster ----------------------------------------
    const int per = TK_BINS / C;
    const int blo = r * per;
    uint32_t mysum = 0;
    for (int i = tid; i < per; i += TK_THREADS) {
      uint32_t t = 0;
      for (int c = 0; c < C; ++c) t += *cluster.map_shared_rank(&sm.hist[blo + i], c);
      sm.hred[i] = t;
      mysum += t;
    }
    mysum = block_sum_u32(mysum, sm.wa);
    if (tid < C) *cluster.map_shared_rank(&sm.stot[r], tid) = mysum;
    cluster.sync();
    // ---- the CTA whose slice holds the boundary picks the bin and broadcasts it -------------
    uint32_t above = 0;
    int bslice = 0;
    for (int c = C - 1; c >= 0; --c) {
      if (above + sm.stot[c] >= need) {
        bslice = c;
        break;
      }
      above += sm.stot[c];
    }
    if (r == bslice && warp == 0) {
      // scan my slice from the top: lane l owns bins [l*per/32, (l+1)*per/32)
      const int pl = per / 32;
      uint32_t lsum = 0;
      for (int i = 0; i < pl; ++i) lsum += sm.hred[lane * pl + i];
      // inclusive suffix sums over lanes (higher lanes hold higher bins)
      uint32_t suf = lsum;
      #pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      const uint32_t above_lane = above + suf - lsum;  // bins above my lane's range
      const bool mine = above_lane < need && above_lane + lsum >= need;
      if (mine) {
        uint32_t acc = above_lane;
        for (int i = pl - 1; i >= 0; --i) {
          const uint32_t h = sm.hred[lane * pl + i];
          if (acc + h >= need) {
            for (int c = 0; c < C; ++c) {
              *cluster.map_shared_rank(&sm.b_bin, c) = static_cast<uint32_t>(blo + lane * pl + i);
              *cluster.map_shared_rank(&sm.b_above, c) = acc;
              *cluster.map_shared_rank(&sm.b_count, c) = h;
            }
            break;
          }
          acc += h;
        }
      }
    }
    cluster.sync();
    const uint32_t bstar = sm.b_bin;
    need -= sm.b_above;
    const uint32_t bcount = sm.b_count;

    if (level > 0 && shift == 0) {  // the bin is a single key value: pure tie
      T = klo + bstar;
      need_eq = need;
      resolved = true;
      break;
    }
    if (bcount <= static_cast<uint32_t>(TK_CAP)) {
      // ---- gather the boundary bin into CTA 0 and rank it exactly ----------------------------
      if (r == 0 && tid == 0) sm.ncoll = 0;
      cluster.sync();
      uint32_t* rn = cluster.map_shared_rank(&sm.ncoll, 0);
      uint32_t* rk = cluster.map_shared_rank(&sm.coll_key[0], 0);
      uint32_t* rp = cluster.map_shared_rank(&sm.coll_pos[0], 0);
      #pragma unroll 4
      for (int s = a0 + tid; s < a1; s += TK_THREADS) {
        const float x = row.val(s);
        const uint32_t k = f32_order_key(x);
        bool in;
        if (level == 0) {
          const float t = (x - gmin) * inv;
          int bin = t >= static_cast<float>(TK_BINS - 1) ? TK_BINS - 1 : (t > 0.f ? static_cast<int>(t) : 0);
          if (x != x) bin = TK_BINS - 1;
          in = bin == static_cast<int>(bstar);
        } else {
          in = k >= klo && k <= khi && ((k - klo) >> shift) == bstar;
        }
        if (in) {
          const uint32_t slot = atomicAdd(rn, 1u);
          if (slot < static_cast<uint32_t>(TK_CAP)) {
            rk[slot] = k;
            rp[slot] = static_cast<uint32_t>(s);
          }
        }
      }
      cluster.sync();
      if (r == 0) {
        const uint32_t n = min(sm.ncoll, static_cast<uint32_t>(TK_CAP));
        for (uint32_t t = tid; t < n; t += TK_THREADS) {
          const uint32_t k = sm.coll_key[t], p = sm.coll_pos[t];
          uint32_t gt = 0, eqlow = 0;
          for (uint32_t j = 0; j < n; ++j) {
            const uint32_t kj = sm.coll_key[j];
            gt += kj > k;
            eqlow += (kj == k) & (sm.coll_pos[j] < p);
          }
          if (gt + eqlow == need - 1) {
            for (int c = 0; c < C; ++c) {
              *cluster.map_shared_rank(&sm.b_T, c) = k;
              *cluster.map_shared_rank(&sm.b_need_eq, c) = need - gt;
            }
          }
        }
      }
      cluster.sync();
      T = sm.b_T;
      need_eq = sm.b_need_eq;
      resolved = true;
      break;
    }
    // ---- refine: next level is a radix digit inside the boundary bin's key range ------------
    if (level == 0) {
      uint32_t lo = 0xFFFFFFFFu, hi = 0u;
      for (int s = a0 + tid; s < a1; s += TK_THREADS) {
        const float x = row.val(s);
        const float t = (x - gmin) * inv;
        int bin = t >= static_cast<float>(TK_BINS - 1) ? TK_BINS - 1 : (t > 0.f ? static_cast<int>(t) : 0);
        if (x != x) bin = TK_BINS - 1;
        if (bin == static_cast<int>(bstar)) {
          const uint32_t k = f32_order_key(x);
          lo = min(lo, k);
          hi = max(hi, k);
        }
      }
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      if (lane == 0) {
        sm.wa[warp] = lo;
        sm.wb[warp] = hi;
      }
      __syncthreads();
      if (warp == 0) {
        lo = lane < TK_WARPS ? sm.wa[lane] : 0xFFFFFFFFu;
        hi = lane < TK_WARPS ? sm.wb[lane] : 0u;
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (lane < C) {
          *cluster.map_shared_rank(&sm.kmin[r], lane) = lo;
          *cluster.map_shared_rank(&sm.kmax[r], lane) = hi;
        }
      }
      cluster.sync();
      klo = 0xFFFFFFFFu;
      khi = 0u;
      for (int c = 0; c < C; ++c) {
        klo = min(klo, sm.kmin[c]);
        khi = max(khi, sm.kmax[c]);
      }
    } else {
      const uint32_t nlo = klo + (bstar << shift);
      const uint64_t nhi = static_cast<uint64_t>(nlo) + ((1ull << shift) - 1ull);
      klo = nlo;
      khi = static_cast<uint32_t>(nhi < khi ? nhi : khi);
    }
    if (klo == khi) {
      T = klo;
      need_eq = need;
      resolved = true;
      break;
    }
    const uint32_t span = khi - klo;
    const int bits = 32 - __clz(span);
    shift = bits > 12 ? bits - 12 : 0;
  }
  (void)resolved;

  // ---- ordered compaction: selected = key > T, or key == T among the first need_eq of them ----
  const int n = max(0, a1 - a0);
  const int per_w = ((n + TK_WARPS - 1) / TK_WARPS + 127) & ~127;  // multiple of 128: 4 chunks per pass
  const int w0 = a0 + warp * per_w;
  const int w1 = min(a1, w0 + per_w);
  uint32_t gt_w = 0, eq_w = 0;
  for (int s0 = w0; s0 < w1; s0 += 128) {
    uint32_t k[4];
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0 + 32 * u + lane;
      k[u] = s < w1 ? f32_order_key(row.val(s)) : 0u;
    }
    #pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool in = s0 + 32 * u + lane < w1;
      gt_w += __popc(__ballot_sync(0xffffffffu, in && k[u] > T));
      eq_w += __popc(__ballot_sync(0xffffffffu, in && k[u] == T));
    }
  }
  if (lane == 0) {
    sm.wa[warp] = gt_w;
    sm.wb[warp] = eq_w;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t g = warp_sum_u32(lane < TK_WARPS ? sm.wa[lane] : 0u);
    const uint32_t e = warp_sum_u32(lane < TK_WARPS ? sm.wb[lane] : 0u);
    if (lane < C) {
      *cluster.map_shared_rank(&sm.cgt[r], lane) = g;
      *cluster.map_shared_rank(&sm.ceq[r], lane) = e;
    }
  }
  cluster.sync();
  uint32_t gt_before = 0, eq_before = 0;
  for (int c = 0; c < r; ++c) {
    gt_before += sm.cgt[c];
    eq_before += sm.ceq[c];
  }
  // exclusive gt / eq prefixes of my warp inside the CTA
  uint32_t gt_wbefore = 0, eq_wbefore = 0;
  for (int w = 0; w < warp; ++w) {
    gt_wbefore += sm.wa[w];
    eq_wbefore += sm.wb[w];
  }
  // a selected element's output slot = nsink + (#greater before it) + min(#equal before it, need_eq)
  {
    uint32_t run_gt = gt_before + gt_wbefore;
    uint32_t run_eq = eq_before + eq_wbefore;
    const uint32_t lim = static_cast<uint32_t>(nsink + nsel);
    for (int s00 = w0; s00 < w1; s00 += 128) {
     uint32_t kk[4];
     #pragma unroll
     for (int u = 0; u < 4; ++u) {
       const int s = s00 + 32 * u + lane;
       kk[u] = s < w1 ? f32_order_key(row.val(s)) : 0u;
     }
     #pragma unroll
     for (int u = 0; u < 4; ++u) {
      const int s = s00 + 32 * u + lane;
      const uint32_t k = kk[u];
      const bool is_gt = s < w1 && k > T;
      const bool is_eq = s < w1 && k == T;
      const uint32_t gtm = __ballot_sync(0xffffffffu, is_gt);
      const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
      const uint32_t lt = lanemask_lt();
      const uint32_t eq_before_me = run_eq + __popc(eqm & lt);
      const bool sel = is_gt || (is_eq && eq_before_me < need_eq);
      const uint32_t o = static_cast<uint32_t>(nsink) + run_gt + __popc(gtm & lt) + min(eq_before_me, need_eq);
      if (sel && o < lim) out[o] = s;  // bounded even if T were wrong
      run_gt += __popc(gtm);
      run_eq += __popc(eqm);
     }
    }
  }
  // keep this CTA's shared memory alive until every remote access of the cluster is done
  cluster.sync();
}

}  // namespace

int launch_topk_mode(const float* scores, int64_t ld, int64_t B, int64_t L, int K, int sink, int window,
                     const int64_t* q_pos, int mode, int div, int32_t* idx, int64_t idx_ld, int32_t* count,
                     int64_t kmax, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  // cluster size: smallest power of two whose chunk fits the shared-memory cache, <= 16
  const int64_t cache_elems = 20 * 1024;  // 80 KB of fp32 scores per CTA (two CTAs per SM)
  int C = 1;
  while (C < TK_MAXC && cdiv(L, C) > cache_elems) C *= 2;
  while (C < 8 && cdiv(L, C) > 16384) C *= 2;  // spread mid-size rows over more SMs
  int64_t chunk = (cdiv(L, C) + 3) / 4 * 4;
  const int cached = chunk <= cache_elems ? 1 : 0;
  if (chunk == 0) chunk = 4;
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.L = static_cast<int>(L);
  a.K = K;
  a.sink = sink;
  a.window = window;
  a.q_pos = q_pos;
  a.mode = mode;
  a.div = div;
  a.idx = idx;
  a.idx_ld = idx_ld;
  a.count = count;
  a.kmax = static_cast<int>(kmax);
  a.chunk = static_cast<int>(chunk);
  a.cached = cached;
  const size_t dyn = cached ? static_cast<size_t>(chunk) * 4 : 0;
  LSA_CUDA_TRY(cudaFuncSetAttribute(k_topk_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(cache_elems * 4)));
  LSA_CUDA_TRY(cudaFuncSetAttribute(k_topk_cluster, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, static_cast<unsigned>(B), 1);
  cfg.blockDim = dim3(TK_THREADS, 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LSA_CUDA_TRY(cudaLaunchKernelEx(&cfg, k_topk_cluster, a));
  return LSA_OK;
}

int launch_topk(const float* scores, int64_t ld, int64_t B, int64_t L, int K, int sink, int window,
                const int64_t* q_pos, int64_t, int32_t* idx, int64_t idx_ld, int32_t* count, int64_t kmax,
                cudaStream_t s) {
  return launch_topk_mode(scores, ld, B, L, K, sink, window, q_pos, MODE_TOKEN, 1, idx, idx_ld, count, kmax, s);
}

}  // namespace lsa
