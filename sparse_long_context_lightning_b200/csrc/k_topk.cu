// Per-query top-K selection (exact, never a full sort), with the sink / window union.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线": S_t = arg topK({I_{t,s}}_{s<=t}, K);
// section "机制一：流式感知索引（SI）/ 预算分解": the sink and the window are fixed, the top-K runs
// over the positions outside them, and the three sets are unioned.
//
// Design (B200): one thread-block cluster of C CTAs (C <= 16) per score row, two CTAs per SM.  Each CTA
// owns a contiguous chunk of the row and, when it fits (<= 16384 scores), keeps it in shared memory (one
// bulk asynchronous copy), so HBM is read once.  The threshold is found by refining the order-preserving
// uint32 key: level 0 histograms 256 bins over a key range that every CTA takes from the same fixed sample of
// the row (keys outside it are clamped into the end bins), each further level one 8-bit
// digit inside the boundary bin.  Per-CTA histograms are all-gathered through distributed shared memory
// (DSMEM), so every CTA finds the boundary bin itself (one cluster barrier per level).  When the
// boundary bin holds <= 1024 elements, its keys are all-gathered too and every CTA finishes the
// refinement locally; the tie shares and every CTA's output offset follow from the gathered counts, so
// the ordered write needs no further communication (it walks per-warp lists of the keys at or above the final
// boundary bin, built by the gather pass, when they fit).  Common case: two cluster barriers.  Each
// CTA runs this code once, so the passes are short rolled loops (a small instruction footprint) rather
// than unrolled code.  All synchronisation is the hardware cluster barrier: no spin-waits on memory, no
// global atomics, no scratch memory.
#include <mutex>

#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

constexpr int TK_THREADS = 1024;
constexpr int TK_WARPS = TK_THREADS / 32;  // <= 32: per-warp arrays are reduced by one warp, lane < TK_WARPS
static_assert(TK_WARPS <= 32, "one warp reduces the per-warp partials");
constexpr int TK_BINS = 256;   // one 8-bit digit of the order key per refinement level
constexpr int TK_CAP = 1024;   // boundary-bin size that is all-gathered and finished locally
constexpr int TK_MAXC = 16;    // cluster size limit (non-portable above 8)
constexpr int TK_CACHE = 24576;  // scores per CTA kept in shared memory (96 KB)
constexpr int TK_PIECES = 4;     // the chunk arrives in this many bulk copies; each warp waits for its own
constexpr int TK_UNROLL = 4;     // groups per lane whose loads are in flight together in a pass
constexpr int TK_WLIST = 64;     // per-warp list of the final pass's keys at or above the boundary bin (cached rows)

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
  int cached;  // chunk <= TK_CACHE: kept in dynamic shared memory
};

// Dynamic shared memory: hall[2][C][TK_BINS] (every CTA's histogram of a level, all-gathered, double
// buffered by level parity), then the cached chunk (scores, converted in place to order keys).
struct TopkSmem {
  uint32_t h[TK_BINS];     // this CTA's histogram of a level / the local refinement histogram
  uint32_t tot[TK_BINS];   // cluster-wide histogram of a level
  uint32_t cand[TK_CAP];   // boundary-bin keys; CTA c's at [segoff[c], segoff[c] + segcnt[c])
  uint8_t cand_w[TK_CAP];  // warp of each of this CTA's own boundary-bin elements (local slot order)
  uint32_t wl_key[TK_WARPS][TK_WLIST];  // cached rows: each warp's keys >= the final boundary bin's low end and
  int32_t wl_pos[TK_WARPS][TK_WLIST];   // their positions, in ascending position order
  uint32_t wl_over;                     // some warp's list overflowed: the ordered write walks the whole chunk
  uint32_t above[TK_MAXC];  // CTA c's elements above the boundary bins of all levels
  uint32_t segoff[TK_MAXC], segcnt[TK_MAXC];
  uint32_t gtb[TK_MAXC], eqb[TK_MAXC];  // CTA c's boundary elements with key > T / key == T
  uint32_t wa[TK_WARPS], wb[TK_WARPS];
  uint32_t wgt[TK_WARPS], weq[TK_WARPS];  // this CTA's elements with key > T / key == T, per warp
  uint32_t ccount;
  uint32_t sel_bin, sel_above, sel_count, sel_total;
  uint64_t load_bar[TK_PIECES];  // one per piece of the chunk's bulk copy
};

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Keys of valid elements are >= 1 (key 0, a negative-NaN pattern, is merged into key 1); key 0 marks a
// position outside this CTA's candidate range, so it is never counted or selected.
__device__ __forceinline__ uint32_t valid_key(float x) { return max(f32_order_key(x), 1u); }
__device__ __forceinline__ bool key_finite(uint32_t k) { return k > 0x007FFFFFu && k < 0xFF800000u; }

// The candidate range of row b, the fixed (sink / window) entries, the padding and the count.  CTA rank 0
// writes everything but the top-K part of the row.
struct RowSetup {
  int nsink, clo, chi, ncand, nsel;
  int32_t* out;
};
__device__ __forceinline__ RowSetup row_setup(const TopkArgs& a, int b, int r, int tid) {
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
  RowSetup rs;
  rs.nsink = nsink;
  rs.clo = clo;
  rs.chi = chi;
  rs.ncand = max(0, chi - clo);
  rs.nsel = a.K > 0 ? min(a.K, rs.ncand) : 0;
  rs.out = a.idx + static_cast<int64_t>(b) * a.idx_ld;
  const int nwin = whi - wlo;
  const int total = nsink + rs.nsel + nwin;
  if (r == 0) {
    for (int i = tid; i < nsink; i += TK_THREADS) rs.out[i] = i;
    for (int i = tid; i < nwin; i += TK_THREADS) rs.out[nsink + rs.nsel + i] = wlo + i;
    for (int i = total + tid; i < a.kmax; i += TK_THREADS) rs.out[i] = -1;
    if (tid == 0) a.count[b] = total;
  }
  return rs;
}

// This CTA's view of its chunk: groups of 4 consecutive positions starting at c0.  Group g holds
// positions c0 + 4g .. c0 + 4g + 3; an element is valid when its position is in [a0, a1).
struct Chunk {
  const float* grow;  // the score row in global memory
  bool vec;           // grow + c0 is 16-byte aligned
  const uint4* keys;  // the chunk's order keys in shared memory (0 = invalid), or nullptr
  int c0, a0, a1;
  __device__ __forceinline__ uint4 from_scores(int g, float4 v) const {
    const int s0 = c0 + 4 * g;
    uint4 k;
    if (s0 >= a0 && s0 + 4 <= a1) {
      k.x = valid_key(v.x);
      k.y = valid_key(v.y);
      k.z = valid_key(v.z);
      k.w = valid_key(v.w);
    } else {
      k.x = (s0 >= a0 && s0 < a1) ? valid_key(v.x) : 0u;
      k.y = (s0 + 1 >= a0 && s0 + 1 < a1) ? valid_key(v.y) : 0u;
      k.z = (s0 + 2 >= a0 && s0 + 2 < a1) ? valid_key(v.z) : 0u;
      k.w = (s0 + 3 >= a0 && s0 + 3 < a1) ? valid_key(v.w) : 0u;
    }
    return k;
  }
  // the group's scores straight from global memory (0 outside [a0, a1))
  __device__ __forceinline__ float4 gload(int g) const {
    const int s0 = c0 + 4 * g;
    // whole group in range of a 16-byte aligned row: one 16-byte load (chunks start at multiples of 4)
    if (vec && s0 >= a0 && s0 + 4 <= a1) return __ldg(reinterpret_cast<const float4*>(grow + s0));
    float4 v;
    v.x = (s0 >= a0 && s0 < a1) ? __ldg(grow + s0) : 0.f;
    v.y = (s0 + 1 >= a0 && s0 + 1 < a1) ? __ldg(grow + s0 + 1) : 0.f;
    v.z = (s0 + 2 >= a0 && s0 + 2 < a1) ? __ldg(grow + s0 + 2) : 0.f;
    v.w = (s0 + 3 >= a0 && s0 + 3 < a1) ? __ldg(grow + s0 + 3) : 0.f;
    return v;
  }
  __device__ __forceinline__ uint4 load(int g) const {
    if (keys) return keys[g];
    return from_scores(g, gload(g));
  }
  // groups g0 + 32u (u < TK_UNROLL) of one lane, all loads issued before any is used (a streamed chunk
  // comes from L2: one load in flight per thread would leave the pass latency-bound); 0 keys past gend
  __device__ __forceinline__ void load_batch(int g0, int gend, uint4 (&k)[TK_UNROLL]) const {
    if (keys) {
      #pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int g = g0 + 32 * u;
        k[u] = g < gend ? keys[g] : make_uint4(0u, 0u, 0u, 0u);
      }
    } else {
      float4 v[TK_UNROLL];
      #pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int g = g0 + 32 * u;
        v[u] = g < gend ? gload(g) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      #pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int g = g0 + 32 * u;
        k[u] = g < gend ? from_scores(g, v[u]) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
};

// f(keys of group g) for this lane's groups gw0 + lane, +32, ... < gw1: one at a time from the shared-memory
// cache, or TK_UNROLL at a time (loads in flight together) when the chunk is streamed from global memory.
template <bool STREAMED, class F>
__device__ __forceinline__ void for_groups(const Chunk& ch, int gw0, int gw1, int lane, F&& f) {
  if (!STREAMED) {
    for (int g = gw0 + lane; g < gw1; g += 32) f(ch.keys[g]);
  } else {
    for (int g0 = gw0 + lane; g0 < gw1; g0 += 32 * TK_UNROLL) {
      uint4 kb[TK_UNROLL];
      ch.load_batch(g0, gw1, kb);
      #pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u)
        if (g0 + 32 * u < gw1) f(kb[u]);
    }
  }
}

// Boundary bin of hist[] (bins ascend with the key): the bin holding the need-th largest element.
// Warp 0 only; lane l scans bins [8l, 8l + 8).  Writes sel_total, and sel_bin / sel_above / sel_count when the
// bins hold at least `need` elements.
__device__ __forceinline__ void find_boundary(TopkSmem& sm, const uint32_t* hist, uint32_t need, int lane) {
  const uint4 v0 = reinterpret_cast<const uint4*>(hist)[2 * lane];
  const uint4 v1 = reinterpret_cast<const uint4*>(hist)[2 * lane + 1];
  const uint32_t t[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  uint32_t lsum = 0;
  #pragma unroll
  for (int j = 0; j < 8; ++j) lsum += t[j];
  uint32_t suf = lsum;  // inclusive suffix sum over lanes (higher lanes hold higher bins)
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += v;
  }
  if (lane == 0) sm.sel_total = suf;  // every bin
  uint32_t acc = suf - lsum;  // elements in bins above this lane's range
  if (acc < need && acc + lsum >= need) {
    for (int j = 7; j >= 0; --j) {
      if (acc + t[j] >= need) {
        sm.sel_bin = static_cast<uint32_t>(lane * 8 + j);
        sm.sel_above = acc;
        sm.sel_count = t[j];
        break;
      }
      acc += t[j];
    }
  }
}

// Level geometry over [klo, khi]: 256 bins of width 2^shift.
__device__ __forceinline__ int level_shift(uint32_t klo, uint32_t khi) {
  const uint32_t span = khi - klo;
  const int bits = span ? 32 - __clz(span) : 0;
  return bits > 8 ? bits - 8 : 0;
}
// Key range [nlo, nhi] of bin `bin` of a level over [klo, khi].
__device__ __forceinline__ void bin_range(uint32_t klo, uint32_t khi, int shift, uint32_t bin, uint32_t& nlo,
                                          uint32_t& nhi) {
  nlo = klo + (bin << shift);
  const uint64_t hi64 = static_cast<uint64_t>(nlo) + ((uint64_t(1) << shift) - 1);
  nhi = static_cast<uint32_t>(hi64 < khi ? hi64 : khi);
}

// Warp-exclusive prefix and warp total of a per-lane count in [0, 7], from three ballots.
__device__ __forceinline__ uint32_t ballot_prefix(uint32_t v, uint32_t lt, uint32_t& total) {
  const uint32_t b0 = __ballot_sync(0xffffffffu, v & 1u);
  const uint32_t b1 = __ballot_sync(0xffffffffu, v & 2u);
  const uint32_t b2 = __ballot_sync(0xffffffffu, v & 4u);
  total = __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
  return __popc(b0 & lt) + 2u * __popc(b1 & lt) + 4u * __popc(b2 & lt);
}

// STREAMED: the chunk exceeds the shared-memory cache (a.cached == 0) and every pass reads it from global
// memory; otherwise it is cached (a.cached == 1).  Two instantiations keep the cached passes' code free of the
// streamed ones' load batching.
template <bool STREAMED>
__global__ void __launch_bounds__(TK_THREADS, 1) k_topk_cluster(TopkArgs a) {
  // every global access of this kernel comes after the previous kernel of the stream has completed
  sm100::pdl_wait();
  sm100::pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char dyn[];
  __shared__ __align__(16) TopkSmem sm;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int r = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cluster_arrive_relaxed();  // the matching wait comes before the first DSMEM access
  uint32_t* hall = reinterpret_cast<uint32_t*>(dyn);  // [2][C][TK_BINS]

  const RowSetup rs = row_setup(a, b, r, tid);
  const int K = a.K;
  const int c0 = r * a.chunk;
  const int c1 = min(a.L, c0 + a.chunk);
  const int a0 = max(c0, rs.clo), a1 = min(c1, rs.chi);  // my candidates
  if (rs.ncand <= K || K <= 0) {  // every candidate, or none, is selected (row-uniform branch)
    if (K > 0)
      for (int s = a0 + tid; s < a1; s += TK_THREADS) rs.out[rs.nsink + (s - rs.clo)] = s;
    cluster_wait();
    return;
  }
  // this thread's sample of the row for level 0's key range (below), loaded before the chunk is staged
  const uint32_t ksample =
      valid_key(__ldg(a.scores + static_cast<int64_t>(b) * a.ld + rs.clo + static_cast<int64_t>(tid) * rs.ncand / TK_THREADS));
  if (tid < TK_MAXC) sm.above[tid] = 0;
  if (tid == 0) sm.wl_over = 0;
  if (tid < TK_WARPS) {
    sm.wgt[tid] = 0;
    sm.weq[tid] = 0;
  }

  // ---- stage the chunk ----
  Chunk ch;
  ch.grow = a.scores + static_cast<int64_t>(b) * a.ld;
  ch.keys = nullptr;
  ch.vec = (reinterpret_cast<uintptr_t>(ch.grow + c0) & 15u) == 0;
  ch.c0 = c0;
  ch.a0 = a0;
  ch.a1 = a1;
  const int ng = a1 > a0 ? (a1 - c0 + 3) / 4 : 0;  // groups [g_lo, ng) hold my candidates
  const int g_lo = a1 > a0 ? (a0 - c0) / 4 : 0;
  float4* cache = reinterpret_cast<float4*>(dyn + static_cast<size_t>(2 * C * TK_BINS) * 4);
  // warp w walks groups [gw0, gw1); lane l takes every 32nd group from gw0 + l
  const int per_w = (ng - g_lo + TK_WARPS - 1) / TK_WARPS;
  const int gw0 = g_lo + warp * per_w;
  const int gw1 = min(ng, gw0 + per_w);
  // Cached rows: groups [g_lo, nvec) arrive in TK_PIECES bulk copies of pg groups (16-byte aligned rows
  // only); the rest -- a ragged last group, or every group of an unaligned row -- is read from global
  // memory by the thread that converts it.  Each warp waits for the pieces its groups lie in, so every
  // copy is waited for before the CTA can exit.
  int nvec = 0, pg = 1;
  if (a.cached) {
    const bool aligned = (reinterpret_cast<uintptr_t>(ch.grow + c0) & 15u) == 0;
    nvec = (aligned && ng > g_lo) ? (a1 - c0) / 4 : 0;
    const int npv = max(0, nvec - g_lo);
    pg = max(1, (npv + TK_PIECES - 1) / TK_PIECES);
    if (tid == 0) {
      for (int p = 0; p < TK_PIECES; ++p) sm100::mbar_init(&sm.load_bar[p], 1);
      sm100::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
      for (int p = 0; p < TK_PIECES; ++p) {
        const int p0 = g_lo + p * pg, p1 = min(nvec, p0 + pg);
        if (p1 > p0) {
          sm100::mbar_expect_tx(&sm.load_bar[p], static_cast<uint32_t>(p1 - p0) * 16u);
          sm100::bulk_load(cache + p0, ch.grow + c0 + 4 * p0, static_cast<uint32_t>(p1 - p0) * 16u, &sm.load_bar[p]);
        } else {
          sm100::mbar_arrive(&sm.load_bar[p]);
        }
      }
    }
    if (gw1 > gw0 && gw0 < nvec) {
      // bounded waits (the copies are in bounds by construction)
      const int plast = (min(gw1, nvec) - 1 - g_lo) / pg;
      for (int p = (gw0 - g_lo) / pg; p <= plast; ++p) sm100::mbar_wait(&sm.load_bar[p], 0);
    }
  }

  // ---- level 0's key range, from a fixed sample of the candidates that every CTA of the cluster reads alike:
  // all CTAs use the same bins without exchanging anything, and keys outside the sampled range are clamped into
  // the end bins (the counts stay exact; only the bins' widths depend on the sample) ----
  uint32_t klo = 0xFFFFFFFFu, khi = 0u, tau = 0u;
  {
    // sample tid is candidate clo + tid ncand / TK_THREADS (ncand > K >= 1 here)
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    if (key_finite(ksample)) {
      lo = ksample;
      hi = ksample;
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
    lo = lane < TK_WARPS ? sm.wa[lane] : 0xFFFFFFFFu;
    hi = lane < TK_WARPS ? sm.wb[lane] : 0u;
    // the smallest of the warps' sample maxima (each the largest of 32 samples: about the 97th percentile, so
    // their minimum sits near the 90th): level 0 counts only the keys at or above it
    uint32_t cut = (lane < TK_WARPS && hi != 0u) ? hi : 0xFFFFFFFFu;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      cut = min(cut, __shfl_xor_sync(0xffffffffu, cut, o));
    }
    klo = lo;
    khi = hi;
    tau = cut;
  }
  if (klo > khi) klo = khi = tau = 0x80000000u;  // no finite sample: every key is clamped into one bin

  // ---- cluster-level refinement: each level histograms one 8-bit digit of (key - klo) in [klo, khi] ----
  // Level 0 covers every valid key: keys outside the finite range are clamped to it, so the first bin's
  // range extends down to key 1 and the last occupied bin's range up to 0xFFFFFFFF.
  uint32_t need = static_cast<uint32_t>(K);
  uint32_t T = 0, need_eq = 0;
  bool gathered = false;
  // mode 0 (the first level): bins over [tau, khi], keys below tau not counted, keys above khi in the top bin;
  // mode 1 (only when fewer than `need` keys reach tau): bins over [klo, khi] with keys outside clamped into the end
  // bins, on the next level's buffers; mode 2: bins over the previous boundary bin, exactly
  const uint32_t klo_all = klo;
  int mode = 0;
  klo = tau;
  for (int level = 0; level < 8; ++level) {
    const int shift = level_shift(klo, khi);
    const uint32_t bmax = (khi - klo) >> shift;  // last occupied bin, <= 255
    uint32_t* hl = hall + (level & 1) * C * TK_BINS;
    if (tid < TK_BINS) sm.h[tid] = 0;
    __syncthreads();
    auto count_keys = [&](const uint4 k4) {
      const uint32_t k[4] = {k4.x, k4.y, k4.z, k4.w};
      #pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (mode == 0) {
          if (k[e] >= klo) atomicAdd(&sm.h[(min(k[e], khi) - klo) >> shift], 1u);
        } else if (mode == 1) {
          if (k[e]) atomicAdd(&sm.h[(min(max(k[e], klo), khi) - klo) >> shift], 1u);
        } else if (k[e] >= klo && k[e] <= khi) {
          atomicAdd(&sm.h[(k[e] - klo) >> shift], 1u);
        }
      }
    };
    if (level == 0 && a.cached) {
      // the scores of my groups become order keys in place (each thread reads back only its own groups)
      for (int g = gw0 + lane; g < gw1; g += 32) {
        const uint4 k = ch.from_scores(g, g < nvec ? cache[g] : ch.gload(g));
        reinterpret_cast<uint4*>(cache)[g] = k;
        count_keys(k);
      }
      ch.keys = reinterpret_cast<const uint4*>(cache);
    } else {
      for_groups<STREAMED>(ch, gw0, gw1, lane, count_keys);
    }
    __syncthreads();
    if (level == 0) cluster_wait();  // every CTA of the cluster has started: DSMEM is addressable
    for (int i = tid; i < TK_BINS * C; i += TK_THREADS) {
      const int c = i / TK_BINS, bin = i - c * TK_BINS;
      *cluster.map_shared_rank(hl + r * TK_BINS + bin, c) = sm.h[bin];
    }
    cluster.sync();
    if (tid < TK_BINS) {
      uint32_t v = 0;
      for (int c = 0; c < C; ++c) v += hl[c * TK_BINS + tid];
      sm.tot[tid] = v;
    }
    __syncthreads();
    if (warp == 0) find_boundary(sm, sm.tot, need, lane);
    __syncthreads();
    if (mode == 0 && sm.sel_total < need) {  // fewer than `need` keys reach tau (row-uniform): all keys, clamped
      mode = 1;
      klo = klo_all;
      continue;
    }
    const uint32_t bstar = sm.sel_bin, bcount = sm.sel_count;
    need -= sm.sel_above;
    if (warp < C) {  // CTA `warp`'s elements above the boundary bin
      uint32_t v = 0;
      for (int j = 0; j < 8; ++j) {
        const uint32_t bin = static_cast<uint32_t>(lane * 8 + j);
        v += bin > bstar ? hl[warp * TK_BINS + bin] : 0u;
      }
      v = warp_sum_u32(v);
      if (lane == 0) sm.above[warp] += v;
    }
    uint32_t nlo, nhi;
    bin_range(klo, khi, shift, bstar, nlo, nhi);
    if (mode == 1 && bstar == 0) nlo = 1u;  // valid keys are >= 1
    if (mode != 2 && bstar == bmax) nhi = 0xFFFFFFFFu;
    mode = 2;
    const bool tie = nlo == nhi;  // the boundary bin is one key value
    const bool gather = !tie && bcount <= static_cast<uint32_t>(TK_CAP);
    if (!tie && !gather) {
      klo = nlo;
      khi = nhi;
      continue;
    }
    // ---- final level: per-warp counts above the bin; the bin's elements gathered (or, for a one-key
    // bin, counted as ties) ----
    if (gather) {
      if (tid < C) {
        uint32_t o = 0;
        for (int c = 0; c < tid; ++c) o += hl[c * TK_BINS + bstar];
        sm.segoff[tid] = o;
        sm.segcnt[tid] = hl[tid * TK_BINS + bstar];
      }
      if (tid == 0) sm.ccount = 0;
      __syncthreads();
    }
    const uint32_t off = gather ? sm.segoff[r] : 0u;
    uint32_t nab = 0, nin = 0;
    auto final_keys = [&](const uint4 k4) {
      const uint32_t k[4] = {k4.x, k4.y, k4.z, k4.w};
      #pragma unroll
      for (int e = 0; e < 4; ++e) {
        nab += k[e] > nhi;
        if (k[e] >= nlo && k[e] <= nhi) {
          if (gather) {
            const uint32_t slot = atomicAdd(&sm.ccount, 1u);
            sm.cand[off + slot] = k[e];
            sm.cand_w[slot] = static_cast<uint8_t>(warp);
          } else {
            ++nin;
          }
        }
      }
    };
    if (!STREAMED) {
      // warp-uniform steps of 32 groups; the keys >= nlo (every key the write can select: T >= nlo) also go to
      // the warp's list, ordered by a ballot prefix, so that the ordered write needs only the lists
      const uint32_t lt = lanemask_lt();
      uint32_t wn = 0;
      for (int g0 = gw0; g0 < gw1; g0 += 32) {
        const int g = g0 + lane;
        const uint4 k4 = g < gw1 ? ch.keys[g] : make_uint4(0u, 0u, 0u, 0u);
        final_keys(k4);
        const uint32_t k[4] = {k4.x, k4.y, k4.z, k4.w};
        uint32_t c = 0;
        #pragma unroll
        for (int e = 0; e < 4; ++e) c += k[e] >= nlo;  // nlo >= 1: invalid slots (key 0) never count
        uint32_t tot;
        uint32_t o = wn + ballot_prefix(c, lt, tot);
        if (wn + tot <= static_cast<uint32_t>(TK_WLIST)) {
          #pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (k[e] >= nlo) {
              sm.wl_key[warp][o] = k[e];
              sm.wl_pos[warp][o] = c0 + 4 * g + e;
              ++o;
            }
          }
        }
        wn += tot;
      }
      if (wn > static_cast<uint32_t>(TK_WLIST) && lane == 0) sm.wl_over = 1u;
      if (lane == 0) sm.wa[warp] = wn;  // this warp's list length (sm.wa is free after the sampled range)
    } else {
      for_groups<STREAMED>(ch, gw0, gw1, lane, final_keys);
    }
    nab = warp_sum_u32(nab);
    nin = warp_sum_u32(nin);
    if (lane == 0) {
      sm.wgt[warp] = nab;  // gathered elements above T are added after the local refinement
      sm.weq[warp] = nin;
    }
    if (tie) {
      T = nlo;
      need_eq = need;
      if (tid < C) {
        sm.gtb[tid] = 0;
        sm.eqb[tid] = hl[tid * TK_BINS + bstar];
      }
    } else {
      if (tid < TK_BINS) {  // both local refinement histograms start empty
        sm.h[tid] = 0;
        sm.tot[tid] = 0;
      }
      __syncthreads();
      const uint32_t mine = sm.segcnt[r];
      for (uint32_t i = tid; i < mine * static_cast<uint32_t>(C); i += TK_THREADS) {
        const uint32_t c = i / mine, j = off + (i - c * mine);
        if (static_cast<int>(c) != r) *cluster.map_shared_rank(&sm.cand[j], static_cast<int>(c)) = sm.cand[j];
      }
      cluster.sync();  // last cluster barrier of this path: no DSMEM access after it
      klo = nlo;
      khi = nhi;
      gathered = true;
    }
    break;
  }

  if (gathered) {
    // ---- local refinement of the gathered boundary bin, redundantly in every CTA: one key per thread
    // (the bin holds <= TK_CAP == TK_THREADS keys); the two histograms alternate by level, so the one
    // for the next level is cleared while warp 0 scans this one: two block barriers per level ----
    static_assert(TK_CAP <= TK_THREADS, "one gathered key per thread");
    const uint32_t n = sm.sel_count;
    const uint32_t key = static_cast<uint32_t>(tid) < n ? sm.cand[tid] : 0u;
    for (int lv = 0; lv < 6; ++lv) {
      const int shift = level_shift(klo, khi);
      uint32_t* hcur = (lv & 1) ? sm.tot : sm.h;
      uint32_t* hnext = (lv & 1) ? sm.h : sm.tot;
      if (static_cast<uint32_t>(tid) < n && key >= klo && key <= khi) atomicAdd(&hcur[(key - klo) >> shift], 1u);
      __syncthreads();
      if (warp == 0) {
        find_boundary(sm, hcur, need, lane);
      } else if (tid < TK_BINS + 32) {
        hnext[tid - 32] = 0u;  // scanned by the previous level, which ended at a barrier
      }
      __syncthreads();
      need -= sm.sel_above;
      uint32_t nlo, nhi;
      bin_range(klo, khi, shift, sm.sel_bin, nlo, nhi);
      klo = nlo;
      khi = nhi;
      if (nlo == nhi) break;  // reached at shift 0 at the latest
    }
    T = klo;
    need_eq = need;
    if (warp < C) {  // CTA `warp`'s boundary elements above / at T
      const uint32_t o = sm.segoff[warp], m = sm.segcnt[warp];
      uint32_t g = 0, e = 0;
      for (uint32_t j = lane; j < m; j += 32) {
        const uint32_t k = sm.cand[o + j];
        g += k > T;
        e += k == T;
      }
      g = warp_sum_u32(g);
      e = warp_sum_u32(e);
      if (lane == 0) {
        sm.gtb[warp] = g;
        sm.eqb[warp] = e;
      }
    }
    // my own boundary elements, attributed to the warps that hold them
    const uint32_t off = sm.segoff[r], mine = sm.segcnt[r];
    for (uint32_t j = tid; j < mine; j += TK_THREADS) {
      const uint32_t k = sm.cand[off + j];
      if (k > T) atomicAdd(&sm.wgt[sm.cand_w[j]], 1u);
      if (k == T) atomicAdd(&sm.weq[sm.cand_w[j]], 1u);
    }
  }
  __syncthreads();

  // ---- this CTA's output offset and its share of the ties (ties go to the lowest positions) ----
  uint32_t base = static_cast<uint32_t>(rs.nsink), eq_seen = 0, take = 0;
  for (int c = 0; c <= r; ++c) {
    const uint32_t tk = min(need_eq - min(eq_seen, need_eq), sm.eqb[c]);
    if (c == r) {
      take = tk;
    } else {
      base += sm.above[c] + sm.gtb[c] + tk;
    }
    eq_seen += sm.eqb[c];
  }
  uint32_t gt_run = 0, eq_run = 0;  // this CTA's elements > T / == T in the warps before mine
  for (int w = 0; w < warp; ++w) {
    gt_run += sm.wgt[w];
    eq_run += sm.weq[w];
  }

  // ---- ordered write: a selected element's slot = base + (#gt before it) + min(#eq before it, take) ----
  const uint32_t lim = static_cast<uint32_t>(rs.nsink + rs.nsel);
  const uint32_t lt = lanemask_lt();
  // one warp-wide step: groups g = (step base) + lane, warp-uniform control flow (ballots)
  auto step = [&](const int g, const uint4 k4) {
    const uint32_t k[4] = {k4.x, k4.y, k4.z, k4.w};
    uint32_t ngt = 0, neq = 0;
    #pragma unroll
    for (int e = 0; e < 4; ++e) {
      ngt += k[e] > T;
      neq += k[e] == T;
    }
    uint32_t gtot, etot = 0, epre = 0;
    const uint32_t gpre = ballot_prefix(ngt, lt, gtot);
    if (__any_sync(0xffffffffu, neq != 0)) epre = ballot_prefix(neq, lt, etot);
    if (etot == 0u) {  // no ties in this step of the warp (the common case): gt elements only
      if (ngt) {
        uint32_t o = base + gt_run + gpre + min(eq_run, take);
        const int s0 = c0 + 4 * g;
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (k[e] > T) {
            if (o < lim) rs.out[o] = s0 + e;  // bounded even if the counts were inconsistent
            ++o;
          }
        }
      }
    } else if (ngt | neq) {
      uint32_t gb = gt_run + gpre, eb = eq_run + epre;
      const int s0 = c0 + 4 * g;
      #pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool gt = k[e] > T, eq = k[e] == T;
        if (gt || (eq && eb < take)) {
          const uint32_t o = base + gb + min(eb, take);
          if (o < lim) rs.out[o] = s0 + e;
        }
        gb += gt;
        eb += eq;
      }
    }
    gt_run += gtot;
    eq_run += etot;
  };
  if (!STREAMED && sm.wl_over == 0u) {
    // the warp's list holds every key it can select, in position order: one key per lane per step
    const int n = static_cast<int>(sm.wa[warp]);
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t k = i < n ? sm.wl_key[warp][i] : 0u;
      const bool gt = k > T, eq = k == T;
      const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
      const uint32_t gb = gt_run + __popc(bg & lt), eb = eq_run + __popc(be & lt);
      if (gt || (eq && eb < take)) {
        const uint32_t o = base + gb + min(eb, take);
        if (o < lim) rs.out[o] = sm.wl_pos[warp][i];  // bounded even if the counts were inconsistent
      }
      gt_run += __popc(bg);
      eq_run += __popc(be);
    }
  } else if (!STREAMED) {
    for (int g0 = gw0; g0 < gw1; g0 += 32) {
      const int g = g0 + lane;
      step(g, g < gw1 ? ch.keys[g] : make_uint4(0u, 0u, 0u, 0u));
    }
  } else {
    for (int gb0 = gw0; gb0 < gw1; gb0 += 32 * TK_UNROLL) {
      uint4 kb[TK_UNROLL];
      ch.load_batch(gb0 + lane, gw1, kb);  // 0 keys past the end, as in every step
      #pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u)  // steps of 32 groups, in order
        if (gb0 + 32 * u < gw1) step(gb0 + 32 * u + lane, kb[u]);
    }
  }
}
// Clusters of C CTAs (one CTA per SM) that can be resident at once on the current device.
int resident_clusters(int C) {
  static std::mutex mu;
  static int table[64][TK_MAXC + 1];
  static bool done[64][TK_MAXC + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev][C]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, 1, 1);
    cfg.blockDim = dim3(TK_THREADS, 1, 1);
    cfg.dynamicSmemBytes = 120 * 1024;  // more than half an SM's shared memory: one CTA per SM
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_topk_cluster<false>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 1;
    }
    table[dev][C] = n;
    done[dev][C] = true;
  }
  return table[dev][C];
}

}  // namespace

int launch_topk_mode(const float* scores, int64_t ld, int64_t B, int64_t L, int K, int sink, int window,
                     const int64_t* q_pos, int mode, int div, int32_t* idx, int64_t idx_ld, int32_t* count,
                     int64_t kmax, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  {
    // the kernel's attributes, once per device (host calls stay off the launch path)
    static std::mutex mu;
    static bool set[64];
    int dev = 0;
    LSA_CUDA_TRY(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !set[dev]) {
      for (const void* f : {reinterpret_cast<const void*>(k_topk_cluster<false>),
                            reinterpret_cast<const void*>(k_topk_cluster<true>)}) {
        LSA_CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          2 * TK_MAXC * TK_BINS * 4 + TK_CACHE * 4));
        LSA_CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
      }
      if (dev >= 0 && dev < 64) set[dev] = true;
    }
  }
  // Cluster size: the one with the least work on the busiest SM -- (chunk + a fixed per-CTA cost) x the
  // number of cluster waves the batch needs.  A chunk larger than the shared-memory cache is streamed from
  // global memory (L2) on every pass; measured per element that costs about what the cached passes do,
  // while smaller clusters save the barriers, so many rows (a prefill chunk: 8192 x 131072) run one CTA
  // per row (5.9 ms against 7.8 ms for 6-CTA clusters) and a few long rows use large clusters.
  int C = TK_MAXC;
  double best = -1.0;
  for (int c = 1; c <= TK_MAXC; ++c) {
    const int64_t chunk = (cdiv(L, c) + 3) / 4 * 4;
    const double waves = static_cast<double>(cdiv(B, resident_clusters(c)));
    const double cost = (static_cast<double>(chunk) + 2048.0) * waves;
    if (best < 0.0 || cost < best) {
      best = cost;
      C = c;
    }
  }
  int64_t chunk = (cdiv(L, C) + 3) / 4 * 4;
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
  a.cached = chunk <= TK_CACHE ? 1 : 0;
  // all-gathered histograms (two levels' worth), then the cached chunk
  const size_t dyn = static_cast<size_t>(2 * C * TK_BINS) * 4 + (a.cached ? static_cast<size_t>(chunk) * 4 : 0);
  LSA_CUDA_TRY(launch_pdl(a.cached ? k_topk_cluster<false> : k_topk_cluster<true>,
                          dim3(C, static_cast<unsigned>(B), 1), dim3(TK_THREADS), dyn, s, static_cast<unsigned>(C), a));
  return LSA_OK;
}

}  // namespace lsa
