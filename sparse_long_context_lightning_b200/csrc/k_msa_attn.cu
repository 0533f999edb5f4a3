// MSA attention per (query, head group), rows on the MMA's M side.
//
// Lecture "从两本账看懂长上下文注意力", section "MiniMax Sparse Attention": each GQA group's query heads attend to
// the 128-token blocks their group kept (plus the local block); "LongCat Sparse Attention（LSA）完全拆解",
// section "DSA 基线": the attention itself is absorbed MQA over 576-dim bf16 latent rows, value = the first 512.
//
// B200 design.  A CTA serves 16 query heads of one query (a group of 8, or a 16-head slice of a group of 2 or 4),
// too few for the MMA's M side; the rows are: S^T = C Q_g^T takes 128 consecutive rows (one kept block) on M, the
// 16 heads on N and the 576 dims in 36 K steps; O^T += V^T P^T takes 128 value dims on M (two 64-dim blocks),
// the heads on N and the block's 128 rows in 8 K steps.  Both run at the MMA's fixed cost per instruction for N = 16, and a block is one TMA box per
// 64-dim slice (its rows are consecutive tokens), so there is no per-row gather.  The value slices are loaded a
// second time for O^T (from L2, a few microseconds after the first read): shared memory holds a ring of slices,
// not whole blocks.  One CTA per (query, 16-head slice), over the blocks its group kept; no partials, no combine.
//
// Warp roles (256 threads): warp 0 loads the logits slices (and Q_g), warp 1 the value-slice pairs, warp 2 owns
// TMEM and issues S^T, warp 3 issues O^T, warps 4-7 run the softmax (thread = row = TMEM lane) and write the
// output.  Per-head softmax statistics are reduced across rows with transposing warp shuffles and one exchange
// of four values per head through shared memory.
#include <algorithm>

#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

using namespace sm100;

__device__ int g_msa_attn_timeout;  // a bounded wait of the kernel gave up
__device__ int g_msa_attn_check;    // a tile's rows were not one run of consecutive tokens

constexpr int MA_THREADS = 256;
constexpr int MA_NH = 16;                        // query heads per group (MMA N)
constexpr int MA_ROWS = 128;                     // rows per tile (one block; MMA M)
constexpr int MA_KB = 9;                         // 64-dim slices of a 576-dim row
constexpr int MA_SLICE = MA_ROWS * 128;          // 16 KB: one slice of a tile
constexpr int MA_QSLICE = MA_NH * 128;           // 2 KB: one slice of Q_g
constexpr int MA_LR = 6;                         // logits ring slots (one slice each)
constexpr int MA_VR = 2;                         // value ring slots (two slices each)
constexpr int MA_P_BYTES = MA_NH * MA_ROWS * 2;  // 4 KB: P^T of a tile, bf16, K-major (16 head rows)
constexpr int MA_MAXT = 512;                     // blocks per union row (idx_ld <= 65536)
constexpr uint32_t TM_S = 0;                     // two S^T buffers, 16 columns each
constexpr uint32_t TM_O = 32;                    // O^T: four 128-dim tiles of 16 columns
constexpr float RESCALE_LOG2 = 8.f;
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr int MA_SMEM =
    1024 + MA_KB * 1024 * 2 + MA_LR * MA_SLICE + MA_VR * 2 * MA_SLICE + 2 * MA_P_BYTES + 2048 + MA_MAXT * 8;
static_assert(MA_SMEM <= 232448, "shared memory");
static_assert(MA_NH * MA_ROWS / 2 * 2 <= MA_LR * MA_SLICE, "epilogue staging fits the logits ring");

// instruction descriptor with the A operand's major-ness: f32 accumulate, bf16 A and B
__host__ __device__ constexpr uint32_t idesc_ab(int M, int N, uint32_t a_mn_major, uint32_t b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
constexpr uint32_t IDESC_S = idesc_ab(MA_ROWS, MA_NH, 0u, 0u);   // A = C tile (K-major), B = Q_g (K-major)
constexpr uint32_t IDESC_PV = idesc_ab(128, MA_NH, 1u, 0u);      // A = V^T (dims contiguous), B = P^T (K-major)

struct MaArgs {
  const int32_t* idx;     // [B, ld] the union of the groups' kept blocks, ascending (whole 128-token blocks, then
                          // the partial local block)
  const uint8_t* gmask;   // [B, ld] bit g: group g kept the entry's block
  int64_t ld;
  const int32_t* count;   // [B]
  int G;
  int L;
  float scale_log2;
  uint16_t* out;  // [B, 128, 512] bf16
  float* lse;     // [B, 128] or null
};

// Bounded wait that also returns false once another role of the CTA has given up.
__device__ __forceinline__ bool wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    #pragma unroll 1
    for (int i = 0; i < 8; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > WAIT_NS) return false;
  }
}
// Warp-uniform form: lane 0 waits (acquire), the warp barrier orders that before every lane's next accesses.
__device__ __forceinline__ bool warp_wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int lane) {
  bool ok = true;
  if (lane == 0) ok = wait_ab(bar, parity, abort_flag);
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}
__device__ __forceinline__ void give_up(volatile int* abort_flag) {
  atomicExch(&g_msa_attn_timeout, 1);
  *abort_flag = 1;
}
__device__ __forceinline__ void drain_mmas(uint64_t* bar) {
  mma_commit(bar);
  (void)mbar_spin(bar, 0, WAIT_NS);
}

// Per-head reduction over the warp's 32 rows of 16 values (head h in v[h]) by transposing exchanges: over lane
// bits 4, 3, 2, 1 each lane keeps the half of its values its bit selects, then lane bit 0 on one value.  Lane l
// ends with head l >> 1 (both lanes of a pair hold it).
template <bool MAX>
__device__ __forceinline__ float head_reduce16(float (&v)[MA_NH], int lane) {
  #pragma unroll
  for (int step = 0; step < 4; ++step) {
    const int half = (MA_NH >> step) / 2, off = 16 >> step;
    const bool upper = (lane & off) != 0;
    #pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float send = upper ? v[i] : v[i + half];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  const float got = __shfl_xor_sync(0xffffffffu, v[0], 1);
  return MAX ? fmaxf(v[0], got) : v[0] + got;
}

__global__ void __launch_bounds__(MA_THREADS, 1)
    k_msa_attn_rows(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_q, MaArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qs = base;                              // Q_g: slice kb at qs + kb * 2 KB (16 heads x 128 B)
  unsigned char* lring = qs + MA_KB * 2048;              // logits ring: slot s at lring + s * 16 KB
  unsigned char* vring = lring + MA_LR * MA_SLICE;       // value ring: slot s (two slices) at vring + s * 32 KB
  unsigned char* pbuf = vring + MA_VR * 2 * MA_SLICE;    // P^T, two buffers of 4 KB
  float* red = reinterpret_cast<float*>(pbuf + 2 * MA_P_BYTES);  // [2][4][16] per-warp head maxima / sums
  float* fin = red + 2 * 4 * MA_NH;                      // [16] final sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(fin + MA_NH);
  uint64_t* q_full = bars;
  uint64_t* lr_full = q_full + 1;         // [MA_LR]
  uint64_t* lr_empty = lr_full + MA_LR;   // [MA_LR]
  uint64_t* vr_full = lr_empty + MA_LR;   // [MA_VR]
  uint64_t* vr_empty = vr_full + MA_VR;   // [MA_VR]
  uint64_t* s_full = vr_empty + MA_VR;    // [2]
  uint64_t* s_empty = s_full + 2;         // [2] (4 softmax warps)
  uint64_t* p_full = s_empty + 2;         // [2] (4 softmax warps)
  uint64_t* pv_done = p_full + 2;         // [2]
  uint64_t* o_done = pv_done + 2;
  uint64_t* drain = o_done + 1;           // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* ntiles_s = const_cast<int*>(abort_flag) + 1;
  int* tfirst = reinterpret_cast<int*>(base + MA_SMEM - 1024 - MA_MAXT * 8);  // [512] this group's blocks: first entry
  int* trows = tfirst + MA_MAXT;                                                // [512] and its number of rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.x;  // query b = bg / 8, heads 16 hs .. 16 hs + 15 (hs = bg % 8) of group hs G / 8
  const int b = bg / 8, hs = bg % 8, g = hs * a.G / 8;
  const int32_t* ridx = a.idx + static_cast<int64_t>(b) * a.ld;
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < MA_LR; ++i) {
      mbar_init(&lr_full[i], 1);
      mbar_init(&lr_empty[i], 1);
    }
    for (int i = 0; i < MA_VR; ++i) {
      mbar_init(&vr_full[i], 1);
      mbar_init(&vr_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&drain[i], 1);
    }
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // Q_g: the group's 16 head rows of query b, nine 64-dim slices (Q is not written by the pipeline's earlier
    // kernels, so it is loaded before the programmatic-launch wait)
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kv);
    mbar_expect_tx(q_full, MA_KB * MA_QSLICE);
    for (int kb = 0; kb < MA_KB; ++kb) tma_load_2d(qs + kb * 2048, &tm_q, q_full, 64 * kb, b * 128 + hs * MA_NH);
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, 128);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_launch_dependents();
  if (warp == 0) {
    // this group's tiles: the union row's blocks (entries j * 128 ..) whose mask has bit g, in order
    int n = a.count[b];
    n = n < 0 ? 0 : (static_cast<int64_t>(n) > a.ld ? static_cast<int>(a.ld) : n);
    const int nblk = min((n + MA_ROWS - 1) / MA_ROWS, MA_MAXT);
    int kept = 0;
    for (int j0 = 0; j0 < nblk; j0 += 32) {
      const int j = j0 + lane;
      const bool mine = j < nblk && ((a.gmask[static_cast<int64_t>(b) * a.ld + static_cast<int64_t>(j) * MA_ROWS] >> g) & 1u);
      const uint32_t bal = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        const int o = kept + __popc(bal & ((1u << lane) - 1u));
        tfirst[o] = j * MA_ROWS;
        trows[o] = min(MA_ROWS, n - j * MA_ROWS);
      }
      kept += __popc(bal);
    }
    if (lane == 0) *ntiles_s = kept;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int ntiles = *ntiles_s;
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 || warp == 1) {
    // ------------------------------------------------------------------ TMA producers
    // warp 0: slices 0..8 of tile t into the logits ring; warp 1: value slices (2p, 2p + 1) of tile t into the
    // value ring.  A tile's rows are tokens first .. first + 127 (TMA fills rows past L with zeros; rows past the
    // count are masked by the softmax).  Before exiting, a producer waits (bounded) for its last copies.
    if (lane == 0 && ntiles > 0) {
      const bool logits = warp == 0;
      int issued = 0;
      bool ok = true;
      for (int t = 0; ok && t < ntiles; ++t) {
        int first = ridx[tfirst[t]];
        first = first < 0 ? 0 : (first >= a.L ? a.L - 1 : first);
        const int nitems = logits ? MA_KB : 4;
        for (int k = 0; k < nitems; ++k) {
          const int idx = t * nitems + k;
          const int nslot = logits ? MA_LR : MA_VR;
          const int slot = idx % nslot;
          uint64_t* full = logits ? &lr_full[slot] : &vr_full[slot];
          uint64_t* empty = logits ? &lr_empty[slot] : &vr_empty[slot];
          if (!wait_ab(empty, ((idx / nslot) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (logits) {
            mbar_expect_tx(full, MA_SLICE);
            tma_load_2d(lring + slot * MA_SLICE, &tm_kv, full, 64 * k, first);
          } else {
            mbar_expect_tx(full, 2 * MA_SLICE);
            tma_load_2d(vring + slot * 2 * MA_SLICE, &tm_kv, full, 64 * (2 * k), first);
            tma_load_2d(vring + slot * 2 * MA_SLICE + MA_SLICE, &tm_kv, full, 64 * (2 * k + 1), first);
          }
          ++issued;
        }
      }
      if (!ok) give_up(abort_flag);
      const int nslot = logits ? MA_LR : MA_VR;
      for (int idx = max(0, issued - nslot); idx < issued; ++idx) {
        const int slot = idx % nslot;
        (void)mbar_spin(logits ? &lr_full[slot] : &vr_full[slot], (idx / nslot) & 1, WAIT_NS);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------------ MMA issuers
    if (lane == 0 && ntiles > 0) {
      const bool logits = warp == 2;
      bool ok = true, issued = false;
      if (logits) {
        ok = mbar_spin(q_full, 0, WAIT_NS);
        for (int t = 0; ok && t < ntiles; ++t) {
          const int x = t & 1;
          if (!wait_ab(&s_empty[x], ((t >> 1) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < MA_KB; ++kb) {
            const int idx = t * MA_KB + kb, slot = idx % MA_LR;
            if (!wait_ab(&lr_full[slot], (idx / MA_LR) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = desc_sw128(smem_u32(lring + slot * MA_SLICE));
            const uint64_t bdesc = desc_sw128(smem_u32(qs + kb * 2048));
            #pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem + TM_S + x * MA_NH, adesc + ((kk * 32) >> 4), bdesc + ((kk * 32) >> 4), IDESC_S,
                      (kb | kk) != 0 ? 1u : 0u);
            mma_commit(&lr_empty[slot]);
            issued = true;
          }
          if (!ok) break;
          mma_commit(&s_full[x]);
        }
      } else {
        for (int t = 0; ok && t < ntiles; ++t) {
          const int x = t & 1;
          if (!wait_ab(&p_full[x], (t >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          for (int pr = 0; pr < 4; ++pr) {
            const int idx = t * 4 + pr, slot = idx % MA_VR;
            if (!wait_ab(&vr_full[slot], (idx / MA_VR) & 1, abort_flag)) {
              ok = false;
              break;
            }
            fence_proxy_async_smem();  // P^T was written by the softmax threads (generic proxy)
            tc_fence_after();
            const uint32_t vaddr = smem_u32(vring + slot * 2 * MA_SLICE);
            const uint32_t paddr = smem_u32(pbuf + x * MA_P_BYTES);
            #pragma unroll
            for (int kk = 0; kk < MA_ROWS / 16; ++kk) {
              // A = V^T: 128 dims (the pair's two 64-dim slices, 16 KB apart) x rows 16 kk .. 16 kk + 15;
              // B = P^T: 16 heads x the same rows (K-major, 64 rows per 128-byte atom, atoms 2 KB apart)
              const uint64_t adesc = desc_sw128_mn(vaddr + kk * 16 * 128, MA_SLICE, 1024);
              const uint64_t bdesc = desc_sw128(paddr + (kk >> 2) * 2048) + (((kk & 3) * 32) >> 4);
              mma_f16(tmem + TM_O + pr * MA_NH, adesc, bdesc, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&vr_empty[slot]);
            issued = true;
          }
          if (!ok) break;
          mma_commit(&pv_done[x]);
        }
        if (ok) mma_commit(o_done);
      }
      if (!ok) {
        give_up(abort_flag);
        if (issued) drain_mmas(&drain[logits ? 0 : 1]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax (warps 4-7), then the output
    // Thread = row r of a tile = TMEM lane r (S^T) and, for O^T, dim 32 q4 + lane of each 128-dim tile.  The
    // per-head reference (the max over every row so far) is identical in every thread.  The loop never breaks:
    // a failed wait clears ok (warp-uniform) and the rest of the work is skipped, so the four warps always run
    // the same named barriers.
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    float m_used[MA_NH], lp[MA_NH];
    #pragma unroll
    for (int h = 0; h < MA_NH; ++h) {
      m_used[h] = -INFINITY;
      lp[h] = 0.f;
    }
    bool ok = ntiles > 0, gave = !ok;
    for (int t = 0; t < ntiles; ++t) {
      const int x = t & 1;
      ok = ok && warp_wait_ab(&s_full[x], (t >> 1) & 1, abort_flag, lane);
      float z[MA_NH];
      if (ok) {
        tc_fence_after();
        uint32_t sr[MA_NH];
        tmem_ld16(tq + TM_S + x * MA_NH, sr);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[x]);
        const bool valid = r < trows[t];
        if (valid && ridx[tfirst[t] + r] != ridx[tfirst[t]] + r) atomicExch(&g_msa_attn_check, 1);  // not one block
        #pragma unroll
        for (int h = 0; h < MA_NH; ++h) z[h] = valid ? __uint_as_float(sr[h]) * a.scale_log2 : -INFINITY;
      } else {
        #pragma unroll
        for (int h = 0; h < MA_NH; ++h) z[h] = -INFINITY;
      }
      // the tile's maximum per head: within the warp, then over the four warps
      float v[MA_NH];
      #pragma unroll
      for (int h = 0; h < MA_NH; ++h) v[h] = z[h];
      const float wm = head_reduce16<true>(v, lane);
      float* rd = red + x * 4 * MA_NH;  // buffer of tile parity: rewritten two tiles later, after the next barrier
      if ((lane & 1) == 0) rd[q4 * MA_NH + (lane >> 1)] = wm;
      named_bar_sync(1, 128);
      float mt[MA_NH];
      #pragma unroll
      for (int j = 0; j < MA_NH / 4; ++j) {
        const float4 a0 = reinterpret_cast<const float4*>(rd)[j], a1 = reinterpret_cast<const float4*>(rd + MA_NH)[j];
        const float4 a2 = reinterpret_cast<const float4*>(rd + 2 * MA_NH)[j], a3 = reinterpret_cast<const float4*>(rd + 3 * MA_NH)[j];
        mt[4 * j] = fmaxf(fmaxf(a0.x, a1.x), fmaxf(a2.x, a3.x));
        mt[4 * j + 1] = fmaxf(fmaxf(a0.y, a1.y), fmaxf(a2.y, a3.y));
        mt[4 * j + 2] = fmaxf(fmaxf(a0.z, a1.z), fmaxf(a2.z, a3.z));
        mt[4 * j + 3] = fmaxf(fmaxf(a0.w, a1.w), fmaxf(a2.w, a3.w));
      }
      // lazy rescale per head: the reference moves only when the head's max grows by more than 2^8
      float alpha[MA_NH];
      bool resc = false;
      #pragma unroll
      for (int h = 0; h < MA_NH; ++h) {
        alpha[h] = 1.f;
        if (m_used[h] == -INFINITY) {
          m_used[h] = mt[h];  // nothing accumulated for this head yet
        } else if (mt[h] > m_used[h] + RESCALE_LOG2) {
          alpha[h] = ex2_approx(m_used[h] - mt[h]);
          m_used[h] = mt[h];
          resc = true;
        }
      }
      uint32_t pk[MA_NH / 2];
      #pragma unroll
      for (int h = 0; h < MA_NH; h += 2) {
        const float p0 = ex2_approx(z[h] - (m_used[h] == -INFINITY ? 0.f : m_used[h]));
        const float p1 = ex2_approx(z[h + 1] - (m_used[h + 1] == -INFINITY ? 0.f : m_used[h + 1]));
        lp[h] = lp[h] * alpha[h] + p0;  // the sums use the fp32 probabilities (O^T uses them rounded to bf16)
        lp[h + 1] = lp[h + 1] * alpha[h + 1] + p1;
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(p0, p1);
        pk[h / 2] = *reinterpret_cast<const uint32_t*>(&p2);
      }
      if (ok && resc) {  // resc is the same in every thread
        // O^T must hold every earlier tile before its head columns are rescaled: tile t-1's O^T MMAs completed
        ok = warp_wait_ab(&pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag, lane);
        if (ok) {
          tc_fence_after();
          #pragma unroll 1
          for (int pr = 0; pr < 4; ++pr) {
            uint32_t o[MA_NH];
            tmem_ld16(tq + TM_O + pr * MA_NH, o);
            tmem_ld_wait();
            #pragma unroll
            for (int h = 0; h < MA_NH; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(tq + TM_O + pr * MA_NH),
                "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]), "r"(o[8]),
                "r"(o[9]), "r"(o[10]), "r"(o[11]), "r"(o[12]), "r"(o[13]), "r"(o[14]), "r"(o[15])
                : "memory");
          }
          tmem_st_wait();
          tc_fence_before();
        }
      }
      // P^T buffer x is free once tile t-2's O^T MMAs completed
      ok = ok && (t < 2 || warp_wait_ab(&pv_done[x], ((t - 2) >> 1) & 1, abort_flag, lane));
      if (ok) {
        // P^T row h (head), K = this row r: atom r / 64 (2 KB), 8-row group h / 8 (1 KB), row h % 8 (128 B),
        // 16-byte chunk ((r % 64) / 8) ^ (h % 8) (128-byte swizzle), bf16 (r % 8)
        unsigned char* pb = pbuf + x * MA_P_BYTES + (r >> 6) * 2048;
        const int ch = (r & 63) >> 3;
        #pragma unroll
        for (int h = 0; h < MA_NH; ++h) {
          const uint32_t word = pk[h >> 1];
          const uint16_t hv = static_cast<uint16_t>((h & 1) ? (word >> 16) : (word & 0xFFFFu));
          *reinterpret_cast<uint16_t*>(pb + (h >> 3) * 1024 + (h & 7) * 128 + ((ch ^ (h & 7)) << 4) + (r & 7) * 2) = hv;
        }
        fence_proxy_async_smem();  // read by the O^T MMAs (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
      }
      if (!ok && !gave) {  // stop the other roles at once (their waits see the abort flag)
        if (lane == 0) give_up(abort_flag);
        gave = true;
      }
    }
    // the sums over every row, per head (buffer ntiles % 2: its last readers passed the last tile's barrier)
    float v2[MA_NH];
    #pragma unroll
    for (int h = 0; h < MA_NH; ++h) v2[h] = lp[h];
    const float wsum = head_reduce16<false>(v2, lane);
    float* rd2 = red + (ntiles & 1) * 4 * MA_NH;
    if ((lane & 1) == 0) rd2[q4 * MA_NH + (lane >> 1)] = wsum;
    named_bar_sync(1, 128);
    const bool have = ok && warp_wait_ab(o_done, 0, abort_flag, lane);
    float inv[MA_NH];
    #pragma unroll
    for (int h = 0; h < MA_NH; ++h) {
      const float l = rd2[h] + rd2[MA_NH + h] + rd2[2 * MA_NH + h] + rd2[3 * MA_NH + h];
      inv[h] = (have && l > 0.f) ? 1.f / l : 0.f;
      if (a.lse && r == h) {
        a.lse[static_cast<int64_t>(b) * 128 + hs * MA_NH + h] =
            (have && l > 0.f) ? (m_used[h] + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
    // O^T / l into a [16 heads][512 dims] bf16 staging area (the logits ring: every S^T MMA has completed), then
    // 16 coalesced 1 KB output rows
    uint16_t* stage = reinterpret_cast<uint16_t*>(lring);
    tc_fence_after();
    #pragma unroll 1
    for (int pr = 0; pr < 4; ++pr) {
      uint32_t o[MA_NH];
      if (have) {
        tmem_ld16(tq + TM_O + pr * MA_NH, o);
        tmem_ld_wait();
      } else {
        #pragma unroll
        for (int h = 0; h < MA_NH; ++h) o[h] = 0u;
      }
      #pragma unroll
      for (int h = 0; h < MA_NH; ++h) {
        const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(o[h]) * inv[h]);
        stage[h * 512 + pr * 128 + r] = *reinterpret_cast<const uint16_t*>(&bv);
      }
    }
    named_bar_sync(1, 128);
    #pragma unroll
    for (int i = 0; i < (MA_NH * 512 * 2 / 16) / 128; ++i) {
      const int e = i * 128 + r;  // 16-byte piece e of the 16 KB
      const int h = e / 64, c = e % 64;
      *reinterpret_cast<uint4*>(a.out + (static_cast<int64_t>(b) * 128 + hs * MA_NH + h) * 512 + 8 * c) =
          reinterpret_cast<const uint4*>(stage)[e];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);

// MSA attention, 128 query heads in G = 2, 4 or 8 groups: one CTA per (query, 16-head slice) over the union row's
// blocks that the slice's group kept.
int launch_msa_attn_rows(const void* q, const void* kv, int64_t L, const int32_t* idx, const uint8_t* gmask, int64_t ld,
                         const int32_t* count, int64_t B, int G, float scale, void* out, float* lse, cudaStream_t s) {
  if ((G != 2 && G != 4 && G != 8) || ld > static_cast<int64_t>(MA_MAXT) * MA_ROWS) return LSA_ERR_UNSUPPORTED;
  CUtensorMap tkv, tq;
  int st = make_map(&tkv, kv, false, L, 576, 64, MA_ROWS);
  if (st) return st;
  st = make_map(&tq, q, false, B * 128, 576, 64, MA_NH);
  if (st) return st;
  MaArgs a;
  a.idx = idx;
  a.gmask = gmask;
  a.ld = ld;
  a.count = count;
  a.G = G;
  a.L = static_cast<int>(L);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_msa_attn_rows), MA_SMEM));
  LSA_CUDA_TRY(launch_pdl(k_msa_attn_rows, dim3(static_cast<unsigned>(B * 8)), dim3(MA_THREADS), MA_SMEM, s, 0u, tkv,
                          tq, a));
  return LSA_OK;
}

// The kernel's flags, read and cleared: give-up (returned) and device check (*check: a tile's rows were not one
// run of consecutive tokens); -1: CUDA error.
int take_msa_attn_flags(int* check) {
  int v = 0, c = 0;
  if (cudaMemcpyFromSymbol(&v, g_msa_attn_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&c, g_msa_attn_check, sizeof(int)) != cudaSuccess) return -1;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_msa_attn_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  if (c != 0 && cudaMemcpyToSymbol(g_msa_attn_check, &zero, sizeof(int)) != cudaSuccess) return -1;
  *check = c;
  return v;
}

}  // namespace lsa
