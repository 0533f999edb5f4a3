// Sparse absorbed-MQA attention over gathered MLA latent rows on tcgen05 tensor cores.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线": u_t = Attn(h_t, {c_s | s in S_t}), the
// 576-dim bf16 latent c_s shared by all 128 heads, value = its first 512 dims; section "瓶颈一": the
// selected 1152-byte rows are scattered, so the kernel is a gather whose memory-level parallelism decides
// the achieved bandwidth.
//
// B200 design.  A 128 x 512 fp32 output accumulator would fill all of TMEM (128 lanes x 512 columns), so
// the value dims are split over two CTAs: CTA (unit, r) owns output columns [256r, 256r + 256) of one
// work unit (query b, a contiguous split of its selected rows).  The two CTAs are independent -- no
// cluster, no per-tile communication: each gathers the full 1152-byte rows of its tiles (the pair reads
// the same rows at about the same time, so the second read is served by L2) and computes the complete
// logits S = Q C^T itself.  Duplicating the logits MMA costs less than exchanging partial logits between
// CTAs, whose DSMEM latency made every tile wait.
//
// TMEM (512 columns): O [0, 256), two S buffers [256, 320), and Q's dims [0, 384) as the A operand of the
// logits MMA [320, 512) (two bf16 per column).  Q's dims [384, 576) stay in shared memory (48 KB).  The
// gathered tile (32 rows x 9 K-blocks of 64 dims, 128-byte swizzled) serves both MMAs: K-major for
// S = Q C^T and MN-major (its first 512 dims) for O += P V, so no transpose is needed.  Online softmax with
// lazy rescale (O is rescaled only when the running max grows by > 2^8).  Splits of one query are merged
// by a small combine kernel (log-sum-exp weights).
//
// Warp roles (288 threads): warps 0-3 gather (16-byte cp.async copies, many rows in flight per SM; a TMA
// gather4 per 4 rows x 128 bytes issued too slowly here), warp 4 issues the MMAs (S two tiles ahead of
// P.V) and owns TMEM, warps 5-8 load Q into TMEM, then run the softmax (one head per thread = one TMEM
// lane) and the epilogue.
#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

using namespace sm100;

__device__ int g_attn_tc_timeout;  // set when a bounded wait of the kernel gave up
__device__ int g_attn_tc_check;    // set when a selected index was outside [0, L) (the row was clamped)

constexpr int AT_THREADS = 736;  // 16 gather warps, 3 MMA-issuing warps, 4 softmax warps
// A warp's 16-byte cp.async copies are issue-latency bound (one CTA reaches ~18 GB/s with 4 gather warps,
// ~36 GB/s with 16, measured), so the gather runs on 16 warps, two rows of each tile per warp.
constexpr int AT_GATHER_WARPS = 16;
constexpr int AT_MMA_WARP = 16;   // logits of even tiles; owns TMEM
constexpr int AT_MMA_WARP2 = 17;  // logits of odd tiles
constexpr int AT_PV_WARP = 18;    // O += P V; warps 19-22: softmax (warp % 4 = the TMEM lane quarter)
constexpr int AT_T = 32;         // gathered rows per tile
constexpr int AT_H = 128;        // heads (MMA M)
constexpr int AT_KB = 9;         // 64-dim K-blocks of a 576-dim row
constexpr int AT_KB_TQ = 6;      // Q K-blocks held in TMEM (dims [0, 384))
constexpr int AT_KB_SQ = AT_KB - AT_KB_TQ;  // Q K-blocks in shared memory (dims [384, 576))
constexpr int AT_STAGES = 4;
constexpr int AT_O_PITCH = 1040;  // epilogue staging: 1 KB of O per head row + 16 B (rows in different banks)
constexpr int AT_QS_BYTES = AT_KB_SQ * AT_H * 128;         // 48 KB
constexpr int AT_KB_BYTES = AT_T * 128;                    // 4 KB: one 64-dim block of a tile
constexpr int AT_STAGE_BYTES = AT_KB * AT_KB_BYTES;        // 36 KB
constexpr int AT_P_BYTES = AT_H * 128;                     // 16 KB (32 bf16 per head used)
constexpr int AT_SMEM = 1024 + AT_QS_BYTES + AT_STAGES * AT_STAGE_BYTES + AT_P_BYTES + 512;
constexpr uint32_t TM_O = 0;    // TMEM columns [0, 256): O
constexpr uint32_t TM_S = 256;  // TMEM columns [256, 320): two S buffers of 32
constexpr uint32_t TM_Q = 320;  // TMEM columns [320, 512): Q dims [0, 384), two bf16 per column
constexpr uint32_t IDESC_S = idesc_mma(128, AT_T, 1u, 0u);
constexpr uint32_t IDESC_PV = idesc_mma(128, 256, 1u, 1u);
constexpr float RESCALE_LOG2 = 8.f;
static_assert(TM_Q + AT_KB_TQ * 32 == 512, "TMEM columns");
static_assert(AT_SMEM <= 232448, "shared memory");
static_assert(AT_H * AT_O_PITCH <= AT_STAGES * AT_STAGE_BYTES, "epilogue staging fits the stages");

struct AtArgs {
  const uint16_t* q;   // absorbed queries [B, 128, 576] bf16
  const uint16_t* kv;  // latent cache [L, 576] bf16
  const int32_t* idx;
  int64_t idx_ld;
  const int32_t* count;
  int B;
  int L;
  int S;        // splits per query of this launch
  int S_total;  // partial slots per query in ws_o / ws_ml (this launch fills [slot0, slot0 + S)); 1 = no partials
  int slot0;
  float scale_log2;
  uint16_t* out;
  float* lse;
  float* ws_o;   // [B, S, 128, 512] fp32 (S > 1)
  float* ws_ml;  // [B, S, 128, 2]   fp32 (S > 1): running max (log2 units), sum
  int contig;    // rows ascending and unique by construction (the hybrid operator's sink + window rows): a tile
                 // whose rows are consecutive positions is one TMA tile load instead of a row gather
};

__global__ void __launch_bounds__(AT_THREADS, 1)
    k_sparse_attn_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv, AtArgs a) {
  // every global access of this kernel comes after the previous kernel of the stream has completed
  sm100::pdl_wait();
  sm100::pdl_launch_dependents();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = base;
  unsigned char* st_s = q_s + AT_QS_BYTES;
  unsigned char* p_s = st_s + AT_STAGES * AT_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + AT_P_BYTES);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + AT_STAGES;
  uint64_t* s_full = kv_empty + AT_STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* q_full = pv_done + 1;   // Q's shared-memory K-blocks landed (TMA)
  uint64_t* qt_full = q_full + 1;   // Q's TMEM part written by the softmax warps (stages 1-3 free again)
  uint64_t* qst_full = qt_full + 1; // Q's TMEM part landed in stages 1-3 (TMA staging)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qst_full + 1);
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = static_cast<int>(blockIdx.x & 1u);  // value half
  const int unit = static_cast<int>(blockIdx.x >> 1);
  const int b = unit / a.S, split = unit % a.S;
  int n = a.count[b];
  n = n < 0 ? 0 : (static_cast<int64_t>(n) > a.idx_ld ? static_cast<int>(a.idx_ld) : n);
  const int rps = ((n + a.S - 1) / a.S + AT_T - 1) / AT_T * AT_T;
  const int row0 = split * rps;
  const int nrows = max(0, min(n, row0 + rps) - row0);
  const int ntiles = (nrows + AT_T - 1) / AT_T;

  if (tid == 0) {
    for (int i = 0; i < AT_STAGES; ++i) {
      mbar_init(&kv_full[i], AT_GATHER_WARPS * 32);  // one cp.async arrival per gather thread
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);  // the four softmax warps have read the buffer
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(q_full, 1);
    mbar_init(qt_full, 4);
    mbar_init(qst_full, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == AT_MMA_WARP) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < AT_GATHER_WARPS) {
    // ------------------------------------------------------------------ gather producers
    // Warp w copies rows 2w, 2w + 1 of every tile: 72 16-byte cp.async chunks per row, placed in the
    // 128-byte-swizzled K-major layout (chunk c of row t at (c & 7 ^ t & 7) * 16 in K-block c / 8).
    if (ntiles > 0) {
      if (tid == 0) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(q_full, AT_KB_SQ * AT_H * 128);
        for (int kb = 0; kb < AT_KB_SQ; ++kb)
          tma_load_2d(q_s + kb * AT_H * 128, &tm_q, q_full, 64 * (AT_KB_TQ + kb), b * AT_H);
        // Q dims [0, 384) are staged in stages 1-3 (free until the softmax warps have moved them into TMEM)
        mbar_expect_tx(qst_full, AT_KB_TQ * AT_H * 128);
        for (int kb = 0; kb < AT_KB_TQ; ++kb)
          tma_load_2d(st_s + AT_STAGE_BYTES + kb * AT_H * 128, &tm_q, qst_full, 64 * kb, b * AT_H);
      }
      const int32_t* rowidx = a.idx + static_cast<int64_t>(b) * a.idx_ld + row0;
      constexpr int CPR = AT_KB * 8;  // 16-byte chunks per row
      // raw row indices (lane l < 2: row 2w + l) are loaded two tiles ahead and clamped at use
      auto load_idx = [&](int i) -> int {
        const int rr = i * AT_T + warp * 2 + (lane & 1);
        return rr < nrows ? rowidx[rr] : 0;
      };
      // contiguous rows: the tile's first position when its rows are consecutive positions, else -1 (the
      // rows are ascending and unique, so first and last decide); loaded two tiles ahead as well
      auto tile_start = [&](int i) -> int {
        if (!a.contig) return -1;
        const int m = min(AT_T, nrows - i * AT_T);
        const int f = rowidx[i * AT_T], l = rowidx[i * AT_T + m - 1];
        return (f >= 0 && l < a.L && l - f == m - 1) ? f : -1;
      };
      int v_a = load_idx(0);
      int v_b = ntiles > 1 ? load_idx(1) : 0;
      int c_a = tile_start(0);
      int c_b = ntiles > 1 ? tile_start(1) : -1;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % AT_STAGES;
        const int v_raw = v_a;
        v_a = v_b;
        if (i + 2 < ntiles) v_b = load_idx(i + 2);
        const int c_now = c_a;
        c_a = c_b;
        if (i + 2 < ntiles) c_b = tile_start(i + 2);
        // stages 1-3 hold the Q staging until the softmax warps have copied it into TMEM
        const bool staged_ok = !(i >= 1 && i < AT_STAGES) || mbar_spin(qt_full, 0);
        if (!staged_ok || !mbar_spin(&kv_empty[st], ((i / AT_STAGES) & 1) ^ 1) || abort_flag) {
          if (lane == 0) {
            atomicExch(&g_attn_tc_timeout, 1);
            abort_flag = 1;
          }
          break;
        }
        unsigned char* dst = st_s + st * AT_STAGE_BYTES;
        if (c_now >= 0) {  // consecutive rows: nine 32-row TMA boxes in the same swizzled layout
          if (tid == 0) {
            mbar_expect_tx(&kv_full[st], AT_STAGE_BYTES);
            for (int kb = 0; kb < AT_KB; ++kb) tma_load_2d(dst + kb * AT_KB_BYTES, &tm_kv, &kv_full[st], 64 * kb, c_now);
          } else {
            mbar_arrive(&kv_full[st]);
          }
          continue;
        }
        if (lane < 2 && i * AT_T + warp * 2 + lane < nrows && (v_raw < 0 || v_raw >= a.L))
          atomicExch(&g_attn_tc_check, 1);
        const int v = v_raw < 0 ? 0 : (v_raw >= a.L ? a.L - 1 : v_raw);
        #pragma unroll
        for (int k = 0; k < (2 * CPR + 31) / 32; ++k) {
          const int q = lane + 32 * k;
          const int rr = q >= CPR ? 1 : 0, c = q - rr * CPR;
          const int row_in_tile = warp * 2 + rr;
          const int srow = __shfl_sync(0xffffffffu, v, rr);  // every lane takes part
          if (q < 2 * CPR) {
            const int kb = c >> 3, c8 = c & 7;
            cp_async16(dst + kb * AT_KB_BYTES + row_in_tile * 128 + ((c8 ^ (row_in_tile & 7)) << 4),
                       a.kv + static_cast<int64_t>(srow) * 576 + c * 8);
          }
        }
        cp_async_arrive_noinc(&kv_full[st]);
      }
    }
  } else if (warp == AT_MMA_WARP || warp == AT_MMA_WARP2) {
    // ------------------------------------------------------------------ logits MMAs
    // One thread issues about one tcgen05.mma per 30 ns, so the logits MMAs (36 per tile) are split over
    // two issuing warps by tile parity, each with its own S buffer; S runs up to two tiles ahead of P.V.
    const int sb = warp == AT_MMA_WARP ? 0 : 1;
    if (ntiles > sb && lane == 0) {
      bool ok = mbar_spin(q_full, 0) && mbar_spin(qt_full, 0);
      tc_fence_after();
      const uint64_t qdesc = desc_sw128(smem_u32(q_s));
      const uint32_t d = tmem + TM_S + sb * AT_T;
      for (int j = sb; ok && j < ntiles; j += 2) {
        const int st = j % AT_STAGES;
        if (!mbar_spin(&kv_full[st], (j / AT_STAGES) & 1) || !mbar_spin(&s_empty[sb], ((j >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();  // the cp.async (generic proxy) writes are read by the tensor cores
        tc_fence_after();
        const uint64_t sdesc = desc_sw128(smem_u32(st_s + st * AT_STAGE_BYTES));
        // dims [0, 384): A = Q from TMEM (8 columns per K = 16 step); descriptors advance in 16-byte units
        #pragma unroll
        for (int kb = 0; kb < AT_KB_TQ; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ta(d, tmem + TM_Q + kb * 32 + kk * 8, sdesc + ((kb * AT_KB_BYTES + kk * 32) >> 4), IDESC_S,
                       (kb | kk) != 0);
        }
        // dims [384, 576): A = Q from shared memory
        #pragma unroll
        for (int kb = 0; kb < AT_KB_SQ; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(d, qdesc + ((kb * AT_H * 128 + kk * 32) >> 4),
                    sdesc + (((AT_KB_TQ + kb) * AT_KB_BYTES + kk * 32) >> 4), IDESC_S, 1u);
        }
        mma_commit(&s_full[sb]);
      }
      if (!ok) {
        atomicExch(&g_attn_tc_timeout, 1);
        abort_flag = 1;
      }
    }
  } else if (warp == AT_PV_WARP) {
    // ------------------------------------------------------------------ O += P V
    if (ntiles > 0 && lane == 0) {
      bool ok = true;
      const uint64_t pdesc = desc_sw128(smem_u32(p_s));
      for (int j = 0; ok && j < ntiles; ++j) {
        const int stj = j % AT_STAGES;
        // P(j) written means the softmax has read S(j): the logits MMAs of tile j are complete
        if (!mbar_spin(p_full, j & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // V = this CTA's value columns [256r, 256r + 256) = K-blocks 4r .. 4r + 3 of the tile, read MN-major
        const uint32_t v_addr = smem_u32(st_s + stj * AT_STAGE_BYTES + 4 * r * AT_KB_BYTES);
        #pragma unroll
        for (int kk = 0; kk < AT_T / 16; ++kk)
          mma_f16(tmem + TM_O, pdesc + ((kk * 32) >> 4), desc_sw128_mn(v_addr + kk * 16 * 128, AT_KB_BYTES, 1024),
                  IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[stj]);
        mma_commit(pv_done);
      }
      if (!ok) {
        atomicExch(&g_attn_tc_timeout, 1);
        abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------------------------ Q into TMEM, softmax + epilogue
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    if (ntiles > 0) {
      // Q row h, dims [0, 384) -> TMEM lane h, columns TM_Q + 32 kb + j hold dims 64 kb + 2j, 64 kb + 2j + 1;
      // read from the TMA staging (128-byte swizzle: chunk c of row h at ((c ^ h) & 7) * 16)
      // every wait of these warps is decided warp-wide: the TMEM loads and stores that follow are warp-collective
      // (.sync.aligned) and must be executed by all 32 lanes or by none
      if (!__all_sync(0xffffffffu, mbar_spin(qst_full, 0))) ok = false;
      #pragma unroll 1
      for (int kb = 0; kb < AT_KB_TQ; ++kb) {
        const unsigned char* src = st_s + AT_STAGE_BYTES + kb * AT_H * 128 + h * 128;
        uint32_t v[32];
        #pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = *reinterpret_cast<const uint4*>(src + ((c ^ (h & 7)) << 4));
          v[4 * c] = x.x;
          v[4 * c + 1] = x.y;
          v[4 * c + 2] = x.z;
          v[4 * c + 3] = x.w;
        }
        tmem_st32(trow + TM_Q + 32 * kb, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qt_full);
    }
    for (int i = 0; ok && i < ntiles; ++i) {
      const int sb = i & 1;
      const int nvalid = min(AT_T, nrows - i * AT_T);
      uint32_t sr[32];
      if (!__all_sync(0xffffffffu, mbar_spin(&s_full[sb], (i >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld32(trow + TM_S + sb * AT_T, sr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      float z[AT_T];
      #pragma unroll
      for (int c = 0; c < AT_T; ++c) z[c] = c < nvalid ? __uint_as_float(sr[c]) * a.scale_log2 : -INFINITY;
      // row max and sum as trees of 8 independent chains (one warp per scheduler: latency, not issue, bound)
      float m8[8];
      #pragma unroll
      for (int j = 0; j < 8; ++j) m8[j] = z[j];
      #pragma unroll
      for (int c = 8; c < AT_T; ++c) m8[c & 7] = fmaxf(m8[c & 7], z[c]);
      const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      float alpha = 1.f;
      bool resc = false;
      if (i == 0) {
        m_used = mt;
      } else if (mt > m_used + RESCALE_LOG2) {
        alpha = ex2_approx(m_used - mt);
        m_used = mt;
        resc = true;
      }
      uint32_t pk[AT_T / 2];
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      #pragma unroll
      for (int c = 0; c < AT_T; c += 2) {
        const float p0 = ex2_approx(z[c] - m_used), p1 = ex2_approx(z[c + 1] - m_used);
        s8[(c >> 1) & 7] += p0 + p1;  // the row sum uses the fp32 probabilities (P . V uses them rounded to bf16)
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(p0, p1);
        pk[c / 2] = *reinterpret_cast<const uint32_t*>(&p2);
      }
      const float psum = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      l = l * alpha + psum;
      // the previous P . V has finished: the P buffer is free and O is stable
      if (i > 0 && !__all_sync(0xffffffffu, mbar_spin(pv_done, (i - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // a warp rescales its O rows when any of its heads' running max grew (alpha = 1 for the other lanes): the
      // TMEM loads / stores are warp-collective, so the branch must not depend on the lane
      if (__any_sync(0xffffffffu, resc)) {
        #pragma unroll 1
        for (int k = 0; k < 8; ++k) {
          uint32_t o[32];
          tmem_ld32(trow + TM_O + 32 * k, o);
          tmem_ld_wait();
          #pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(trow + TM_O + 32 * k, o);
        }
        tmem_st_wait();
      }
      // P row h (32 bf16 = 64 B) into the 128-byte-swizzled K-major A tile
      unsigned char* prow = p_s + h * 128;
      #pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) * 16)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (!ok) {
      atomicExch(&g_attn_tc_timeout, 1);
      abort_flag = 1;
    }
    // ---- epilogue
    const bool have = __all_sync(0xffffffffu, ok && ntiles > 0 && mbar_spin(pv_done, (ntiles - 1) & 1));
    tc_fence_after();
    const int64_t orow = static_cast<int64_t>(b) * AT_H + h;
    // O (row h = this thread's TMEM lane) is staged in the stage memory -- free once the last P.V completed --
    // with a padded row pitch (no bank conflicts), then written with one bulk copy per row
    unsigned char* srow = st_s + h * AT_O_PITCH;
    if (a.S_total == 1) {
      const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
      #pragma unroll 1
      for (int k = 0; k < 8; ++k) {
        uint32_t o[32];
        if (have) {
          tmem_ld32(trow + TM_O + 32 * k, o);
          tmem_ld_wait();
        } else {
          #pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        uint32_t pk[16];
        #pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv);
          pk[c / 2] = *reinterpret_cast<const uint32_t*>(&v);
        }
        uint4* d4 = reinterpret_cast<uint4*>(srow + 64 * k);
        #pragma unroll
        for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      bulk_store_global(a.out + orow * 512 + 256 * r, srow, 512);
      if (r == 0 && a.lse) a.lse[orow] = (have && l > 0.f) ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      const int64_t prow_i = (static_cast<int64_t>(b) * a.S_total + a.slot0 + split) * AT_H + h;
      #pragma unroll 1
      for (int k = 0; k < 8; ++k) {
        uint32_t o[32];
        if (have) {
          tmem_ld32(trow + TM_O + 32 * k, o);
          tmem_ld_wait();
        } else {
          #pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        float4* d4 = reinterpret_cast<float4*>(srow + 128 * k);
        #pragma unroll
        for (int c = 0; c < 8; ++c)
          d4[c] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]), __uint_as_float(o[4 * c + 2]),
                              __uint_as_float(o[4 * c + 3]));
      }
      fence_proxy_async_smem();
      bulk_store_global(a.ws_o + prow_i * 512 + 256 * r, srow, 1024);
      if (r == 0) {
        a.ws_ml[prow_i * 2 + 0] = have ? m_used : -INFINITY;
        a.ws_ml[prow_i * 2 + 1] = have ? l : 0.f;
      }
    }
    bulk_commit();
    bulk_wait_read0();  // the staging rows are read before the CTA can exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == AT_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the splits of one (query, head): LSE-weighted sum of the partial outputs.  Every load is issued before
// any is used (one L2 round trip) for up to 8 splits; more splits fall back to a second pass.
constexpr int CB_MAXS = 8;
__global__ void __launch_bounds__(128) k_attn_combine(const float* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                                      int S, uint16_t* __restrict__ out, float* __restrict__ lse) {
  // every global access of this kernel comes after the previous kernel of the stream has completed
  sm100::pdl_wait();
  sm100::pdl_launch_dependents();
  const int64_t bh = blockIdx.x;  // b * 128 + h
  const int b = static_cast<int>(bh / AT_H), h = static_cast<int>(bh % AT_H);
  const int64_t p0 = static_cast<int64_t>(b) * S * AT_H + h;  // partial of split s: p0 + s * AT_H
  float2 ml[CB_MAXS];
  float4 v[CB_MAXS];
  #pragma unroll
  for (int sp = 0; sp < CB_MAXS; ++sp) {
    if (sp < S) {
      ml[sp] = reinterpret_cast<const float2*>(ws_ml)[p0 + sp * AT_H];
      v[sp] = reinterpret_cast<const float4*>(ws_o + (p0 + sp * AT_H) * 512)[threadIdx.x];
    }
  }
  float mstar = -INFINITY;
  #pragma unroll
  for (int sp = 0; sp < CB_MAXS; ++sp)
    if (sp < S && ml[sp].y > 0.f) mstar = fmaxf(mstar, ml[sp].x);
  for (int sp = CB_MAXS; sp < S; ++sp) {
    const float2 m = reinterpret_cast<const float2*>(ws_ml)[p0 + sp * AT_H];
    if (m.y > 0.f) mstar = fmaxf(mstar, m.x);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  if (mstar != -INFINITY) {
    #pragma unroll
    for (int sp = 0; sp < CB_MAXS; ++sp) {
      if (sp < S && ml[sp].y > 0.f) {
        const float wgt = exp2f(ml[sp].x - mstar);
        lsum += wgt * ml[sp].y;
        acc.x += wgt * v[sp].x;
        acc.y += wgt * v[sp].y;
        acc.z += wgt * v[sp].z;
        acc.w += wgt * v[sp].w;
      }
    }
    for (int sp = CB_MAXS; sp < S; ++sp) {
      const float2 m = reinterpret_cast<const float2*>(ws_ml)[p0 + sp * AT_H];
      if (!(m.y > 0.f)) continue;
      const float wgt = exp2f(m.x - mstar);
      const float4 x = reinterpret_cast<const float4*>(ws_o + (p0 + sp * AT_H) * 512)[threadIdx.x];
      lsum += wgt * m.y;
      acc.x += wgt * x.x;
      acc.y += wgt * x.y;
      acc.z += wgt * x.z;
      acc.w += wgt * x.w;
    }
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&lo);
  pk.y = *reinterpret_cast<const uint32_t*>(&hi);
  reinterpret_cast<uint2*>(out + bh * 512)[threadIdx.x] = pk;
  if (lse && threadIdx.x == 0) lse[bh] = lsum > 0.f ? (mstar + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
}

// The hybrid operator's two index sets from a selection row (sink | sparse | window, lsa_topk_select's layout):
// the sparse entries, and the fixed (sink + window) entries -- contiguous position ranges.
__global__ void __launch_bounds__(256) k_hfa_split(const int32_t* __restrict__ idx, int64_t idx_ld,
                                                   const int32_t* __restrict__ count, int sink, int window,
                                                   const int64_t* __restrict__ q_pos, int32_t* __restrict__ sp,
                                                   int32_t* __restrict__ sp_cnt, int32_t* __restrict__ fx,
                                                   int64_t fx_ld, int32_t* __restrict__ fx_cnt) {
  const int b = blockIdx.x;
  const int qp = static_cast<int>(q_pos[b]);
  const int nsink = min(sink, qp + 1);
  const int wlo = window > 0 ? max(qp - window + 1, nsink) : qp + 1;
  const int nwin = qp + 1 - wlo;
  int n = count[b];
  n = n < 0 ? 0 : (static_cast<int64_t>(n) > idx_ld ? static_cast<int>(idx_ld) : n);
  const int ndyn = max(0, n - nsink - nwin);
  const int32_t* row = idx + static_cast<int64_t>(b) * idx_ld;
  for (int i = threadIdx.x; i < ndyn; i += 256) sp[static_cast<int64_t>(b) * idx_ld + i] = row[nsink + i];
  for (int i = threadIdx.x; i < nsink + nwin; i += 256)
    fx[static_cast<int64_t>(b) * fx_ld + i] = i < nsink ? i : wlo + (i - nsink);
  if (threadIdx.x == 0) {
    sp_cnt[b] = ndyn;
    fx_cnt[b] = nsink + nwin;
  }
}

// Head padding for the tensor-core kernels (128 heads = the MMA's M): qp[b, h] = q[b, h] for h < H, else 0 (576-dim
// bf16 rows as 72 16-byte units); out[b, h] = outp[b, h] and lse[b, h] = lsep[b, h] for h < H.
__global__ void k_pad_heads(const uint4* __restrict__ q, int H, int64_t B, uint4* __restrict__ qp) {
  const int64_t total = B * AT_H * 72;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / 72;
    const int c = static_cast<int>(i % 72);
    const int64_t b = r / AT_H;
    const int h = static_cast<int>(r % AT_H);
    qp[i] = h < H ? q[(b * H + h) * 72 + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}
__global__ void k_unpad_heads(const uint4* __restrict__ outp, const float* __restrict__ lsep, int H, int64_t B,
                              uint4* __restrict__ out, float* __restrict__ lse) {
  const int64_t total = B * H * 64;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / 64;
    const int c = static_cast<int>(i % 64);
    const int64_t b = r / H;
    const int h = static_cast<int>(r % H);
    out[i] = outp[(b * AT_H + h) * 64 + c];
    if (lse != nullptr && c == 0) lse[r] = lsep[b * AT_H + h];
  }
}

int splits_for(int64_t B) {
  int64_t s = 148 / (2 * (B > 0 ? B : 1));
  if (s < 1) s = 1;
  if (s > 32) s = 32;
  return static_cast<int>(s);
}

}  // namespace

int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);
int sm_count();
int launch_attn_simt(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                     const int32_t* count, int64_t B, int H, float scale, void* out, float* lse, cudaStream_t s);

int attn2_units(int64_t B, int64_t idx_ld);
int launch_sparse_attn_2p(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                          const int32_t* count, int64_t B, float scale, void* out, float* lse, void* ws, int S,
                          cudaStream_t s);

// Partial slots per query of lsa_sparse_attn with 128 heads: the two-pass kernel's work units when the batch
// fits one wave of it (decode batches), else the value-half kernel's splits.
static int attn_slots(int64_t B, int64_t idx_ld) {
  const int s2 = attn2_units(B, idx_ld);
  return s2 > 0 ? s2 : splits_for(B);
}

size_t attn2_ws_bytes(int64_t B, int S);

// Head counts below 128 run on the 128-head tensor-core kernels with zero-padded queries: padded queries
// [B, 128, 576] bf16 | padded outputs [B, 128, 512] bf16 | padded lse [B, 128] | the 128-head call's scratch.
static bool padded_heads(int H) { return H == 16 || H == 32 || H == 64; }
static size_t pad_bytes(int64_t B) {
  return align_up(static_cast<size_t>(B) * AT_H * 576 * 2, 256) + align_up(static_cast<size_t>(B) * AT_H * 512 * 2, 256) +
         align_up(static_cast<size_t>(B) * AT_H * 4, 256);
}

size_t sparse_attn_ws_bytes(int64_t B, int64_t idx_ld, int H) {
  if (padded_heads(H)) return pad_bytes(B) + sparse_attn_ws_bytes(B, idx_ld, AT_H);
  if (H != AT_H) return 0;
  const int s2 = attn2_units(B, idx_ld);
  if (s2 > 0) return attn2_ws_bytes(B, s2);
  const int S = splits_for(B);
  if (S == 1) return 0;
  const size_t o = align_up(static_cast<size_t>(B) * S * AT_H * 512 * 4, 256);
  return o + align_up(static_cast<size_t>(B) * S * AT_H * 2 * 4, 256);
}


int launch_sparse_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                       const int32_t* count, int64_t B, int H, float scale, void* out, float* lse, void* ws,
                       size_t ws_bytes, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  if (padded_heads(H) && L < (int64_t(1) << 31)) {
    // the query's heads in the first H rows of zero-padded 128-head queries, the 128-head kernels, then the
    // real rows back
    const size_t need = sparse_attn_ws_bytes(B, idx_ld, H);
    if (ws == nullptr || !aligned256(ws) || ws_bytes < need) return LSA_ERR_WORKSPACE;
    unsigned char* base = static_cast<unsigned char*>(ws);
    void* qp = base;
    void* outp = base + align_up(static_cast<size_t>(B) * AT_H * 576 * 2, 256);
    float* lsep = reinterpret_cast<float*>(static_cast<unsigned char*>(outp) +
                                           align_up(static_cast<size_t>(B) * AT_H * 512 * 2, 256));
    const int grid = sm_count() * 4;
    k_pad_heads<<<grid, 256, 0, s>>>(static_cast<const uint4*>(q), H, B, static_cast<uint4*>(qp));
    LSA_CUDA_TRY(cudaGetLastError());
    const int st = launch_sparse_attn(qp, kv, L, idx, idx_ld, count, B, AT_H, scale, outp, lsep, base + pad_bytes(B),
                                      ws_bytes - pad_bytes(B), s);
    if (st != LSA_OK) return st;
    k_unpad_heads<<<grid, 256, 0, s>>>(static_cast<const uint4*>(outp), lsep, H, B, static_cast<uint4*>(out), lse);
    return cuda_status(cudaGetLastError());
  }
  if (H != AT_H || L >= (int64_t(1) << 31)) return launch_attn_simt(q, kv, L, idx, idx_ld, count, B, H, scale, out, lse, s);
  const int S2 = attn2_units(B, idx_ld);
  const int S = S2 > 0 ? S2 : splits_for(B);
  const size_t need = sparse_attn_ws_bytes(B, idx_ld, H);
  if (S > 1 && (ws == nullptr || !aligned256(ws) || ws_bytes < need)) return LSA_ERR_WORKSPACE;
  if (!aligned16(q)) return LSA_ERR_INVALID_ARG;
  // decode batches: one SM per (query, row range), rows read once, logits computed once
  if (S2 > 0) return launch_sparse_attn_2p(q, kv, L, idx, idx_ld, count, B, scale, out, lse, ws, S2, s);
  CUtensorMap tq, tkv;
  int st = make_map(&tq, q, false, B * AT_H, 576, 64, AT_H);
  if (st) return st;
  st = make_map(&tkv, kv, false, L, 576, 64, AT_T);
  if (st) return st;
  if (!aligned16(q)) return LSA_ERR_INVALID_ARG;
  AtArgs a;
  a.contig = 0;
  a.q = static_cast<const uint16_t*>(q);
  a.kv = static_cast<const uint16_t*>(kv);
  a.idx = idx;
  a.idx_ld = idx_ld;
  a.count = count;
  a.B = static_cast<int>(B);
  a.L = static_cast<int>(L);
  a.S = S;
  a.S_total = S;
  a.slot0 = 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.ws_o = S > 1 ? static_cast<float*>(ws) : nullptr;
  a.ws_ml = S > 1 ? reinterpret_cast<float*>(static_cast<unsigned char*>(ws) +
                                             align_up(static_cast<size_t>(B) * S * AT_H * 512 * 4, 256))
                  : nullptr;
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_sparse_attn_tc), AT_SMEM));
  const int64_t grid = 2 * B * S;
  if (grid > 0x7FFFFFFF) return LSA_ERR_UNSUPPORTED;
  LSA_CUDA_TRY(launch_pdl(k_sparse_attn_tc, dim3(static_cast<unsigned>(grid)), dim3(AT_THREADS), AT_SMEM, s, 0u, tq, tkv,
                          a));
  if (S > 1) {
    LSA_CUDA_TRY(launch_pdl(k_attn_combine, dim3(static_cast<unsigned>(B * AT_H)), dim3(128), 0, s, 0u,
                            static_cast<const float*>(a.ws_o), static_cast<const float*>(a.ws_ml), S, a.out, lse));
  }
  return LSA_OK;
}

// Hybrid (sparse + contiguous) operator: workspace = partials of S_sp + S_fix slots (the two branches' splits)
// | ml of those | sparse rows [B, idx_ld] | fixed rows [B, sink + window] | two counts.
struct HfaLayout {
  int S_sp, S_fix;  // splits of the sparse and the fixed branch (the SMs shared by their row budgets)
  size_t o_ml, o_sp, o_fx, o_spc, o_fxc, total;
};
static HfaLayout hfa_layout(int64_t B, int64_t idx_ld, int sink, int window) {
  HfaLayout h;
  const int S = splits_for(B);
  const int64_t fixed = static_cast<int64_t>(sink) + window;
  const int64_t sparse = max(int64_t(0), idx_ld - fixed);
  h.S_fix = fixed + sparse > 0 ? static_cast<int>((S * fixed + (fixed + sparse) / 2) / (fixed + sparse)) : 0;
  h.S_fix = min(max(h.S_fix, 1), max(S - 1, 1));
  h.S_sp = max(S - h.S_fix, 1);
  const int St = h.S_sp + h.S_fix;
  size_t o = align_up(static_cast<size_t>(B) * St * AT_H * 512 * 4, 256);
  h.o_ml = o;
  o = align_up(o + static_cast<size_t>(B) * St * AT_H * 2 * 4, 256);
  h.o_sp = o;
  o = align_up(o + static_cast<size_t>(B) * idx_ld * 4, 256);
  h.o_fx = o;
  o = align_up(o + static_cast<size_t>(B) * (sink + window) * 4, 256);
  h.o_spc = o;
  o = align_up(o + static_cast<size_t>(B) * 4, 256);
  h.o_fxc = o;
  h.total = align_up(o + static_cast<size_t>(B) * 4, 256);
  return h;
}

size_t hybrid_attn_ws_bytes(int64_t B, int64_t idx_ld, int H, int sink, int window) {
  if (H != AT_H) return 0;
  return hfa_layout(B, idx_ld, sink, window).total;
}

// a second, non-blocking stream and fork / join events per device (created on first use)
static int side_stream(cudaStream_t* side, cudaEvent_t* fork, cudaEvent_t* join) {
  static std::mutex mu;
  static cudaStream_t st[64];
  static cudaEvent_t ef[64], ej[64];
  int dev = 0;
  LSA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return LSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!st[dev]) {
    LSA_CUDA_TRY(cudaStreamCreateWithFlags(&st[dev], cudaStreamNonBlocking));
    LSA_CUDA_TRY(cudaEventCreateWithFlags(&ef[dev], cudaEventDisableTiming));
    LSA_CUDA_TRY(cudaEventCreateWithFlags(&ej[dev], cudaEventDisableTiming));
  }
  *side = st[dev];
  *fork = ef[dev];
  *join = ej[dev];
  return LSA_OK;
}

int launch_hybrid_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                       const int32_t* count, int64_t B, int H, int sink, int window, const int64_t* q_pos,
                       float scale, void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  // other head counts: one pass over the union (the same result, computed at once)
  if (H != AT_H || L >= (int64_t(1) << 31)) return launch_attn_simt(q, kv, L, idx, idx_ld, count, B, H, scale, out, lse, s);
  const HfaLayout h = hfa_layout(B, idx_ld, sink, window);
  if (ws == nullptr || !aligned256(ws) || ws_bytes < h.total) return LSA_ERR_WORKSPACE;
  if (!aligned16(q)) return LSA_ERR_INVALID_ARG;
  CUtensorMap tq, tkv;
  int st = make_map(&tq, q, false, B * AT_H, 576, 64, AT_H);
  if (st) return st;
  st = make_map(&tkv, kv, false, L, 576, 64, AT_T);
  if (st) return st;
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
  const int ss = side_stream(&side, &ev_fork, &ev_join);
  if (ss) return ss;
  unsigned char* base = static_cast<unsigned char*>(ws);
  int32_t* sp = reinterpret_cast<int32_t*>(base + h.o_sp);
  int32_t* fx = reinterpret_cast<int32_t*>(base + h.o_fx);
  int32_t* spc = reinterpret_cast<int32_t*>(base + h.o_spc);
  int32_t* fxc = reinterpret_cast<int32_t*>(base + h.o_fxc);
  const int64_t fx_ld = sink + window;
  k_hfa_split<<<static_cast<unsigned>(B), 256, 0, s>>>(idx, idx_ld, count, sink, window, q_pos, sp, spc, fx,
                                                       fx_ld > 0 ? fx_ld : 1, fxc);
  LSA_CUDA_TRY(cudaGetLastError());
  AtArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.kv = static_cast<const uint16_t*>(kv);
  a.B = static_cast<int>(B);
  a.L = static_cast<int>(L);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.S_total = h.S_sp + h.S_fix;
  a.ws_o = reinterpret_cast<float*>(base);
  a.ws_ml = reinterpret_cast<float*>(base + h.o_ml);
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_sparse_attn_tc), AT_SMEM));
  // fixed branch (sink + window, contiguous: TMA tile loads) on the side stream: slots [S_sp, S_sp + S_fix)
  LSA_CUDA_TRY(cudaEventRecord(ev_fork, s));
  LSA_CUDA_TRY(cudaStreamWaitEvent(side, ev_fork, 0));
  AtArgs af = a;
  af.idx = fx;
  af.idx_ld = fx_ld > 0 ? fx_ld : 1;
  af.count = fxc;
  af.S = h.S_fix;
  af.slot0 = h.S_sp;
  af.contig = 1;
  // a plain launch: its inputs arrive through the fork event, not from the side stream's previous kernel
  k_sparse_attn_tc<<<static_cast<unsigned>(2 * B * h.S_fix), AT_THREADS, AT_SMEM, side>>>(tq, tkv, af);
  LSA_CUDA_TRY(cudaGetLastError());
  LSA_CUDA_TRY(cudaEventRecord(ev_join, side));
  // sparse branch (row gathers) on the caller's stream: slots [0, S_sp)
  AtArgs as = a;
  as.idx = sp;
  as.idx_ld = idx_ld;
  as.count = spc;
  as.S = h.S_sp;
  as.slot0 = 0;
  as.contig = 0;
  LSA_CUDA_TRY(launch_pdl(k_sparse_attn_tc, dim3(static_cast<unsigned>(2 * B * h.S_sp)), dim3(AT_THREADS), AT_SMEM, s,
                          0u, tq, tkv, as));
  // merge: the online-softmax (LSE) combination of all S + 1 partials
  LSA_CUDA_TRY(cudaStreamWaitEvent(s, ev_join, 0));
  LSA_CUDA_TRY(launch_pdl(k_attn_combine, dim3(static_cast<unsigned>(B * AT_H)), dim3(128), 0, s, 0u,
                          static_cast<const float*>(a.ws_o), static_cast<const float*>(a.ws_ml), h.S_sp + h.S_fix, a.out,
                          lse));
  return LSA_OK;
}

// The kernel's give-up flag, read and cleared (1: a bounded wait gave up since the last call; -1: CUDA error);
// *check receives (and clears) the index-range flag.
int take_attn_timeout(int* check) {
  int v = 0, c = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&c, g_attn_tc_check, sizeof(int)) != cudaSuccess) return -1;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_attn_tc_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  if (c != 0 && cudaMemcpyToSymbol(g_attn_tc_check, &zero, sizeof(int)) != cudaSuccess) return -1;
  *check = c;
  return v;
}

}  // namespace lsa
