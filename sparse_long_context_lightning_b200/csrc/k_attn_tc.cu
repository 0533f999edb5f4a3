// Sparse absorbed-MQA attention over gathered MLA latent rows on tcgen05 tensor cores.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线": u_t = Attn(h_t, {c_s | s in S_t}), the
// 576-dim bf16 latent c_s shared by all 128 heads, value = its first 512 dims; section "瓶颈一": the
// selected 1152-byte rows are scattered, so the kernel is a gather whose memory-level parallelism decides
// the achieved bandwidth.
//
// B200 design.  A 128 x 512 fp32 output accumulator fills all of TMEM (128 lanes x 512 columns), leaving
// no room for the logits, so one work unit (query b, a contiguous split of its selected rows) runs on a
// 2-CTA cluster: CTA r owns output columns [256r, 256r+256) and latent dims D_0 = [0, 256), D_1 =
// [256, 576).  Each CTA gathers only its own part of every selected row (512 or 640 bytes, disjoint), with
// 16-byte cp.async copies from four gather warps into 128-byte-swizzled shared memory (many rows in flight
// per SM; a TMA gather4 per 4 rows x 128 bytes issued too slowly here), computes the partial logits
// S_r = Q[:, D_r] . C[:, D_r]^T, and the two partials are exchanged through distributed shared memory
// (one bulk shared-to-shared copy per warp and tile, completing on the peer's mbarrier).  Both CTAs then hold the same logits,
// run the same online softmax (lazy rescale: O is rescaled only when the running max grows by > 2^8),
// and each accumulates P . V[:, its 256 columns] in TMEM.  The gathered tile serves both MMAs: K-major for
// S = Q C^T and MN-major for O += P V, so no transpose is needed.  Splits of one query are merged by a
// small combine kernel (log-sum-exp weights).
//
// Warp roles (288 threads): warps 0-3 gather, warp 4 issues MMAs (S two tiles ahead of P.V) and owns TMEM,
// warps 5-8 run the softmax (one head per thread = one TMEM lane) and the epilogue.
#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

using namespace sm100;

__device__ int g_attn_tc_timeout;  // set when a bounded wait of the kernel gave up

constexpr int AT_THREADS = 288;  // 4 gather warps, 1 MMA warp, 4 softmax warps
constexpr int AT_GATHER_WARPS = 4;
constexpr int AT_MMA_WARP = 4;
constexpr int AT_SM_TID0 = 160;  // first softmax thread
constexpr int AT_T = 32;   // gathered rows per tile
constexpr int AT_H = 128;  // heads (MMA M)
constexpr int AT_KBQ_MAX = 5;
constexpr int AT_STAGES = 4;
constexpr int AT_Q_BYTES = AT_KBQ_MAX * AT_H * 128;        // 80 KB
constexpr int AT_KB_BYTES = AT_T * 128;                    // 4 KB: one 64-dim block of a tile
constexpr int AT_STAGE_BYTES = AT_KBQ_MAX * AT_KB_BYTES;   // 20 KB
constexpr int AT_P_BYTES = AT_H * 128;                     // 16 KB
constexpr int AT_SX_FLOATS = AT_H * AT_T;                   // 16 KB: partial logits [head][row], 16-byte chunks
                                                            // of a row swizzled by (head & 7)
constexpr uint32_t AT_SX_TX = AT_H * AT_T * 4;              // bytes the peer sends per tile
constexpr int AT_SMEM = 1024 + AT_Q_BYTES + AT_STAGES * AT_STAGE_BYTES + AT_P_BYTES + 3 * AT_SX_FLOATS * 4 + 512;
constexpr uint32_t TM_O = 0;    // TMEM columns [0, 256): O
constexpr uint32_t TM_S = 256;  // TMEM columns [256, 320): two S buffers of 32
constexpr uint32_t IDESC_S = idesc_mma(128, AT_T, 1u, 0u);
constexpr uint32_t IDESC_PV = idesc_mma(128, 256, 1u, 1u);
constexpr float RESCALE_LOG2 = 8.f;

struct AtArgs {
  const uint16_t* kv;  // latent cache [L, 576] bf16
  const int32_t* idx;
  int64_t idx_ld;
  const int32_t* count;
  int B;
  int L;
  int S;  // splits per query
  float scale_log2;
  uint16_t* out;
  float* lse;
  float* ws_o;   // [B, S, 128, 512] fp32 (S > 1)
  float* ws_ml;  // [B, S, 128, 2]   fp32 (S > 1): running max (log2 units), sum
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(AT_THREADS, 1)
    k_sparse_attn_tc(const __grid_constant__ CUtensorMap tm_q, AtArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = base;
  unsigned char* st_s = q_s + AT_Q_BYTES;
  unsigned char* p_s = st_s + AT_STAGES * AT_STAGE_BYTES;
  float* sx_s = reinterpret_cast<float*>(p_s + AT_P_BYTES);
  float* sx_out = sx_s + 2 * AT_SX_FLOATS;  // staging of this CTA's partial logits for the bulk copy
  uint64_t* bars = reinterpret_cast<uint64_t*>(sx_out + AT_SX_FLOATS);  // after two receive buffers + staging
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + AT_STAGES;
  uint64_t* s_full = kv_empty + AT_STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* sx_full = pv_done + 1;  // [2]: the peer's partial logits of tile i landed in buffer i & 1
  uint64_t* q_full = sx_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(q_full + 1);
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t r = cluster_ctarank();
  const uint32_t peer = r ^ 1u;
  const int unit = blockIdx.x >> 1;
  const int b = unit / a.S, split = unit % a.S;
  const int kbq = r ? 5 : 4;
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
      mbar_init(&s_empty[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(&sx_full[0], 1);
    mbar_init(&sx_full[1], 1);
    mbar_init(q_full, 1);
    abort_flag = 0;
    fence_mbar_init();
    // arm both receive buffers for their first tile: each phase completes when the peer's bytes land
    mbar_expect_tx(&sx_full[0], AT_SX_TX);
    mbar_expect_tx(&sx_full[1], AT_SX_TX);
  }
  if (warp == AT_MMA_WARP) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < AT_GATHER_WARPS) {
    // ------------------------------------------------------------------ gather producers
    // Warp w copies rows 8w..8w+7 of every tile: 16-byte cp.async chunks of this CTA's slice of each row,
    // placed in the 128-byte-swizzled K-major layout (chunk c of row t at (c ^ (t & 7)) * 16 in its K-block).
    if (ntiles > 0) {
      if (tid == 0) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(q_full, kbq * AT_H * 128);
        for (int kb = 0; kb < kbq; ++kb)
          tma_load_2d(q_s + kb * AT_H * 128, &tm_q, q_full, 256 * static_cast<int>(r) + 64 * kb, b * AT_H);
      }
      const int32_t* rowidx = a.idx + static_cast<int64_t>(b) * a.idx_ld + row0;
      const uint16_t* kvr = a.kv + 256 * r;  // this CTA's slice starts at latent dim 256 r
      const int cpr = kbq * 8;              // 16-byte chunks per row
      // raw row indices (lane l < 8: row 8w + l) are loaded two tiles ahead and clamped at use
      auto load_idx = [&](int i) -> int {
        const int rr = i * AT_T + warp * 8 + (lane & 7);
        return rr < nrows ? rowidx[rr] : 0;
      };
      int v_a = load_idx(0);
      int v_b = ntiles > 1 ? load_idx(1) : 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % AT_STAGES;
        const int v_raw = v_a;
        v_a = v_b;
        if (i + 2 < ntiles) v_b = load_idx(i + 2);
        if (!mbar_spin(&kv_empty[st], ((i / AT_STAGES) & 1) ^ 1) || abort_flag) {
          if (lane == 0) {
            atomicExch(&g_attn_tc_timeout, 1);
            abort_flag = 1;
          }
          break;
        }
        const int v = v_raw < 0 ? 0 : (v_raw >= a.L ? a.L - 1 : v_raw);
        unsigned char* dst = st_s + st * AT_STAGE_BYTES;
        for (int q = lane; q < 8 * cpr; q += 32) {
          const int rr = q / cpr, c = q - rr * cpr;
          const int row_in_tile = warp * 8 + rr;
          const int srow = __shfl_sync(0xffffffffu, v, rr);  // every lane takes part: rr < 8
          const int kb = c >> 3, c8 = c & 7;
          cp_async16(dst + kb * AT_KB_BYTES + row_in_tile * 128 + ((c8 ^ (row_in_tile & 7)) << 4),
                     kvr + static_cast<int64_t>(srow) * 576 + c * 8);
        }
        cp_async_arrive_noinc(&kv_full[st]);
      }
    }
  } else if (warp == AT_MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    // S = Q C^T runs two tiles ahead of O += P V, so the softmax never waits for its next logits
    if (ntiles > 0 && lane == 0) {
      bool ok = mbar_spin(q_full, 0);
      const uint32_t q_addr = smem_u32(q_s);
      const uint32_t p_addr = smem_u32(p_s);
      auto issue_s = [&](int j) -> bool {
        const int st = j % AT_STAGES, sb = j & 1;
        if (!mbar_spin(&kv_full[st], (j / AT_STAGES) & 1) || !mbar_spin(&s_empty[sb], ((j >> 1) & 1) ^ 1)) return false;
        fence_proxy_async_smem();  // the cp.async (generic proxy) writes are read by the tensor cores
        tc_fence_after();
        const uint32_t s_addr = smem_u32(st_s + st * AT_STAGE_BYTES);
        for (int kb = 0; kb < kbq; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + TM_S + sb * AT_T, desc_sw128(q_addr + kb * AT_H * 128 + kk * 32),
                    desc_sw128(s_addr + kb * AT_KB_BYTES + kk * 32), IDESC_S, (kb | kk) != 0);
        }
        mma_commit(&s_full[sb]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int stj = j % AT_STAGES;
        if (!mbar_spin(p_full, j & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(st_s + stj * AT_STAGE_BYTES);
        #pragma unroll
        for (int kk = 0; kk < AT_T / 16; ++kk)
          mma_f16(tmem + TM_O, desc_sw128(p_addr + kk * 32), desc_sw128_mn(v_addr + kk * 16 * 128, AT_KB_BYTES, 1024),
                  IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[stj]);
        mma_commit(pv_done);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && ntiles > 1) ok = issue_s(1);
      for (int i = 0; ok && i < ntiles; ++i) {
        if (i + 2 < ntiles && !issue_s(i + 2)) ok = false;
        if (ok && !issue_pv(i)) ok = false;
      }
      if (!ok) {
        atomicExch(&g_attn_tc_timeout, 1);
        abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t peer_sx = mapa(smem_u32(sx_s), peer);
    const uint32_t peer_sx_full = mapa(smem_u32(sx_full), peer);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // read S(j) from TMEM, free the buffer, stage this warp's 32 rows in shared memory and send them to the
    // peer's receive buffer j & 1 as one 4 KB bulk copy per warp (all four complete on the peer's mbarrier)
    auto fetch_and_send = [&](int j, uint32_t (&sr)[32]) -> bool {
      const int sb = j & 1;
      if (!mbar_spin(&s_full[sb], (j >> 1) & 1)) return false;
      tc_fence_after();
      tmem_ld32(trow + TM_S + sb * AT_T, sr);
      tmem_ld_wait();
      tc_fence_before();
      // this warp's staging rows are free once its previous bulk copy has read them
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      float4* row = reinterpret_cast<float4*>(sx_out + h * AT_T);
      #pragma unroll
      for (int c = 0; c < AT_T / 4; ++c)
        row[c ^ (h & 7)] = make_float4(__uint_as_float(sr[4 * c]), __uint_as_float(sr[4 * c + 1]),
                                       __uint_as_float(sr[4 * c + 2]), __uint_as_float(sr[4 * c + 3]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t off = static_cast<uint32_t>((sb * AT_SX_FLOATS + q4 * 32 * AT_T) * 4);
        bulk_store_peer(peer_sx + off, sx_out + q4 * 32 * AT_T, 32 * AT_T * 4, peer_sx_full + sb * 8);
        bulk_commit();
      }
      return true;
    };
    uint32_t sr[32];
    if (ntiles > 0) ok = fetch_and_send(0, sr);
    for (int i = 0; ok && i < ntiles; ++i) {
      const int sb = i & 1;
      const int nvalid = min(AT_T, nrows - i * AT_T);
      // the peer's partial logits of tile i.  Its receive buffer for tile i+1 is free: the peer read tile
      // i-1 from it before sending tile i, which has arrived.
      if (!mbar_wait_cluster(&sx_full[sb], (i >> 1) & 1)) {
        ok = false;
        break;
      }
      const float4* sxrow = reinterpret_cast<const float4*>(sx_s + sb * AT_SX_FLOATS + h * AT_T);
      float sp[AT_T];
      #pragma unroll
      for (int c = 0; c < AT_T / 4; ++c) {
        const float4 v = sxrow[c ^ (h & 7)];
        sp[4 * c] = v.x;
        sp[4 * c + 1] = v.y;
        sp[4 * c + 2] = v.z;
        sp[4 * c + 3] = v.w;
      }
      // re-arm buffer sb for tile i+2 (before this CTA sends tile i+1, so before the peer can send i+2)
      if (tid == AT_SM_TID0 && i + 2 < ntiles) mbar_expect_tx(&sx_full[sb], AT_SX_TX);
      uint32_t sr_next[32];
      if (i + 1 < ntiles && !fetch_and_send(i + 1, sr_next)) {
        ok = false;
        break;
      }
      float z[AT_T];
      float mt = -INFINITY;
      #pragma unroll
      for (int c = 0; c < AT_T; ++c) {
        const float sfull = __uint_as_float(sr[c]) + sp[c];
        z[c] = c < nvalid ? sfull * a.scale_log2 : -INFINITY;
        mt = fmaxf(mt, z[c]);
      }
      float alpha = 1.f;
      bool resc = false;
      if (i == 0) {
        m_used = mt;
      } else if (mt > m_used + RESCALE_LOG2) {
        alpha = exp2f(m_used - mt);
        m_used = mt;
        resc = true;
      }
      uint32_t pk[AT_T / 2];
      float psum = 0.f;
      #pragma unroll
      for (int c = 0; c < AT_T; c += 2) {
        const float p0 = exp2f(z[c] - m_used), p1 = exp2f(z[c + 1] - m_used);
        psum += p0 + p1;  // the row sum uses the fp32 probabilities (P . V uses them rounded to bf16)
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(p0, p1);
        pk[c / 2] = *reinterpret_cast<const uint32_t*>(&p2);
      }
      l = l * alpha + psum;
      // the previous P . V has finished: the P buffer is free and O is stable
      if (i > 0 && !mbar_spin(pv_done, (i - 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (resc) {
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
      #pragma unroll
      for (int c = 0; c < 32; ++c) sr[c] = sr_next[c];
    }
    if (!ok) {
      atomicExch(&g_attn_tc_timeout, 1);
      abort_flag = 1;
    }
    // ---- epilogue
    if (lane == 0) bulk_wait_read0();  // this warp's last outgoing copy has read its staging rows
    const bool have = ok && ntiles > 0 && mbar_spin(pv_done, (ntiles - 1) & 1);
    tc_fence_after();
    const int64_t orow = static_cast<int64_t>(b) * AT_H + h;
    if (a.S == 1) {
      const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
      uint16_t* dst = a.out + orow * 512 + 256 * r;
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
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * k);
        #pragma unroll
        for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      if (r == 0 && a.lse) a.lse[orow] = (have && l > 0.f) ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      const int64_t prow_i = (static_cast<int64_t>(b) * a.S + split) * AT_H + h;
      float* dst = a.ws_o + prow_i * 512 + 256 * r;
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
        float4* d4 = reinterpret_cast<float4*>(dst + 32 * k);
        #pragma unroll
        for (int c = 0; c < 8; ++c)
          d4[c] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]), __uint_as_float(o[4 * c + 2]),
                              __uint_as_float(o[4 * c + 3]));
      }
      if (r == 0) {
        a.ws_ml[prow_i * 2 + 0] = have ? m_used : -INFINITY;
        a.ws_ml[prow_i * 2 + 1] = have ? l : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == AT_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the splits of one (query, head): LSE-weighted sum of the partial outputs.
__global__ void __launch_bounds__(128) k_attn_combine(const float* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                                      int S, uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int64_t bh = blockIdx.x;  // b * 128 + h
  const int b = static_cast<int>(bh / AT_H), h = static_cast<int>(bh % AT_H);
  float mstar = -INFINITY;
  for (int s = 0; s < S; ++s) {
    const int64_t pi = (static_cast<int64_t>(b) * S + s) * AT_H + h;
    if (ws_ml[pi * 2 + 1] > 0.f) mstar = fmaxf(mstar, ws_ml[pi * 2]);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  if (mstar != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const int64_t pi = (static_cast<int64_t>(b) * S + s) * AT_H + h;
      const float ls = ws_ml[pi * 2 + 1];
      if (!(ls > 0.f)) continue;
      const float wgt = exp2f(ws_ml[pi * 2] - mstar);
      lsum += wgt * ls;
      const float4 v = reinterpret_cast<const float4*>(ws_o + pi * 512)[threadIdx.x];
      acc.x += wgt * v.x;
      acc.y += wgt * v.y;
      acc.z += wgt * v.z;
      acc.w += wgt * v.w;
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

int splits_for(int64_t B) {
  int64_t s = 148 / (2 * (B > 0 ? B : 1));
  if (s < 1) s = 1;
  if (s > 32) s = 32;
  return static_cast<int>(s);
}

}  // namespace

int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);
int launch_attn_simt(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                     const int32_t* count, int64_t B, int H, float scale, void* out, float* lse, cudaStream_t s);

size_t sparse_attn_ws_bytes(int64_t B, int64_t, int H) {
  if (H != AT_H) return 0;
  const int S = splits_for(B);
  if (S == 1) return 0;
  const size_t o = align_up(static_cast<size_t>(B) * S * AT_H * 512 * 4, 256);
  return o + align_up(static_cast<size_t>(B) * S * AT_H * 2 * 4, 256);
}

int attn_launches_per_call(int64_t B, int H) { return (H == AT_H && splits_for(B) > 1) ? 2 : 1; }

int launch_sparse_attn(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                       const int32_t* count, int64_t B, int H, float scale, void* out, float* lse, void* ws,
                       size_t ws_bytes, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  if (H != AT_H || L >= (int64_t(1) << 31)) return launch_attn_simt(q, kv, L, idx, idx_ld, count, B, H, scale, out, lse, s);
  const int S = splits_for(B);
  const size_t need = sparse_attn_ws_bytes(B, idx_ld, H);
  if (S > 1 && (ws == nullptr || !aligned256(ws) || ws_bytes < need)) return LSA_ERR_WORKSPACE;
  CUtensorMap tq;
  const int st = make_map(&tq, q, false, B * AT_H, 576, 64, AT_H);
  if (st) return st;
  AtArgs a;
  a.kv = static_cast<const uint16_t*>(kv);
  a.idx = idx;
  a.idx_ld = idx_ld;
  a.count = count;
  a.B = static_cast<int>(B);
  a.L = static_cast<int>(L);
  a.S = S;
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
  k_sparse_attn_tc<<<static_cast<unsigned>(grid), AT_THREADS, AT_SMEM, s>>>(tq, a);
  LSA_CUDA_TRY(cudaGetLastError());
  if (S > 1) {
    k_attn_combine<<<static_cast<unsigned>(B * AT_H), 128, 0, s>>>(a.ws_o, a.ws_ml, S, a.out, lse);
    LSA_CUDA_TRY(cudaGetLastError());
  }
  return LSA_OK;
}

}  // namespace lsa
