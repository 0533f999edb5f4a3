// Sparse absorbed-MQA attention for decode batches: one SM per (query, range of selected rows), two passes.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线": u_t = Attn(h_t, {c_s | s in S_t}) over the
// selected 576-dim bf16 latent rows c_s, shared by all 128 heads, value = the first 512 dims; section "瓶颈一":
// the rows are scattered 1152-byte records, so the achieved gather bandwidth decides the stage.
//
// B200 design.  A work unit is a query b and a contiguous range of at most 8 tiles of 32 of its selected rows;
// the units of a decode batch fill the SMs once (one CTA per SM).  Each unit's rows are read once from HBM and
// its logits are computed once, for all 128 heads:
//   pass 1  gathers whole rows (16-byte cp.async into the 128-byte-swizzled K-major tile), computes the logits
//           S = Q C^T on the tensor cores (Q dims [0, 384) as the A operand in TMEM, dims [384, 576) in shared
//           memory), runs the online softmax, keeps P (bf16) of every tile in shared memory and accumulates
//           O[:, 0:256) += P V[:, 0:256);
//   pass 2  gathers only value dims [256, 512) of the same rows again (512 bytes per row, mostly served by L2)
//           and accumulates O[:, 256:512) += P V[:, 256:512) from the kept P, into the TMEM columns that held S
//           and Q in pass 1, replaying pass 1's (rare) rescales of the running softmax reference.
// A 128 x 512 fp32 accumulator is all of TMEM, so the two value halves cannot both live beside Q and S; the
// second half costs a 512-byte L2 read per row instead of a second CTA that would gather the full rows and
// recompute the logits.  Units of one query are merged by the combine kernel (log-sum-exp weights).
//
// Warp roles (736 threads): warps 0-15 gather (two rows of each tile per warp), 16 and 17 issue the logits
// MMAs of even / odd tiles (16 owns TMEM), 18 issues the P.V MMAs of both passes, 19-22 move Q into TMEM,
// run the softmax (one head per thread = one TMEM lane) and write the output.
#include <algorithm>

#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

using namespace sm100;

__device__ int g_attn2_timeout;  // a bounded wait of the kernel gave up
__device__ int g_attn2_check;    // a selected index was outside [0, L) (the row was clamped)

constexpr int A2_THREADS = 736;
constexpr int A2_GATHER_WARPS = 16;
constexpr int A2_MMA_WARP = 16;   // logits of even tiles; owns TMEM
constexpr int A2_MMA_WARP2 = 17;  // logits of odd tiles
constexpr int A2_PV_WARP = 18;    // O += P V (both passes); warps 19-22: softmax and epilogue
constexpr int A2_T = 32;          // rows per tile
constexpr int A2_H = 128;         // heads (MMA M)
constexpr int A2_KB = 9;          // 64-dim K-blocks of a 576-dim row
constexpr int A2_KB_TQ = 6;       // Q K-blocks held in TMEM (dims [0, 384))
constexpr int A2_KB_SQ = 3;       // Q K-blocks in shared memory (dims [384, 576))
constexpr int A2_MAXT = 8;        // tiles per work unit (P of every tile is kept)
constexpr int A2_STAGES = 3;
constexpr int A2_O_PITCH = 1040;  // epilogue staging: 1 KB per head row + 16 B (rows in different banks)
constexpr int A2_QS_BYTES = A2_KB_SQ * A2_H * 128;          // 48 KB
constexpr int A2_KB_BYTES = A2_T * 128;                     // 4 KB: one 64-dim block of a tile
constexpr int A2_STAGE_BYTES = A2_KB * A2_KB_BYTES;         // 36 KB
constexpr int A2_P_BYTES = (A2_MAXT / 2) * A2_H * 128;      // 64 KB: two tiles' P per 128-byte head row
constexpr int A2_M_BYTES = A2_MAXT * A2_H * 4;              // running softmax reference after each tile
constexpr int A2_IDX_BYTES = A2_MAXT * A2_T * 4;            // the unit's row indices (pass 2 re-reads them)
constexpr int A2_BAR_BYTES = 512;
constexpr int A2_SMEM =
    1024 + A2_QS_BYTES + A2_STAGES * A2_STAGE_BYTES + A2_P_BYTES + A2_M_BYTES + A2_IDX_BYTES + A2_BAR_BYTES;
constexpr uint32_t TM_O0 = 0;    // O value dims [0, 256)
constexpr uint32_t TM_S = 256;   // pass 1: two S buffers of 32 columns
constexpr uint32_t TM_Q = 320;   // pass 1: Q dims [0, 384), two bf16 per column
constexpr uint32_t TM_O1 = 256;  // pass 2: O value dims [256, 512)
constexpr uint32_t IDESC_S = idesc_mma(128, A2_T, 1u, 0u);
constexpr uint32_t IDESC_PV = idesc_mma(128, 256, 1u, 1u);
constexpr float RESCALE_LOG2 = 8.f;
constexpr uint64_t WAIT_NS = 2000000000ull;
static_assert(TM_Q + A2_KB_TQ * 32 == 512, "TMEM columns");
static_assert(A2_SMEM <= 232448, "shared memory");
static_assert(A2_KB_TQ * A2_H * 128 <= A2_STAGE_BYTES + A2_P_BYTES, "Q staging fits stage 2 + the P area");
static_assert(A2_H * A2_O_PITCH <= A2_QS_BYTES + A2_STAGES * A2_STAGE_BYTES, "epilogue staging fits");

struct A2Args {
  const uint16_t* q;   // absorbed queries [B, 128, 576] bf16
  const uint16_t* kv;  // latent cache [L, 576] bf16
  const int32_t* idx;
  int64_t idx_ld;
  const int32_t* count;
  int L;
  int S;  // work units per query; 1: the output is written directly
  float scale_log2;
  uint16_t* out;
  float* lse;
  float* ws_o;   // [B, S, 128, 512] fp32 (S > 1)
  float* ws_ml;  // [B, S, 128, 2]   fp32 (S > 1): softmax reference (log2 units), sum
};

// Bounded wait that also returns false once another role of the CTA has given up.
__device__ __forceinline__ bool wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    #pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_test_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > WAIT_NS) return false;
  }
}

__device__ __forceinline__ void give_up(volatile int* abort_flag) {
  atomicExch(&g_attn2_timeout, 1);
  *abort_flag = 1;
}

// An issuing thread that gave up waits (bounded) until its MMAs have completed, so that TMEM is not released
// under them.
__device__ __forceinline__ void drain_mmas(uint64_t* bar) {
  mma_commit(bar);
  (void)mbar_spin(bar, 0, WAIT_NS);
}

__global__ void __launch_bounds__(A2_THREADS, 1)
    k_sparse_attn_2p(const __grid_constant__ CUtensorMap tm_q, A2Args a) {
  // every global access of this kernel comes after the previous kernel of the stream has completed
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = base;
  unsigned char* st_s = q_s + A2_QS_BYTES;
  unsigned char* p_s = st_s + A2_STAGES * A2_STAGE_BYTES;
  float* m_s = reinterpret_cast<float*>(p_s + A2_P_BYTES);
  int* idx_s = reinterpret_cast<int*>(m_s + A2_MAXT * A2_H);
  uint64_t* bars = reinterpret_cast<uint64_t*>(idx_s + A2_MAXT * A2_T);
  uint64_t* kv_full = bars;                // [3] the gather of a ring tile landed (512 cp.async arrivals)
  uint64_t* kv_empty = kv_full + 3;        // [3] the P.V that read the ring tile completed
  uint64_t* s_full = kv_empty + 3;         // [2] logits of a tile complete
  uint64_t* s_empty = s_full + 2;          // [2] the softmax warps have read the S buffer
  uint64_t* p_full = s_empty + 2;          // [8] P of tile j written (pass 1 rescale of O0 done)
  uint64_t* pv_done = p_full + A2_MAXT;    // [8] pass-1 P.V of tile j complete
  uint64_t* pv1_done = pv_done + A2_MAXT;  // [8] pass-2 P.V of tile j complete
  uint64_t* resc_done = pv1_done + A2_MAXT;  // pass 2: the softmax warps rescaled O1 (one phase per event)
  uint64_t* q_full = resc_done + 1;        // Q's shared-memory K-blocks landed (TMA)
  uint64_t* qst_full = q_full + 1;         // Q's TMEM part landed in the staging area (TMA)
  uint64_t* qt_full = qst_full + 1;        // Q's TMEM part written by the four softmax warps
  uint64_t* drain = qt_full + 1;           // [3] per issuing thread, used only after a give-up
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* resc_any = reinterpret_cast<int*>(tmem_holder + 2);  // [8] some head rescaled O at tile j (pass 1)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.S));
  const int unit = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.S));
  int n = a.count[b];
  n = n < 0 ? 0 : (static_cast<int64_t>(n) > a.idx_ld ? static_cast<int>(a.idx_ld) : n);
  const int T = (n + A2_T - 1) / A2_T;
  const int t0 = static_cast<int>(static_cast<int64_t>(unit) * T / a.S);
  const int t1 = static_cast<int>(static_cast<int64_t>(unit + 1) * T / a.S);
  int ntiles = t1 - t0;
  if (ntiles > A2_MAXT) {  // the host sizes S so that this never happens
    if (tid == 0) atomicExch(&g_attn2_check, 1);
    ntiles = 0;
  }
  const int row0 = t0 * A2_T;
  const int nrows = ntiles > 0 ? min(n, t1 * A2_T) - row0 : 0;

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) {
      mbar_init(&kv_full[i], A2_GATHER_WARPS * 32);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&drain[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
    }
    for (int i = 0; i < A2_MAXT; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&pv1_done[i], 1);
      resc_any[i] = 0;
    }
    mbar_init(resc_done, 4);
    mbar_init(q_full, 1);
    mbar_init(qst_full, 1);
    mbar_init(qt_full, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == A2_MMA_WARP) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < A2_GATHER_WARPS) {
    // ------------------------------------------------------------------ gather
    // Ring tile i < ntiles: whole rows of pass-1 tile i (72 16-byte chunks per row); i >= ntiles: value dims
    // [256, 512) of pass-2 tile i - ntiles (chunks 32..63).  Warp w copies rows 2w, 2w + 1 of each tile, chunk c
    // of row t at K-block c / 8, byte ((c & 7) ^ (t & 7)) * 16 of the row's 128-byte line (128-byte swizzle).
    if (ntiles > 0) {
      if (tid == 0) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(q_full, A2_KB_SQ * A2_H * 128);
        for (int kb = 0; kb < A2_KB_SQ; ++kb)
          tma_load_2d(q_s + kb * A2_H * 128, &tm_q, q_full, 64 * (A2_KB_TQ + kb), b * A2_H);
        // Q dims [0, 384) are staged in stage 2 and the P area until the softmax warps move them into TMEM
        mbar_expect_tx(qst_full, A2_KB_TQ * A2_H * 128);
        for (int kb = 0; kb < A2_KB_TQ; ++kb)
          tma_load_2d(st_s + 2 * A2_STAGE_BYTES + kb * A2_H * 128, &tm_q, qst_full, 64 * kb, b * A2_H);
      }
      const int32_t* rowidx = a.idx + static_cast<int64_t>(b) * a.idx_ld + row0;
      const int my_row = warp * 2 + (lane & 1);  // lanes 0 and 1 hold the indices of the warp's two rows
      auto load_idx = [&](int i) -> int {
        const int rr = i * A2_T + my_row;
        return rr < nrows ? rowidx[rr] : 0;
      };
      int v_a = load_idx(0);
      int v_b = ntiles > 1 ? load_idx(1) : 0;
      const int nring = 2 * ntiles;
      for (int i = 0; i < nring; ++i) {
        const int st = i % A2_STAGES;
        int v;
        if (i < ntiles) {
          const int v_raw = v_a;
          v_a = v_b;
          if (i + 2 < ntiles) v_b = load_idx(i + 2);
          const bool in_range = v_raw >= 0 && v_raw < a.L;
          if (lane < 2 && i * A2_T + my_row < nrows && !in_range) atomicExch(&g_attn2_check, 1);
          v = in_range ? v_raw : (v_raw < 0 ? 0 : a.L - 1);
          if (lane < 2) idx_s[i * A2_T + my_row] = v;  // read back by the same lane in pass 2
        } else {
          v = idx_s[(i - ntiles) * A2_T + my_row];
        }
        // stage 2 holds the Q staging until the softmax warps have moved it into TMEM
        bool ok = i != 2 || wait_ab(qt_full, 0, abort_flag);
        ok = ok && wait_ab(&kv_empty[st], ((i / A2_STAGES) & 1) ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) give_up(abort_flag);
          break;
        }
        unsigned char* dst = st_s + st * A2_STAGE_BYTES;
        if (i < ntiles) {
          #pragma unroll
          for (int k = 0; k < (2 * 72 + 31) / 32; ++k) {
            const int q = lane + 32 * k;
            const int rr = q >= 72 ? 1 : 0, c = q - rr * 72;
            const int t = warp * 2 + rr;
            const int srow = __shfl_sync(0xffffffffu, v, rr);
            if (q < 2 * 72)
              cp_async16(dst + (c >> 3) * A2_KB_BYTES + t * 128 + (((c & 7) ^ (t & 7)) << 4),
                         a.kv + static_cast<int64_t>(srow) * 576 + c * 8);
          }
        } else {
          #pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int c = 32 + lane;
            const int t = warp * 2 + rr;
            const int srow = __shfl_sync(0xffffffffu, v, rr);
            cp_async16(dst + (c >> 3) * A2_KB_BYTES + t * 128 + (((c & 7) ^ (t & 7)) << 4),
                       a.kv + static_cast<int64_t>(srow) * 576 + c * 8);
          }
        }
        cp_async_arrive_noinc(&kv_full[st]);
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
      if (tid == 0) {  // the Q loads have landed before the CTA can exit (they always complete)
        (void)mbar_spin(q_full, 0, WAIT_NS);
        (void)mbar_spin(qst_full, 0, WAIT_NS);
      }
    }
  } else if (warp == A2_MMA_WARP || warp == A2_MMA_WARP2) {
    // ------------------------------------------------------------------ logits MMAs (pass 1)
    // One thread issues about one tcgen05.mma per 30 ns, so the 36 logits MMAs of a tile are issued by two
    // warps by tile parity, each into its own S buffer.
    const int sb = warp == A2_MMA_WARP ? 0 : 1;
    if (ntiles > sb && lane == 0) {
      bool ok = wait_ab(q_full, 0, abort_flag) && wait_ab(qt_full, 0, abort_flag);
      bool issued = false;
      tc_fence_after();
      const uint64_t qdesc = desc_sw128(smem_u32(q_s));
      const uint32_t d = tmem + TM_S + sb * A2_T;
      for (int j = sb; ok && j < ntiles; j += 2) {
        const int st = j % A2_STAGES;
        if (!wait_ab(&kv_full[st], (j / A2_STAGES) & 1, abort_flag) ||
            !wait_ab(&s_empty[sb], ((j >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        fence_proxy_async_smem();  // the cp.async (generic proxy) writes are read by the tensor cores
        tc_fence_after();
        const uint64_t sdesc = desc_sw128(smem_u32(st_s + st * A2_STAGE_BYTES));
        #pragma unroll
        for (int kb = 0; kb < A2_KB_TQ; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ta(d, tmem + TM_Q + kb * 32 + kk * 8, sdesc + ((kb * A2_KB_BYTES + kk * 32) >> 4), IDESC_S,
                       (kb | kk) != 0);
        }
        #pragma unroll
        for (int kb = 0; kb < A2_KB_SQ; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(d, qdesc + ((kb * A2_H * 128 + kk * 32) >> 4),
                    sdesc + (((A2_KB_TQ + kb) * A2_KB_BYTES + kk * 32) >> 4), IDESC_S, 1u);
        }
        mma_commit(&s_full[sb]);
        issued = true;
      }
      if (!ok) {
        give_up(abort_flag);
        if (issued) drain_mmas(&drain[sb]);
      }
    }
  } else if (warp == A2_PV_WARP) {
    // ------------------------------------------------------------------ O += P V (both passes)
    if (ntiles > 0 && lane == 0) {
      bool ok = true, issued = false;
      // pass 1: O0 += P_j V_j[:, 0:256)
      for (int j = 0; ok && j < ntiles; ++j) {
        if (!wait_ab(&p_full[j], 0, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int st = j % A2_STAGES;
        const uint64_t pdesc = desc_sw128(smem_u32(p_s + (j >> 1) * A2_H * 128)) + (((j & 1) * 64) >> 4);
        const uint32_t v_addr = smem_u32(st_s + st * A2_STAGE_BYTES);
        #pragma unroll
        for (int kk = 0; kk < A2_T / 16; ++kk)
          mma_f16(tmem + TM_O0, pdesc + ((kk * 32) >> 4), desc_sw128_mn(v_addr + kk * 16 * 128, A2_KB_BYTES, 1024),
                  IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[st]);
        mma_commit(&pv_done[j]);
        issued = true;
      }
      // pass 2: O1 += P_j V_j[:, 256:512), into the columns of S and Q (every logits MMA has completed and the
      // last S was read: p_full of the last tile was observed above)
      int events = 0;
      for (int j = 0; ok && j < ntiles; ++j) {
        const int i = ntiles + j, st = i % A2_STAGES;
        if (!wait_ab(&kv_full[st], (i / A2_STAGES) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (j > 0 && resc_any[j]) {  // replay pass 1's rescale at this tile on O1
          if (!wait_ab(resc_done, events & 1, abort_flag)) {
            ok = false;
            break;
          }
          ++events;
        }
        fence_proxy_async_smem();
        tc_fence_after();
        const uint64_t pdesc = desc_sw128(smem_u32(p_s + (j >> 1) * A2_H * 128)) + (((j & 1) * 64) >> 4);
        const uint32_t v_addr = smem_u32(st_s + st * A2_STAGE_BYTES + 4 * A2_KB_BYTES);
        #pragma unroll
        for (int kk = 0; kk < A2_T / 16; ++kk)
          mma_f16(tmem + TM_O1, pdesc + ((kk * 32) >> 4), desc_sw128_mn(v_addr + kk * 16 * 128, A2_KB_BYTES, 1024),
                  IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[st]);
        mma_commit(&pv1_done[j]);
      }
      if (!ok) {
        give_up(abort_flag);
        if (issued) drain_mmas(&drain[2]);
      }
    }
  } else {
    // ------------------------------------------------------------------ Q into TMEM, softmax, epilogue
    const int q4 = warp & 3;
    const int h = q4 * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    if (ntiles > 0) {
      // Q row h, dims [0, 384) -> TMEM lane h, columns TM_Q + 32 kb + j hold dims 64 kb + 2j, 64 kb + 2j + 1
      // (read from the TMA staging: chunk c of row h at ((c ^ h) & 7) * 16).  Every wait here is decided
      // warp-wide: the TMEM loads and stores are warp-collective.
      ok = __all_sync(0xffffffffu, wait_ab(qst_full, 0, abort_flag));
      if (ok) {
        #pragma unroll 1
        for (int kb = 0; kb < A2_KB_TQ; ++kb) {
          const unsigned char* src = st_s + 2 * A2_STAGE_BYTES + kb * A2_H * 128 + h * 128;
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
        // the P area doubles as Q staging: all four warps have read it before any P is written
        ok = __all_sync(0xffffffffu, wait_ab(qt_full, 0, abort_flag));
      }
    }
    // ---- pass 1: softmax of each tile's logits, P kept per tile
    for (int i = 0; ok && i < ntiles; ++i) {
      const int sb = i & 1;
      const int nvalid = min(A2_T, nrows - i * A2_T);
      if (!__all_sync(0xffffffffu, wait_ab(&s_full[sb], (i >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(trow + TM_S + sb * A2_T, sr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      float z[A2_T];
      #pragma unroll
      for (int c = 0; c < A2_T; ++c) z[c] = c < nvalid ? __uint_as_float(sr[c]) * a.scale_log2 : -INFINITY;
      float m8[8];
      #pragma unroll
      for (int j = 0; j < 8; ++j) m8[j] = z[j];
      #pragma unroll
      for (int c = 8; c < A2_T; ++c) m8[c & 7] = fmaxf(m8[c & 7], z[c]);
      const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      float alpha = 1.f;
      bool resc = false;
      if (i == 0) {
        m_used = mt;
      } else if (mt > m_used + RESCALE_LOG2) {  // lazy rescale: only when the max grows by more than 2^8
        alpha = ex2_approx(m_used - mt);
        m_used = mt;
        resc = true;
      }
      m_s[i * A2_H + h] = m_used;
      uint32_t pk[A2_T / 2];
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      #pragma unroll
      for (int c = 0; c < A2_T; c += 2) {
        const float p0 = ex2_approx(z[c] - m_used), p1 = ex2_approx(z[c + 1] - m_used);
        s8[(c >> 1) & 7] += p0 + p1;  // the row sum uses the fp32 probabilities (P . V uses them rounded to bf16)
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(p0, p1);
        pk[c / 2] = *reinterpret_cast<const uint32_t*>(&p2);
      }
      l = l * alpha + ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      if (__any_sync(0xffffffffu, resc)) {
        // the warp rescales its O0 rows (alpha = 1 for heads whose reference did not move) once the previous
        // tile's P.V has completed; pass 2 replays it on O1
        if (lane == 0) resc_any[i] = 1;
        if (!__all_sync(0xffffffffu, wait_ab(&pv_done[i - 1], 0, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        #pragma unroll 1
        for (int k = 0; k < 8; ++k) {
          uint32_t o[32];
          tmem_ld32(trow + TM_O0 + 32 * k, o);
          tmem_ld_wait();
          #pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(trow + TM_O0 + 32 * k, o);
        }
        tmem_st_wait();
      }
      // P row h of tile i (32 bf16 = 64 B) -> K elements [32 (i & 1), +32) of head row h in P block i / 2
      unsigned char* prow = p_s + (i >> 1) * A2_H * 128 + h * 128;
      #pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((((i & 1) * 4 + c) ^ (h & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i]);
    }
    if (!ok) give_up(abort_flag);
    // ---- pass 2: the rescales of pass 1, replayed on O1 (every warp takes part; alpha = 1 where nothing moved)
    named_bar_sync(1, 128);  // resc_any and m_s of every softmax warp are visible
    for (int j = 1; ok && j < ntiles; ++j) {
      if (!resc_any[j]) continue;
      if (!__all_sync(0xffffffffu, wait_ab(&pv1_done[j - 1], 0, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float alpha = ex2_approx(m_s[(j - 1) * A2_H + h] - m_s[j * A2_H + h]);
      #pragma unroll 1
      for (int k = 0; k < 8; ++k) {
        uint32_t o[32];
        tmem_ld32(trow + TM_O1 + 32 * k, o);
        tmem_ld_wait();
        #pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
        tmem_st32(trow + TM_O1 + 32 * k, o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(resc_done);
    }
    if (!ok) give_up(abort_flag);
    // ---- epilogue: O row h of both value halves (rows staged in the Q / stage memory, free once the last
    // pass-2 P.V completed; one bulk copy per row)
    const bool have =
        __all_sync(0xffffffffu, ok && ntiles > 0 && wait_ab(&pv1_done[ntiles > 0 ? ntiles - 1 : 0], 0, abort_flag));
    tc_fence_after();
    const int64_t orow = static_cast<int64_t>(b) * A2_H + h;
    unsigned char* srow = q_s + h * A2_O_PITCH;
    if (a.S == 1) {
      const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
      #pragma unroll 1
      for (int k = 0; k < 16; ++k) {  // 16 x 32 columns: O0 then O1
        uint32_t o[32];
        if (have) {
          tmem_ld32(trow + (k < 8 ? TM_O0 + 32 * k : TM_O1 + 32 * (k - 8)), o);
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
      bulk_store_global(a.out + orow * 512, srow, 1024);
      bulk_commit();
      if (a.lse) a.lse[orow] = (have && l > 0.f) ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      const int64_t prow_i = (static_cast<int64_t>(b) * a.S + unit) * A2_H + h;
      #pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        if (half == 1) bulk_wait_read0();  // this row's staging is free again
        #pragma unroll 1
        for (int k = 0; k < 8; ++k) {
          uint32_t o[32];
          if (have) {
            tmem_ld32(trow + (half == 0 ? TM_O0 : TM_O1) + 32 * k, o);
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
        bulk_store_global(a.ws_o + prow_i * 512 + 256 * half, srow, 1024);
        bulk_commit();
      }
      a.ws_ml[prow_i * 2 + 0] = have ? m_used : -INFINITY;
      a.ws_ml[prow_i * 2 + 1] = have ? l : 0.f;
    }
    bulk_wait_read0();  // the staging rows are read before the CTA can exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == A2_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);
int launch_attn_combine(const float* ws_o, const float* ws_ml, int S, int64_t B, void* out, float* lse,
                        cudaStream_t s);

// Work units per query for the two-pass kernel, or 0 when the batch does not fit one wave of it (every unit at
// most 8 tiles of 32 rows, at most 148 units).  Among the unit counts that keep the largest unit smallest, the
// fewest (each unit writes a 256 KB partial that the combine reads back).
int attn2_units(int64_t B, int64_t idx_ld) {
  if (B <= 0) return 0;
  const int64_t T = (idx_ld + A2_T - 1) / A2_T;
  if (T == 0) return 1;
  const int64_t smin = (T + A2_MAXT - 1) / A2_MAXT;
  if (smin * B > 148) return 0;
  int64_t s = std::min<int64_t>(148 / B, (T + 3) / 4);
  s = std::max(s, smin);
  const int64_t tps = (T + s - 1) / s;
  s = (T + tps - 1) / tps;
  return static_cast<int>(s);
}

int launch_sparse_attn_2p(const void* q, const void* kv, int64_t L, const int32_t* idx, int64_t idx_ld,
                          const int32_t* count, int64_t B, float scale, void* out, float* lse, void* ws, int S,
                          cudaStream_t s) {
  CUtensorMap tq;
  int st = make_map(&tq, q, false, B * A2_H, 576, 64, A2_H);
  if (st) return st;
  A2Args a;
  a.q = static_cast<const uint16_t*>(q);
  a.kv = static_cast<const uint16_t*>(kv);
  a.idx = idx;
  a.idx_ld = idx_ld;
  a.count = count;
  a.L = static_cast<int>(L);
  a.S = S;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.ws_o = S > 1 ? static_cast<float*>(ws) : nullptr;
  a.ws_ml = S > 1 ? reinterpret_cast<float*>(static_cast<unsigned char*>(ws) +
                                             align_up(static_cast<size_t>(B) * S * A2_H * 512 * 4, 256))
                  : nullptr;
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_sparse_attn_2p), A2_SMEM));
  LSA_CUDA_TRY(launch_pdl(k_sparse_attn_2p, dim3(static_cast<unsigned>(B * S)), dim3(A2_THREADS), A2_SMEM, s, 0u, tq, a));
  if (S > 1) return launch_attn_combine(a.ws_o, a.ws_ml, S, B, out, lse, s);
  return LSA_OK;
}

// The kernel's flags, read and cleared: give-up (1: a bounded wait gave up since the last call) and device check
// (1: an index outside [0, L) was clamped); -1: CUDA error.
int take_attn2_flags(int* check) {
  int v = 0, c = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn2_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(&c, g_attn2_check, sizeof(int)) != cudaSuccess) return -1;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_attn2_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  if (c != 0 && cudaMemcpyToSymbol(g_attn2_check, &zero, sizeof(int)) != cudaSuccess) return -1;
  *check = c;
  return v;
}

}  // namespace lsa
