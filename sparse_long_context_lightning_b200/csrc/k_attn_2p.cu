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
//           S = Q C^T on the tensor cores with all of Q (576 dims = 288 columns) as the A operand in TMEM, and
//           runs the online softmax; P (bf16) of every tile is kept in shared memory.  A stage is released as
//           soon as its logits MMAs complete; each tile's logits are split over two issuing warps (two K-half
//           accumulators), two tiles at a time, and four row tiles are in flight;
//   pass 2  gathers value dims [0, 512) of the same rows again (1 KB per row, mostly served by L2) and
//           accumulates O = P V for both value halves (all 512 TMEM columns), replaying pass 1's (rare)
//           rescales of the running softmax reference.
// A 128 x 512 fp32 accumulator is all of TMEM, so O cannot live beside Q and S: the value dims cost a second
// (L2) read per row instead of a second CTA that would gather the full rows and recompute the logits.  Units of
// one query are merged by the combine kernel (log-sum-exp weights).
//
// Warp roles (768 threads): warps 0-15 gather (two rows of each tile per warp), 16-19 issue the logits MMAs
// (16 and 17 for even tiles, 18 and 19 for odd ones, one K half each; 16 owns TMEM; 19 also issues pass 2's
// P.V MMAs), 20-23 move Q into TMEM and run
// the softmax (one head per thread = one TMEM lane).  The output is written by the twenty gather and softmax
// warps (five per TMEM lane quarter).
#include <cuda_fp16.h>

#include <algorithm>

#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {
namespace {

using namespace sm100;

__device__ int g_attn2_timeout;  // a bounded wait of the kernel gave up
__device__ int g_attn2_check;    // a selected index was outside [0, L) (the row was clamped)

constexpr int A2_THREADS = 768;
constexpr int A2_GATHER_WARPS = 16;
constexpr int A2_LOGIT_WARP0 = 16;  // warps 16-19 issue the logits; 16 owns TMEM
constexpr int A2_PV_WARP = 19;      // also issues pass 2's P.V
constexpr int A2_SOFTMAX_WARP0 = 20;  // warps 20-23
constexpr int A2_T = 32;          // rows per tile
constexpr int A2_H = 128;         // heads (MMA M)
constexpr int A2_KB = 9;          // 64-dim K-blocks of a 576-dim row
constexpr int A2_MAXT = 8;        // tiles per work unit (P of every tile is kept)
constexpr int A2_STAGES = 4;      // tile j uses stage j % 4
constexpr int A2_QSLOTS = 9;      // Q's 64-dim blocks, all staged at once (stages 1-3 and the P area)
constexpr int A2_KB_BYTES = A2_T * 128;                     // 4 KB: one 64-dim block of a tile
constexpr int A2_STAGE_BYTES = A2_KB * A2_KB_BYTES;         // 36 KB
constexpr int A2_QKB_BYTES = A2_H * 128;                    // 16 KB: one 64-dim block of Q
constexpr int A2_P_BYTES = (A2_MAXT / 2) * A2_H * 128;      // 64 KB: two tiles' P per 128-byte head row
constexpr int A2_M_BYTES = A2_MAXT * A2_H * 4;              // running softmax reference after each tile
constexpr int A2_IDX_BYTES = A2_MAXT * A2_T * 4;            // the unit's row indices (pass 2 re-reads them)
constexpr int A2_FIN_BYTES = A2_H * 4 * 2;                  // final sum and reference per head (epilogue)
constexpr int A2_BAR_BYTES = 512;
constexpr int A2_SMEM = 1024 + A2_STAGES * A2_STAGE_BYTES + A2_P_BYTES + A2_M_BYTES + A2_IDX_BYTES + A2_FIN_BYTES +
                        A2_BAR_BYTES;
constexpr uint32_t TM_S = 0;     // pass 1: two S buffers of two 32-column partials [0, 128)
constexpr uint32_t TM_Q = 224;   // pass 1: Q dims [0, 576), two bf16 per column [224, 512)
constexpr uint32_t TM_O0 = 0;    // pass 2: O value dims [0, 256)
constexpr uint32_t TM_O1 = 256;  // pass 2: O value dims [256, 512)
constexpr uint32_t IDESC_S = idesc_mma(128, A2_T, 1u, 0u);
constexpr uint32_t IDESC_PV = idesc_mma(128, 256, 1u, 1u);
constexpr float RESCALE_LOG2 = 8.f;
constexpr uint64_t WAIT_NS = 2000000000ull;
static_assert(TM_Q + A2_KB * 32 == 512 && TM_S + A2_STAGES * A2_T <= TM_Q, "TMEM columns");
static_assert(A2_SMEM <= 232448, "shared memory");
static_assert(A2_STAGE_BYTES + A2_QSLOTS * A2_QKB_BYTES <= A2_STAGES * A2_STAGE_BYTES + A2_P_BYTES,
              "Q staging fits stages 1-3 and the P area");
static_assert(20 * 4096 <= A2_STAGES * A2_STAGE_BYTES, "epilogue staging: 4 KB per output warp in the stages");

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
  __half* ws_o;  // [B, S, 128, 512] fp16 (S > 1): unit u's O, unnormalised, times 2^-e (e per row)
  float* ws_ml;  // [B, S, 128, 2]   fp32 (S > 1): softmax reference + e (log2 units), sum times 2^-e
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

// O rows of this thread's TMEM lane scaled by alpha (both value halves), warp-collective.
__device__ __forceinline__ void rescale_o(uint32_t trow, float alpha) {
  #pragma unroll 1
  for (int k = 0; k < 16; ++k) {
    uint32_t o[32];
    tmem_ld32(trow + 32 * k, o);
    tmem_ld_wait();
    #pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
    tmem_st32(trow + 32 * k, o);
  }
  tmem_st_wait();
}

__global__ void __launch_bounds__(A2_THREADS, 1)
    k_sparse_attn_2p(const __grid_constant__ CUtensorMap tm_q, A2Args a) {
  // Q, the barriers and TMEM are set up while the previous kernel of the stream may still run (programmatic
  // dependent launch): Q is an input the pipeline's previous kernels do not write; every other global access
  // (indices, counts, cache, outputs) comes after pdl_wait()
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* st_s = base;
  unsigned char* p_s = st_s + A2_STAGES * A2_STAGE_BYTES;  // P of every tile; Q staging slots before that
  float* m_s = reinterpret_cast<float*>(p_s + A2_P_BYTES);
  int* idx_s = reinterpret_cast<int*>(m_s + A2_MAXT * A2_H);
  float* fin_s = reinterpret_cast<float*>(idx_s + A2_MAXT * A2_T);  // [128] final sums, [128] final references
  uint64_t* bars = reinterpret_cast<uint64_t*>(fin_s + 2 * A2_H);
  uint64_t* kv_full = bars;                     // [4] a ring tile's gather landed (512 cp.async arrivals)
  uint64_t* kv_empty = kv_full + A2_STAGES;     // [4] the MMAs that read the ring tile completed
  uint64_t* s_full = kv_empty + A2_STAGES;      // [4] logits of a tile complete
  uint64_t* s_empty = s_full + A2_STAGES;       // [4] the softmax warps have read the S buffer
  uint64_t* p_full = s_empty + A2_STAGES;       // [8] P of tile j written
  uint64_t* pv_done = p_full + A2_MAXT;         // [8] pass-2 P.V of tile j complete
  uint64_t* resc_done = pv_done + A2_MAXT;      // pass 2: the softmax warps rescaled O (one phase per event)
  uint64_t* q_slot = resc_done + 1;             // [9] Q's 64-dim block kb landed in its staging slot (TMA)
  uint64_t* qt_full = q_slot + A2_QSLOTS;       // all of Q written into TMEM by the four softmax warps
  uint64_t* drain = qt_full + 1;                // [4] per issuing thread, used only after a give-up
  unsigned char* q_st = st_s + A2_STAGE_BYTES;  // Q staging: block kb at q_st + kb * 16 KB
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* resc_any = reinterpret_cast<int*>(tmem_holder + 2);  // [8] some head's reference moved at tile j
  int* have_s = resc_any + A2_MAXT;                         // the softmax warps completed both passes

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.S));
  const int unit = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.S));
  if (tid == 0) {
    for (int i = 0; i < A2_STAGES; ++i) {
      mbar_init(&kv_full[i], A2_GATHER_WARPS * 32);
      mbar_init(&kv_empty[i], 2);
      mbar_init(&s_full[i], 2);  // buffers 0, 1 used
      mbar_init(&s_empty[i], 4);
      mbar_init(&drain[i], 1);
    }
    for (int i = 0; i < A2_QSLOTS; ++i) mbar_init(&q_slot[i], 1);
    for (int i = 0; i < A2_MAXT; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      resc_any[i] = 0;
    }
    mbar_init(resc_done, 4);
    mbar_init(qt_full, 4);
    *abort_flag = 0;
    *have_s = 0;
    fence_mbar_init();
    // all of Q into the staging slots at once, before the count is known (an empty unit waits for these loads
    // before it exits)
    tma_prefetch_desc(&tm_q);
    for (int kb = 0; kb < A2_QSLOTS; ++kb) {
      mbar_expect_tx(&q_slot[kb], A2_QKB_BYTES);
      tma_load_2d(q_st + kb * A2_QKB_BYTES, &tm_q, &q_slot[kb], 64 * kb, b * A2_H);
    }
  }
  if (warp == A2_LOGIT_WARP0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_launch_dependents();
  // units split the row range by idx_ld (not by count), so the index loads need not wait for the count
  const int T_ld = static_cast<int>((a.idx_ld + A2_T - 1) / A2_T);
  const int t0 = static_cast<int>(static_cast<int64_t>(unit) * T_ld / a.S);
  const int t1 = static_cast<int>(static_cast<int64_t>(unit + 1) * T_ld / a.S);
  const int row0 = t0 * A2_T;
  const int32_t* rowidx = a.idx + static_cast<int64_t>(b) * a.idx_ld + row0;
  const int rows_ld = static_cast<int>(min(static_cast<int64_t>(t1 * A2_T), a.idx_ld)) - row0;  // readable entries
  // gather warps: the raw indices of their rows of the first two tiles, loaded beside the count
  const int my_row = (warp & 15) * 2 + (lane & 1);
  int v_a = 0, v_b = 0;
  if (warp < A2_GATHER_WARPS) {
    if (my_row < rows_ld) v_a = rowidx[my_row];
    if (A2_T + my_row < rows_ld) v_b = rowidx[A2_T + my_row];
  }
  int n = a.count[b];
  n = n < 0 ? 0 : (static_cast<int64_t>(n) > a.idx_ld ? static_cast<int>(a.idx_ld) : n);
  const int nrows = max(0, min(n, t1 * A2_T) - row0);
  int ntiles = (nrows + A2_T - 1) / A2_T;
  if (ntiles > A2_MAXT) {  // the host sizes S so that this never happens
    if (tid == 0) atomicExch(&g_attn2_check, 1);
    ntiles = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);  // this warp's TMEM lane quarter
  const int h = (warp & 3) * 32 + lane;                                          // = its head in the epilogue

  if (warp < A2_GATHER_WARPS) {
    // ------------------------------------------------------------------ gather
    // Ring tile i < ntiles: whole rows of pass-1 tile i (72 16-byte chunks per row); i >= ntiles: value dims
    // [0, 512) of pass-2 tile i - ntiles (chunks 0..63).  Warp w copies rows 2w, 2w + 1 of each tile, chunk c
    // of row t at K-block c / 8, byte ((c & 7) ^ (t & 7)) * 16 of the row's 128-byte line (128-byte swizzle).
    if (ntiles > 0) {
      const int nring = 2 * ntiles;
      for (int i = 0; i < nring; ++i) {
        const int st = i % A2_STAGES;
        int v;
        if (i < ntiles) {
          const int rr = i * A2_T + my_row;
          const int v_raw = v_a;
          v_a = v_b;
          if (i + 2 < ntiles && (i + 2) * A2_T + my_row < rows_ld) v_b = rowidx[(i + 2) * A2_T + my_row];
          const bool in_range = v_raw >= 0 && v_raw < a.L;
          if (lane < 2 && rr < nrows && !in_range) atomicExch(&g_attn2_check, 1);
          v = (rr < nrows && in_range) ? v_raw : (rr < nrows && v_raw >= a.L ? a.L - 1 : 0);
          if (lane < 2) idx_s[rr] = v;  // read back by the same lane in pass 2
        } else {
          v = idx_s[(i - ntiles) * A2_T + my_row];
        }
        // stages 1-3 hold the Q staging until the softmax warps have moved Q into TMEM
        bool ok = (i == 0 || i >= A2_STAGES) || wait_ab(qt_full, 0, abort_flag);
        ok = ok && wait_ab(&kv_empty[st], ((i / A2_STAGES) & 1) ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) give_up(abort_flag);
          break;
        }
        unsigned char* dst = st_s + st * A2_STAGE_BYTES;
        const int nch = i < ntiles ? 72 : 64;  // chunks per row
        #pragma unroll
        for (int k = 0; k < (2 * 72 + 31) / 32; ++k) {
          const int q = lane + 32 * k;
          const int rr = q >= nch ? 1 : 0, c = q - rr * nch;
          const int t = warp * 2 + rr;
          const int srow = __shfl_sync(0xffffffffu, v, rr);
          if (q < 2 * nch)
            cp_async16(dst + (c >> 3) * A2_KB_BYTES + t * 128 + (((c & 7) ^ (t & 7)) << 4),
                       a.kv + static_cast<int64_t>(srow) * 576 + c * 8);
        }
        cp_async_arrive_noinc(&kv_full[st]);
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
  } else if (warp < A2_SOFTMAX_WARP0) {
    // ------------------------------------------------------------------ logits MMAs (pass 1), P.V (pass 2)
    // One thread issues about one tcgen05.mma per 30-50 ns, so a tile's 36 logits MMAs (K = 576 in steps of 16)
    // are split over a warp pair: warp 16 + 2 (j % 2) issues K steps 0-17 and the next warp steps 18-35 of tile j,
    // each into its own partial S accumulator of buffer j % 2 (the softmax adds the two).  Two tiles' logits
    // are in flight, each at about half the latency of one warp issuing all 36.
    const int lw = warp - A2_LOGIT_WARP0;
    const int pair = lw >> 1, khalf = lw & 1;
    if (lane == 0 && ntiles > 0) {
      bool ok = true, issued = false;
      if (ntiles > pair) {
        ok = wait_ab(qt_full, 0, abort_flag);
        tc_fence_after();
        const uint32_t d = tmem + TM_S + pair * 2 * A2_T + khalf * A2_T;
        for (int j = pair; ok && j < ntiles; j += 2) {
          const int st = j % A2_STAGES;
          if (!wait_ab(&kv_full[st], (j / A2_STAGES) & 1, abort_flag) ||
              !wait_ab(&s_empty[pair], ((j >> 1) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();  // the cp.async (generic proxy) writes are read by the tensor cores
          tc_fence_after();
          const uint64_t sdesc = desc_sw128(smem_u32(st_s + st * A2_STAGE_BYTES));
          #pragma unroll
          for (int k = 0; k < 18; ++k) {
            const int ks = khalf * 18 + k, kb = ks >> 2, kk = ks & 3;
            mma_f16_ta(d, tmem + TM_Q + kb * 32 + kk * 8, sdesc + ((kb * A2_KB_BYTES + kk * 32) >> 4), IDESC_S,
                       k != 0);
          }
          mma_commit(&kv_empty[st]);  // the stage is free once both halves' logits have read it
          mma_commit(&s_full[pair]);
          issued = true;
        }
      }
      if (ok && warp == A2_PV_WARP) {
        // pass 2: O[:, 0:256) += P_j V_j[:, 0:256), O[:, 256:512) += P_j V_j[:, 256:512), into the columns of S
        // and Q (every logits MMA has completed and the last S was read: p_full of the last tile)
        int events = 0;
        ok = wait_ab(&p_full[ntiles - 1], 0, abort_flag);
        for (int j = 0; ok && j < ntiles; ++j) {
          const int i = ntiles + j, st = i % A2_STAGES;
          if (!wait_ab(&kv_full[st], (i / A2_STAGES) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (j > 0 && resc_any[j]) {  // replay pass 1's rescale at this tile on O
            if (!wait_ab(resc_done, events & 1, abort_flag)) {
              ok = false;
              break;
            }
            ++events;
          }
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t pdesc = desc_sw128(smem_u32(p_s + (j >> 1) * A2_H * 128)) + (((j & 1) * 64) >> 4);
          const uint32_t v_addr = smem_u32(st_s + st * A2_STAGE_BYTES);
          #pragma unroll
          for (int half = 0; half < 2; ++half) {
            #pragma unroll
            for (int kk = 0; kk < A2_T / 16; ++kk)
              mma_f16(tmem + (half ? TM_O1 : TM_O0), pdesc + ((kk * 32) >> 4),
                      desc_sw128_mn(v_addr + half * 4 * A2_KB_BYTES + kk * 16 * 128, A2_KB_BYTES, 1024), IDESC_PV,
                      (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&kv_empty[st]);  // two arrivals: the stage barrier counts the two logits halves of pass 1
          mma_commit(&kv_empty[st]);
          mma_commit(&pv_done[j]);
          issued = true;
        }
      }
      if (!ok) {
        give_up(abort_flag);
        if (issued) drain_mmas(&drain[lw]);
      }
    }
  } else {
    // ------------------------------------------------------------------ Q into TMEM, softmax (pass 1)
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    if (ntiles > 0) {
      // Q row h, 64-dim block kb -> TMEM lane h, columns TM_Q + 32 kb + j hold dims 64 kb + 2j, 64 kb + 2j + 1,
      // read from its TMA staging slot (chunk c of row h at ((c ^ h) & 7) * 16).  This loop always runs to the end
      // (no break: every Q load has landed before the CTA can exit); its waits are on TMA loads, which always
      // complete, and are bounded all the same.  Every wait is decided warp-wide: the TMEM stores are
      // warp-collective.
      #pragma unroll 1
      for (int kb = 0; kb < A2_KB; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_spin(&q_slot[kb], 0, WAIT_NS))) ok = false;
        const unsigned char* src = q_st + kb * A2_QKB_BYTES + h * 128;
        uint32_t v[32];
        #pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = *reinterpret_cast<const uint4*>(src + ((c ^ (h & 7)) << 4));
          v[4 * c] = x.x;
          v[4 * c + 1] = x.y;
          v[4 * c + 2] = x.z;
          v[4 * c + 3] = x.w;
        }
        if (ok) tmem_st32(trow + TM_Q + 32 * kb, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qt_full);
      // the P area and stages 1-3 double as Q staging: all four warps are past it before any P is written
      ok = ok && __all_sync(0xffffffffu, wait_ab(qt_full, 0, abort_flag));
    }
    for (int i = 0; ok && i < ntiles; ++i) {
      const int sb = i & 1;
      const int nvalid = min(A2_T, nrows - i * A2_T);
      if (!__all_sync(0xffffffffu, wait_ab(&s_full[sb], (i >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[32], sr2[32];
      tmem_ld32(trow + TM_S + sb * 2 * A2_T, sr);  // the two K-half partial logits
      tmem_ld32(trow + TM_S + sb * 2 * A2_T + A2_T, sr2);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      float z[A2_T];
      #pragma unroll
      for (int c = 0; c < A2_T; ++c)
        z[c] = c < nvalid ? (__uint_as_float(sr[c]) + __uint_as_float(sr2[c])) * a.scale_log2 : -INFINITY;
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
      if (__any_sync(0xffffffffu, resc) && lane == 0) resc_any[i] = 1;
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
      // P row h of tile i (32 bf16 = 64 B) -> K elements [32 (i & 1), +32) of head row h in P block i / 2
      unsigned char* prow = p_s + (i >> 1) * A2_H * 128 + h * 128;
      #pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((((i & 1) * 4 + c) ^ (h & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[i]);
    }
    if (!ok) give_up(abort_flag);
    // ---- pass 2: the rescales of pass 1, replayed on O (every warp takes part; alpha = 1 where nothing moved)
    named_bar_sync(1, 128);  // resc_any and m_s of every softmax warp are visible
    for (int j = 1; ok && j < ntiles; ++j) {
      if (!resc_any[j]) continue;
      if (!__all_sync(0xffffffffu, wait_ab(&pv_done[j - 1], 0, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      rescale_o(trow, ex2_approx(m_s[(j - 1) * A2_H + h] - m_s[j * A2_H + h]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(resc_done);
    }
    if (!ok) give_up(abort_flag);
    const bool have = __all_sync(0xffffffffu, ok && ntiles > 0 && wait_ab(&pv_done[ntiles > 0 ? ntiles - 1 : 0], 0, abort_flag));
    fin_s[h] = l;
    fin_s[A2_H + h] = m_used;
    if (have && lane == 0) atomicAdd(have_s, 1);
    if (a.S == 1 && a.lse) {
      a.lse[static_cast<int64_t>(b) * A2_H + h] = (have && l > 0.f) ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
  // ------------------------------------------------------------------ output (gather and softmax warps)
  // Five warps per TMEM lane quarter (four gather warps, one softmax warp) write O's eight 64-column chunks of
  // each row: the output normalised to bf16 (one unit per query), else the unit's partial in fp16.  A partial row
  // is scaled by a power of two 2^-e that brings its largest magnitude into [2^13, 2^14) (fp16 keeps 11
  // significant bits over that whole range); e is folded into the row's softmax reference and sum, so the
  // combine needs no other change.  A warp passes each chunk of its 32 rows through a private 4 KB staging tile
  // (128-byte rows, 16-byte pieces swizzled by row) so that every store instruction writes four whole
  // 128-byte lines.
  if (warp < A2_GATHER_WARPS || warp >= A2_SOFTMAX_WARP0) {
    named_bar_sync(2, (A2_GATHER_WARPS + 4) * 32);  // fin_s, have_s; every gather copy has landed
    if (ntiles == 0 && tid == 0) {
      for (int kb = 0; kb < A2_QSLOTS; ++kb) (void)mbar_spin(&q_slot[kb], 0, WAIT_NS);  // Q loads of an empty unit
    }
    const bool have = *reinterpret_cast<volatile int*>(have_s) == 4;
    const int rank = warp < A2_GATHER_WARPS ? warp / 4 : 4;  // this warp's place among its quarter's five
    unsigned char* stg = st_s + (warp < A2_GATHER_WARPS ? warp : warp - 4) * 4096;
    float* rmax_s = reinterpret_cast<float*>(p_s);  // [5][128]: each rank's largest |O| per row
    const float l = fin_s[h];
    float mul = (have && l > 0.f) ? 1.f / l : 0.f;  // S == 1: normalise
    int e = 0;
    tc_fence_after();
    if (a.S > 1) {
      float mx = 0.f;
      #pragma unroll 1
      for (int c = rank; c < 8; c += 5) {
        if (have) {  // both 32-column halves of the chunk in flight before one wait
          uint32_t o[32], o2[32];
          tmem_ld32(trow + 64 * c, o);
          tmem_ld32(trow + 64 * c + 32, o2);
          tmem_ld_wait();
          #pragma unroll
          for (int k = 0; k < 32; ++k) mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(o[k])), fabsf(__uint_as_float(o2[k]))));
        }
      }
      rmax_s[rank * A2_H + h] = mx;
      named_bar_sync(3, (A2_GATHER_WARPS + 4) * 32);
      float rm = 0.f;
      #pragma unroll
      for (int k = 0; k < 5; ++k) rm = fmaxf(rm, rmax_s[k * A2_H + h]);
      const int E = static_cast<int>((__float_as_uint(rm) >> 23) & 0xFFu) - 127;  // rm in [2^E, 2^(E+1))
      e = min(max(E - 13, -64), 64);
      mul = have ? __uint_as_float(static_cast<uint32_t>(127 - e) << 23) : 0.f;  // 2^-e, exact
      if (rank == 4) {
        const int64_t prow_i = (static_cast<int64_t>(b) * a.S + unit) * A2_H + h;
        a.ws_ml[prow_i * 2 + 0] = have ? fin_s[A2_H + h] + static_cast<float>(e) : -INFINITY;
        a.ws_ml[prow_i * 2 + 1] = have ? l * mul : 0.f;
      }
    }
    #pragma unroll 1
    for (int c = rank; c < 8; c += 5) {
      // this row's 64 columns of chunk c as eight 16-byte pieces of 16-bit values (two loads of 32 columns)
      #pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint32_t o[32];
        if (have) {
          tmem_ld32(trow + 64 * c + 32 * part, o);
          tmem_ld_wait();
        } else {
          #pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t pk[4];
          #pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const float x0 = __uint_as_float(o[8 * k + 2 * q2]) * mul, x1 = __uint_as_float(o[8 * k + 2 * q2 + 1]) * mul;
            if (a.S == 1) {
              const __nv_bfloat162 bb = __floats2bfloat162_rn(x0, x1);
              pk[q2] = *reinterpret_cast<const uint32_t*>(&bb);
            } else {
              const __half2 hh = __floats2half2_rn(x0, x1);
              pk[q2] = *reinterpret_cast<const uint32_t*>(&hh);
            }
          }
          const int piece = 4 * part + k;
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((piece ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      __syncwarp();
      // instruction i writes staging rows 4i .. 4i + 3: lane -> row 4i + lane / 8, 16-byte piece lane % 8
      #pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + (lane >> 3), pc = lane & 7;
        const uint4 v = *reinterpret_cast<const uint4*>(stg + r * 128 + ((pc ^ (r & 7)) << 4));
        const int hr = (warp & 3) * 32 + r;
        if (a.S == 1) {
          *reinterpret_cast<uint4*>(a.out + (static_cast<int64_t>(b) * A2_H + hr) * 512 + 64 * c + 8 * pc) = v;
        } else {
          const int64_t prow_r = (static_cast<int64_t>(b) * a.S + unit) * A2_H + hr;
          *reinterpret_cast<uint4*>(a.ws_o + prow_r * 512 + 64 * c + 8 * pc) = v;
        }
      }
      __syncwarp();  // the staging tile is read before the next chunk overwrites it
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == A2_LOGIT_WARP0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge of one (query, head)'s units: out = sum_u 2^(m_u - m*) O_u / sum_u 2^(m_u - m*) l_u (fp16 partials, their
// scale already folded into m_u and l_u), lse = m* + log2(sum).  Each thread owns 4 columns.  One pass over the
// units in batches of 8 whose loads (references, sums and values) are all issued before any is used; the running
// reference m* moves batch by batch (online rescaling of the accumulators).
constexpr int CB2_BATCH = 8;
__global__ void __launch_bounds__(128) k_attn2_combine(const __half* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                                       int S, uint16_t* __restrict__ out, float* __restrict__ lse) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t bh = blockIdx.x;  // b * 128 + h
  const int b = static_cast<int>(bh / A2_H), h = static_cast<int>(bh % A2_H);
  const int64_t p0 = static_cast<int64_t>(b) * S * A2_H + h;  // row of unit u: p0 + u * 128
  float mstar = -INFINITY, lsum = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int u0 = 0; u0 < S; u0 += CB2_BATCH) {
    uint2 v[CB2_BATCH];
    float2 ml[CB2_BATCH];
    #pragma unroll
    for (int k = 0; k < CB2_BATCH; ++k) {
      if (u0 + k < S) {
        ml[k] = reinterpret_cast<const float2*>(ws_ml)[p0 + (u0 + k) * A2_H];
        v[k] = reinterpret_cast<const uint2*>(ws_o + (p0 + (u0 + k) * A2_H) * 512)[threadIdx.x];
      }
    }
    float mb = -INFINITY;
    #pragma unroll
    for (int k = 0; k < CB2_BATCH; ++k)
      if (u0 + k < S && ml[k].y > 0.f) mb = fmaxf(mb, ml[k].x);
    if (mb == -INFINITY) continue;
    if (mb > mstar) {
      const float r = exp2f(mstar - mb);  // 0 while nothing has been accumulated
      lsum *= r;
      #pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] *= r;
      mstar = mb;
    }
    #pragma unroll
    for (int k = 0; k < CB2_BATCH; ++k) {
      if (u0 + k < S && ml[k].y > 0.f) {
        const float wgt = exp2f(ml[k].x - mstar);
        lsum += wgt * ml[k].y;
        const float2 a0 = __half22float2(*reinterpret_cast<const __half2*>(&v[k].x));
        const float2 a1 = __half22float2(*reinterpret_cast<const __half2*>(&v[k].y));
        acc[0] += wgt * a0.x;
        acc[1] += wgt * a0.y;
        acc[2] += wgt * a1.x;
        acc[3] += wgt * a1.y;
      }
    }
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&lo);
  pk.y = *reinterpret_cast<const uint32_t*>(&hi);
  reinterpret_cast<uint2*>(out + bh * 512)[threadIdx.x] = pk;
  if (lse && threadIdx.x == 0) lse[bh] = lsum > 0.f ? (mstar + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);

// Work units per query for the two-pass kernel, or 0 when the batch does not fit one wave of it (every unit at
// most 8 tiles of 32 rows, at most 148 units).  Among the unit counts that keep the largest unit smallest, the
// fewest (each unit writes a 256 KB partial that the combine reads back).
// Workspace of the two-pass kernel with S units per query: fp16 partials [B, S, 128, 512] | (m, l) [B, S, 128, 2].
size_t attn2_ml_offset(int64_t B, int S) { return align_up(static_cast<size_t>(B) * S * A2_H * 512 * 2, 256); }
size_t attn2_ws_bytes(int64_t B, int S) {
  if (S <= 1) return 0;
  return attn2_ml_offset(B, S) + align_up(static_cast<size_t>(B) * S * A2_H * 2 * 4, 256);
}

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
  a.ws_o = S > 1 ? static_cast<__half*>(ws) : nullptr;
  a.ws_ml = S > 1 ? reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + attn2_ml_offset(B, S)) : nullptr;
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_sparse_attn_2p), A2_SMEM));
  LSA_CUDA_TRY(launch_pdl(k_sparse_attn_2p, dim3(static_cast<unsigned>(B * S)), dim3(A2_THREADS), A2_SMEM, s, 0u, tq, a));
  if (S > 1) {
    LSA_CUDA_TRY(launch_pdl(k_attn2_combine, dim3(static_cast<unsigned>(B * A2_H)), dim3(128), 0, s, 0u,
                            static_cast<const __half*>(a.ws_o), static_cast<const float*>(a.ws_ml), S,
                            static_cast<uint16_t*>(out), lse));
  }
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
