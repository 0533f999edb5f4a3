// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "LongCat Sparse Attention（LSA）完全拆解", section "DSA 基线", equation
//   I_{t,s} = sum_j w_{t,j} * ReLU(q^I_{t,j} . k^I_s),
// H_I heads sharing one MQA key, ReLU instead of softmax, bf16 or FP8.
//
// The dense part is the contraction D[s, (b,j)] = k_s . q_{b,j}: keys are the MMA's M side (128 keys per
// tile), the (query, head) pairs of a 256-column chunk are its N side, d_I is K.  With keys on the TMEM
// lanes, the ReLU / weight / head-sum epilogue is a per-thread reduction over one TMEM row segment: no
// cross-thread traffic.  Grid: (query chunk) x (key range); the 256-row query chunk stays in shared
// memory, key tiles stream through a TMA ring.  Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer
// (and TMEM owner), warps 2..9 = epilogue (two warpgroups, one per 128-column half of the chunk).
// TMEM holds two 256-column fp32 accumulators so the epilogue of tile i overlaps the MMAs of tile i+1.
#include "lsa_common.cuh"
#include "sm100.cuh"

namespace lsa {

int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);
int sm_count();

namespace {

using namespace sm100;

constexpr int IX_THREADS = 576;  // producer, MMA, 16 epilogue warps

// Set (never cleared by the kernel) when a bounded wait of this kernel gave up.
__device__ int g_index_tc_timeout;
constexpr int IX_TILE_M = 128;  // keys per tile
constexpr int IX_CHUNK_N = 256; // (query, head) columns per chunk

template <bool FP8>
struct IxCfg {
  static constexpr int KB = FP8 ? 1 : 2;                     // 128-byte K-blocks per 128-dim row
  static constexpr int TILE_BYTES = IX_TILE_M * 128 * KB;    // key tile
  static constexpr int Q_BYTES = IX_CHUNK_N * 128 * KB;      // query chunk
  static constexpr int STAGES = FP8 ? 6 : 4;
  static constexpr int KSTEPS = 4 * KB;                      // MMA instructions per tile (32 B of K each)
  static constexpr uint32_t IDESC = idesc_mma(IX_TILE_M, IX_CHUNK_N, FP8 ? 0u : 1u);
  static constexpr int SMEM = 1024 + Q_BYTES + STAGES * TILE_BYTES + 2048;
};

struct IxArgs {
  const float* w;
  const float* q_scale;
  const float* k_scale;
  const int64_t* q_pos;
  float* scores;
  int64_t ld;
  int L;
  int B;
  int H_I;
  int n_chunks;
  int ntiles;
  int tiles_per_range;
  int split_rows;  // SPLITS > 1: rows between the key matrices that are summed (the exact bf16 split parts)
};

// NP partial sums of w[c] ReLU(D[c]) over the 64 columns of an epilogue thread, partial j over columns
// [64 j / NP, 64 (j + 1) / NP); r holds columns [PW q, PW q + PW).  The 64 weights stay in registers for the whole
// kernel: re-reading them from shared memory every tile (a broadcast load still returns 4 bytes per lane through
// the shared-memory crossbar) costs about as many shared-memory cycles as the tensor cores' operand reads.
template <int NP, int PW>
__device__ __forceinline__ void relu_weighted_piece(const float (&w)[64], const uint32_t (&r)[PW], int q,
                                                    float (&p)[NP]) {
  #pragma unroll
  for (int c = 0; c < PW; ++c) {
    const int col = PW * q + c;
    p[col / (64 / NP)] = fmaf(w[col], fmaxf(__uint_as_float(r[c]), 0.f), p[col / (64 / NP)]);
  }
}

// order-preserving map of floats onto unsigned keys (0 lies below every float) and back
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Grouped block maxima of one tile for one warp (32 keys x the 64 heads of query b): given the G group sums v of
// each key, their max over the warp's keys, then over the tile's four lane quarters through shared memory -- the
// quarter that contributes last writes the G block scores and clears the slot (its next user is four tiles
// later, which no warp reaches before every warp has finished this tile).
template <int G>
__device__ __forceinline__ void block_max_epilogue(const IxArgs& a, float (&v)[G], int s, int b, int64_t qpb,
                                                   int tile, int lane, uint32_t* mx, uint32_t* cnt) {
  constexpr int LG = G == 1 ? 0 : (G == 2 ? 1 : (G == 4 ? 2 : 3));
  const bool valid = b < a.B && s < a.L && s <= qpb;
  #pragma unroll
  for (int g = 0; g < G; ++g) v[g] = valid ? v[g] : -INFINITY;
  // max over the warp's 32 keys of each group sum, as a transposing reduction: each exchange over lane bit
  // 4, 3, 2 halves the values a lane holds (it keeps the half its bit selects), then the remaining lane bits are
  // reduced on one value; lane l ends with group l >> (5 - LG) (G - 1 + 5 - LG shuffles instead of 5 G)
  #pragma unroll
  for (int step = 0; step < LG; ++step) {
    const int half = (G >> step) / 2, off = 16 >> step;
    const bool upper = (lane & off) != 0;
    #pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float send = upper ? v[i] : v[i + half];
      v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
  }
  #pragma unroll
  for (int off = 16 >> LG; off > 0; off >>= 1) v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], off));
  if ((lane & ((32 >> LG) - 1)) == 0) atomicMax(&mx[lane >> (5 - LG)], float_key(v[0]));
  __syncwarp();  // every group's maximum is in before lane 0 counts this quarter
  if (lane == 0) {
    __threadfence_block();
    if (atomicAdd(cnt, 1u) == 3u) {
      #pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint32_t k = atomicExch(&mx[g], 0u);
        if (b < a.B) a.scores[(static_cast<int64_t>(b) * G + g) * a.ld + tile] = key_float(k);
      }
      atomicExch(cnt, 0u);
    }
  }
}

// The chunk's 256 (query, head) weights (times the FP8 query scales) into shared memory, by the 512 epilogue
// threads (e = 0..511), which then synchronise among themselves (named barrier 1).
__device__ __forceinline__ void load_weights(float* wsm, const IxArgs& a, int b0, int e) {
  if (e < IX_CHUNK_N) {
    const int b = b0 + e / a.H_I, j = e % a.H_I;
    float v = 0.f;
    if (b < a.B) v = a.w[static_cast<int64_t>(b) * a.H_I + j] * (a.q_scale ? a.q_scale[static_cast<int64_t>(b) * a.H_I + j] : 1.f);
    wsm[e] = v;
  }
  named_bar_sync(1, IX_THREADS - 64);
}

// SPLITS > 1 (bf16 only): each key is the sum of SPLITS bf16 rows, split_rows apart in the key matrix (the
// exact three-part bf16 split of an fp32 key): a tile's accumulator takes SPLITS consecutive key stages
// before its epilogue.  q_pos == nullptr: no causal mask.
// G > 0 (bf16, H_I = 64): grouped block maxima instead of token scores -- for each query b, group g of index
// heads [8g', ...) (64 / G heads each) and 128-key tile t, scores[(b G + g) ld + t] = the max over the tile's keys
// s <= q_pos[b] of sum_{j in g} w_j ReLU(q_j . k_s) (-inf when none): the block scores of group-wise block
// selection, without writing token scores.
template <bool FP8, int SPLITS, int G>
__global__ void __launch_bounds__(IX_THREADS, 1)
    k_index_score_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q, IxArgs a) {
  static_assert(SPLITS == 1 || !FP8, "split keys are bf16");
  static_assert(G == 0 || (!FP8 && SPLITS == 1 && 64 % G == 0), "grouped block maxima: bf16 keys, H_I = 64");
  // every global access of this kernel comes after the previous kernel of the stream has completed
  sm100::pdl_wait();
  sm100::pdl_launch_dependents();
  using C = IxCfg<FP8>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = base;
  unsigned char* k_s = q_s + C::Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(k_s + C::STAGES * C::TILE_BYTES);
  uint64_t* full = bars;                  // [STAGES]
  uint64_t* empty = bars + C::STAGES;     // [STAGES]
  uint64_t* tfull = bars + 2 * C::STAGES; // [2]
  uint64_t* tempty = tfull + 2;           // [2]
  uint64_t* qfull = tempty + 2;           // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qfull + 1);
  // [256] weights of this chunk's (query, head) pairs, 16-byte aligned: the epilogue reads them as float4
  float* wsm = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(bars) + 256);
  // G > 0: running block maxima (order keys) per [tile mod 4][column group][group] and the number of lane
  // quarters that have contributed per [tile mod 4][column group]
  uint32_t* gmax = reinterpret_cast<uint32_t*>(wsm + IX_CHUNK_N);
  uint32_t* gcnt = gmax + 4 * 4 * 8;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x % a.n_chunks;
  const int range = blockIdx.x / a.n_chunks;
  const int t_begin = range * a.tiles_per_range;
  const int t_end = min(a.ntiles, t_begin + a.tiles_per_range);
  const int n_my = max(0, t_end - t_begin);
  const int qpc = IX_CHUNK_N / a.H_I;  // queries per chunk
  const int b0 = chunk * qpc;

  if (tid == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);
    }
    mbar_init(qfull, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_my > 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_q);
      mbar_expect_tx(qfull, C::Q_BYTES);
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_2d(q_s + kb * IX_CHUNK_N * 128, &tm_q, qfull, kb * (FP8 ? 128 : 64), chunk * IX_CHUNK_N);
      for (int j = 0; j < n_my * SPLITS; ++j) {  // stage j: tile j / SPLITS, split part j % SPLITS
        const int st = j % C::STAGES;
        const uint32_t par = ((j / C::STAGES) & 1) ^ 1;
        if (!mbar_wait(&empty[st], par)) {
          atomicExch(&g_index_tc_timeout, 1);
          abort_flag = 1;
          break;
        }
        mbar_expect_tx(&full[st], C::TILE_BYTES);
        const int row = (t_begin + j / SPLITS) * IX_TILE_M + (j % SPLITS) * a.split_rows;
        unsigned char* dst = k_s + st * C::TILE_BYTES;
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(dst + kb * IX_TILE_M * 128, &tm_k, &full[st], kb * (FP8 ? 128 : 64), row);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_my > 0) {
      bool ok = mbar_wait(qfull, 0);
      // descriptors of the first K step; a step's are these plus its byte offset / 16 (the start-address
      // field holds shared addresses < 256 KB, so the addition never carries out of it)
      const uint64_t q_desc = desc_sw128(smem_u32(q_s));
      const uint64_t k_desc = desc_sw128(smem_u32(k_s));
      for (int i = 0; ok && i < n_my; ++i) {
        const int buf = i & 1;
        if (!mbar_wait(&tempty[buf], ((i >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        #pragma unroll 1
        for (int p = 0; p < SPLITS; ++p) {
          const int j = i * SPLITS + p;
          const int st = j % C::STAGES;
          if (!mbar_wait(&full[st], (j / C::STAGES) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = k_desc + static_cast<uint64_t>((st * C::TILE_BYTES) >> 4);
          #pragma unroll
          for (int k = 0; k < C::KSTEPS; ++k) {
            const int kb = k >> 2, kk = k & 3;
            const uint64_t ad = kd + static_cast<uint64_t>((kb * IX_TILE_M * 128 + kk * 32) >> 4);
            const uint64_t bd = q_desc + static_cast<uint64_t>((kb * IX_CHUNK_N * 128 + kk * 32) >> 4);
            if (FP8)
              mma_f8(tmem + buf * IX_CHUNK_N, ad, bd, C::IDESC, (p | k) != 0);
            else
              mma_f16(tmem + buf * IX_CHUNK_N, ad, bd, C::IDESC, (p | k) != 0);
          }
          mma_commit(&empty[st]);
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
      }
      if (!ok) {
        atomicExch(&g_index_tc_timeout, 1);
        abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..17)
    // warp e handles TMEM lanes 32*(warp % 4) .. +31 (its keys) and chunk columns [64*(e/4), +64)
    if (G > 0 && tid - 64 < 4 * 4 * 8 + 16) gmax[tid - 64] = 0u;  // cleared before the epilogue barrier
    load_weights(wsm, a, b0, tid - 64);  // off the producer's critical path: needed at the first tfull
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int col0 = (ew >> 2) * 64;
    const int nq = 64 / a.H_I;  // queries in this warp's 64 columns (1 or 2)
    const int64_t qpb = (G > 0 && b0 + (col0 >> 6) < a.B) ? a.q_pos[b0 + (col0 >> 6)] : -1;  // grouped: one query
    constexpr int NP = G > 2 ? G : 2;  // partial sums per key: one per group, or one per 32 columns
    constexpr int PW = 16;               // TMEM columns per load
    float wr[64];
    #pragma unroll
    for (int c = 0; c < 64; c += 4) {
      const float4 v = *reinterpret_cast<const float4*>(wsm + col0 + c);
      wr[c] = v.x;
      wr[c + 1] = v.y;
      wr[c + 2] = v.z;
      wr[c + 3] = v.w;
    }
    // FP8: the key scales two tiles ahead (a scale read in the tile that uses it would put a global load's latency
    // in every tile); the queries' positions once
    const int s_lane = t_begin * IX_TILE_M + quarter * 32 + lane;
    auto key_scale = [&](int t) -> float {
      const int sk = s_lane + t * IX_TILE_M;
      return (FP8 && t < n_my && sk < a.L) ? a.k_scale[sk] : 1.f;
    };
    float ks0 = key_scale(0), ks1 = key_scale(1);
    const int bA = b0 + col0 / a.H_I, bB = bA + 1;
    const int64_t posA = (a.q_pos && bA < a.B) ? a.q_pos[bA] : INT64_MAX;
    const int64_t posB = (a.q_pos && nq == 2 && bB < a.B) ? a.q_pos[bB] : INT64_MAX;
    for (int i = 0; i < n_my; ++i) {
      const int buf = i & 1;
      const float ks = ks0;
      ks0 = ks1;
      ks1 = key_scale(i + 2);
      // decided warp-wide: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (i >> 1) & 1))) {
        atomicExch(&g_index_tc_timeout, 1);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * IX_CHUNK_N + col0;
      // PW columns at a time (64 weights + PW columns live; 18 warps leave 96 registers a thread), two or G
      // partial sums
      float p[NP];
      #pragma unroll
      for (int j = 0; j < NP; ++j) p[j] = 0.f;
      #pragma unroll
      for (int q = 0; q < 64 / PW; ++q) {
        uint32_t r[PW];
        tmem_ld16(taddr + PW * q, r);
        tmem_ld_wait();
        if (q == 64 / PW - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);  // the accumulator columns are in registers now
        }
        relu_weighted_piece<NP, PW>(wr, r, q, p);
      }
      const int s = (t_begin + i) * IX_TILE_M + quarter * 32 + lane;
      if constexpr (G > 0) {
        float v[G > 0 ? G : 1];
        #pragma unroll
        for (int g = 0; g < G; ++g) {
          v[g] = 0.f;
          #pragma unroll
          for (int j = g * (NP / G); j < (g + 1) * (NP / G); ++j) v[g] += p[j];
        }
        block_max_epilogue<G>(a, v, s, b0 + (col0 >> 6), qpb, t_begin + i, lane,
                              gmax + ((i & 3) * 4 + (ew >> 2)) * 8, gcnt + (i & 3) * 4 + (ew >> 2));
        continue;
      }
      const float acc0 = p[0], acc1 = p[1];
      if (s < a.L) {
        if (nq == 1) {
          if (bA < a.B) a.scores[static_cast<int64_t>(bA) * a.ld + s] = s > posA ? -INFINITY : (acc0 + acc1) * ks;
        } else {
          if (bA < a.B) a.scores[static_cast<int64_t>(bA) * a.ld + s] = s > posA ? -INFINITY : acc0 * ks;
          if (bB < a.B) a.scores[static_cast<int64_t>(bB) * a.ld + s] = s > posB ? -INFINITY : acc1 * ks;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool FP8, int SPLITS, int G = 0>
int launch_tc(const void* q, const float* q_scale, const float* w, const void* k, const float* k_scale, int64_t B,
              int H_I, int64_t L, const int64_t* q_pos, float* scores, int64_t ld, cudaStream_t s) {
  using C = IxCfg<FP8>;
  CUtensorMap tk, tq;
  const int boxc = FP8 ? 128 : 64;
  int st = make_map(&tk, k, FP8, L * SPLITS, 128, boxc, IX_TILE_M);
  if (st) return st;
  st = make_map(&tq, q, FP8, B * H_I, 128, boxc, IX_CHUNK_N);
  if (st) return st;
  IxArgs a;
  a.w = w;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.q_pos = q_pos;
  a.scores = scores;
  a.ld = ld;
  a.L = static_cast<int>(L);
  a.B = static_cast<int>(B);
  a.H_I = H_I;
  a.n_chunks = static_cast<int>(cdiv(B * H_I, IX_CHUNK_N));
  a.ntiles = static_cast<int>(cdiv(L, IX_TILE_M));
  const int sms = sm_count();
  int ranges = a.n_chunks >= sms ? 1 : static_cast<int>(cdiv(sms, a.n_chunks));
  if (ranges > a.ntiles) ranges = a.ntiles;
  a.tiles_per_range = static_cast<int>(cdiv(a.ntiles, ranges));
  a.split_rows = static_cast<int>(L);
  ranges = static_cast<int>(cdiv(a.ntiles, a.tiles_per_range));
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_index_score_tc<FP8, SPLITS, G>), C::SMEM));
  const int64_t grid = static_cast<int64_t>(a.n_chunks) * ranges;
  return cuda_status(launch_pdl(k_index_score_tc<FP8, SPLITS, G>, dim3(static_cast<unsigned>(grid)), dim3(IX_THREADS),
                                C::SMEM, s, 0u,
                                tk, tq, a));
}

}  // namespace

// ------------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D row-major [rows, cols] map with a (box_cols x box_rows) box and the 128-byte swizzle.
int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows) {
  EncodeTiledFn fn = encoder();
  if (!fn) {
    set_last_error("cuTensorMapEncodeTiled unavailable");
    return LSA_ERR_CUDA;
  }
  const int esz = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * esz)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled failed");
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

int launch_score_simt(const void* q, const float* q_scale, const float* w, const void* k, const float* k_scale,
                      int dtype, int64_t B, int H_I, int d_I, int64_t L, const int64_t* q_pos, float* scores,
                      int64_t ld, cudaStream_t s);

// Tensor-core path for d_I = 128 with 32 or 64 heads; other shapes use the CUDA-core kernel.
int launch_index_score(const void* q, const float* q_scale, const float* w, const void* k, const float* k_scale,
                       int dtype, int64_t B, int H_I, int d_I, int64_t L, const int64_t* q_pos, float* scores,
                       int64_t ld, cudaStream_t s) {
  if (B == 0 || L == 0) return LSA_OK;
  const bool tc = d_I == 128 && (H_I == 32 || H_I == 64) && aligned16(q) && aligned16(k) && L >= IX_TILE_M &&
                  L < (int64_t(1) << 31);
  if (!tc) return launch_score_simt(q, q_scale, w, k, k_scale, dtype, B, H_I, d_I, L, q_pos, scores, ld, s);
  const bool fp8 = dtype == LSA_FP8_E4M3;
  if (fp8) return launch_tc<true, 1>(q, q_scale, w, k, k_scale, B, H_I, L, q_pos, scores, ld, s);
  return launch_tc<false, 1>(q, q_scale, w, k, k_scale, B, H_I, L, q_pos, scores, ld, s);
}

// Grouped block maxima (group-wise block selection): scores[(b G + g) ld + t] for 128-key tiles t; bf16,
// d_I = 128, H_I = 64, G in {1, 2, 4, 8}; the caller checks the shapes.
int launch_block_max_tc(const void* q, const float* w, const void* k, int64_t B, int64_t L, int G,
                        const int64_t* q_pos, float* scores, int64_t ld, cudaStream_t s) {
  if (B == 0 || L == 0) return LSA_OK;
  switch (G) {
    case 1: return launch_tc<false, 1, 1>(q, nullptr, w, k, nullptr, B, 64, L, q_pos, scores, ld, s);
    case 2: return launch_tc<false, 1, 2>(q, nullptr, w, k, nullptr, B, 64, L, q_pos, scores, ld, s);
    case 4: return launch_tc<false, 1, 4>(q, nullptr, w, k, nullptr, B, 64, L, q_pos, scores, ld, s);
    case 8: return launch_tc<false, 1, 8>(q, nullptr, w, k, nullptr, B, 64, L, q_pos, scores, ld, s);
    default: return LSA_ERR_UNSUPPORTED;
  }
}

// Representative scores on the tensor cores: key n = split[n] + split[NB + n] + split[2 NB + n], the exact
// three-part bf16 split of an fp32 representative, so every product with a bf16 query is exact and only
// the fp32 accumulation rounds (as on the CUDA cores).  No causal mask.  Shapes: d_I = 128, H_I in {32, 64},
// NB >= 128; the caller checks them.
int launch_centroid_score_tc(const void* q, const float* w, const void* split, int64_t B, int H_I, int64_t NB,
                             float* scores, int64_t ld, cudaStream_t s) {
  if (B == 0 || NB == 0) return LSA_OK;
  return launch_tc<false, 3>(q, nullptr, w, split, nullptr, B, H_I, NB, nullptr, scores, ld, s);
}

// The kernel's give-up flag, read and cleared (1: a bounded wait gave up since the last call; -1: CUDA error)
int take_index_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_index_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_index_tc_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace lsa
