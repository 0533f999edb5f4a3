// Two-level tree search over the Flat buckets (the Tree form of bucket selection).
//
// "LSA 稀疏注意力會省顯存嗎", section 二 step 3: the Tree version searches level by level and keeps
// candidates at each level; "超长上下文LSA注意力技术开源", section "Qwen LSA注意力优化原理与核心创新": the
// query scans cluster centres only, then picks buckets.  Level 2 holds the parents (parent p = mean of the
// centres of buckets [p F, min((p+1) F, NB))); the kept parents' children are scored here by a gather (the
// candidates are scattered over the bucket table, so there is no dense tile to put on the tensor cores), the
// rest of the search is the cluster top-K and the Flat expansion.
#include "lsa_common.cuh"
#include "sm100.cuh"

#include <algorithm>

namespace lsa {

int sm_count();
int make_map(CUtensorMap* m, const void* ptr, bool fp8, int64_t rows, int64_t cols, int box_cols, int box_rows);

namespace {

constexpr int TS_THREADS = 256;
constexpr int TS_WARPS = TS_THREADS / 32;
constexpr int TS_PER_CTA = 64;  // candidates per CTA (8 per warp)

// parents[p, d] = (sum over the children of centroids[c, d], in order) / (number of children)
__global__ void k_tree_parents(const float* __restrict__ reps, int64_t NB, int d_I, int F, int64_t NP,
                               float* __restrict__ parents) {
  const int64_t total = NP * d_I;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = e / d_I;
    const int d = static_cast<int>(e % d_I);
    const int64_t c0 = p * F, c1 = min(c0 + F, NB);
    float acc = 0.f;
    for (int64_t c = c0; c < c1; ++c) acc += reps[c * d_I + d];
    parents[e] = acc / static_cast<float>(c1 - c0);
  }
}

// Candidate slot c of query b is child (c mod F) of the (c / F)-th kept parent; its score is the indexer
// formula on the child's centre, in fp32: cscore[b, c] = sum_j w[b,j] max(0, q[b,j,:] . reps[child,:]).
// Slots past the kept parents or the bucket table get -inf and child -1.  One warp per candidate: lane l owns
// heads l and l + 32 (the query staged transposed, [d][64], so the lanes read consecutive words), the
// centre row is staged per warp.
__global__ void __launch_bounds__(TS_THREADS) k_tree_child_score(const uint16_t* __restrict__ q,
                                                                 const float* __restrict__ w, int H_I, int d_I,
                                                                 const float* __restrict__ reps, int64_t NB, int F,
                                                                 const int32_t* __restrict__ kp, int64_t kp_ld,
                                                                 const int32_t* __restrict__ kpc, int64_t n_cand,
                                                                 float* __restrict__ cscore,
                                                                 int32_t* __restrict__ cid, int64_t ldc) {
  __shared__ float qT[128 * 64];
  __shared__ float wsm[64];
  __shared__ float rb[TS_WARPS][128];
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < 128 * 64; e += TS_THREADS) {
    const int d = e >> 6, j = e & 63;
    qT[e] = (j < H_I && d < d_I) ? bf16_bits_to_f32(q[(static_cast<int64_t>(b) * H_I + j) * d_I + d]) : 0.f;
  }
  if (tid < 64) wsm[tid] = tid < H_I ? w[static_cast<int64_t>(b) * H_I + tid] : 0.f;
  __syncthreads();
  const int nkp = kpc[b];
  float* rw = rb[warp];
  for (int i = 0; i < TS_PER_CTA / TS_WARPS; ++i) {
    const int64_t c = static_cast<int64_t>(blockIdx.x) * TS_PER_CTA + i * TS_WARPS + warp;
    if (c >= n_cand) break;  // warp-uniform
    const int64_t slot = c / F;
    int64_t child = -1;
    if (slot < nkp && slot < kp_ld) {
      const int32_t par = kp[static_cast<int64_t>(b) * kp_ld + slot];
      if (par >= 0) child = static_cast<int64_t>(par) * F + c % F;
    }
    if (child < 0 || child >= NB) {  // warp-uniform
      if (lane == 0) {
        cscore[static_cast<int64_t>(b) * ldc + c] = -INFINITY;
        cid[static_cast<int64_t>(b) * ldc + c] = -1;
      }
      continue;
    }
    for (int d = lane; d < d_I; d += 32) rw[d] = reps[child * d_I + d];
    __syncwarp();
    float a0 = 0.f, a1 = 0.f;
    for (int d = 0; d < d_I; ++d) {
      const float r = rw[d];
      a0 = fmaf(qT[d * 64 + lane], r, a0);
      a1 = fmaf(qT[d * 64 + 32 + lane], r, a1);
    }
    float v = wsm[lane] * fmaxf(a0, 0.f) + wsm[32 + lane] * fmaxf(a1, 0.f);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      cscore[static_cast<int64_t>(b) * ldc + c] = v;
      cid[static_cast<int64_t>(b) * ldc + c] = static_cast<int32_t>(child);
    }
    __syncwarp();  // rw is rewritten by the next candidate
  }
}

// kept[b, :] = the bucket ids of the selected candidate slots, in the top-K's order, without the empty
// slots (child -1); kcount[b] of them.  One warp per query, ordered ballot compaction.
__global__ void k_tree_map(const int32_t* __restrict__ kpos, int64_t kpos_ld, const int32_t* __restrict__ kposc,
                           const int32_t* __restrict__ cid, int64_t ldc, int64_t n_cand,
                           int32_t* __restrict__ kept, int64_t kept_ld, int32_t* __restrict__ kcount) {
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int n = static_cast<int>(min(static_cast<int64_t>(max(kposc[b], 0)), kpos_ld));
  int base = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    int32_t bucket = -1;
    if (i < n) {
      const int32_t p = kpos[static_cast<int64_t>(b) * kpos_ld + i];
      if (p >= 0 && p < n_cand) bucket = cid[static_cast<int64_t>(b) * ldc + p];
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, bucket >= 0);
    const int slot = base + __popc(bal & ((1u << lane) - 1u));
    if (bucket >= 0 && slot < kept_ld) kept[static_cast<int64_t>(b) * kept_ld + slot] = bucket;
    base += __popc(bal);
  }
  if (lane == 0) kcount[b] = static_cast<int32_t>(min(static_cast<int64_t>(base), kept_ld));
}

// ---------------------------------------------------------------------------------------------------------------
// The kept parents' children on the tensor cores (F = 64, H_I = 64, d_I = 128).  A kept parent's 64 children are 64
// consecutive rows of the bucket centres, so two kept parents of one query make an M = 128 tile of centre rows,
// loaded by TMA boxes from the centres' exact three-part bf16 split (hi | mid | lo, NB rows apart); the query's 64
// heads are N and d_I = 128 is K.  The three parts accumulate into one fp32 accumulator (every product is exact:
// the query is bf16 and each part holds 8 significand bits of the fp32 centre), so the scores equal the CUDA-core
// scorer's up to the order of the fp32 sums.  Epilogue: one child per thread (TMEM lane), sum_j w_j ReLU(acc_j).
constexpr int TC_F = 64;        // children per parent (rows per TMA box)
constexpr int TC_KB_BYTES = TC_F * 128;                 // 8 KB: one 64-dim block of one parent's children
constexpr int TC_A_BYTES = 3 * 2 * 2 * TC_KB_BYTES;     // 96 KB: [part][64-dim block][parent of the pair]
constexpr int TC_Q_BYTES = 2 * TC_KB_BYTES;             // 16 KB: the query's 64 heads
constexpr int TC_SMEM = 1024 + TC_A_BYTES + TC_Q_BYTES + 512;
constexpr uint32_t TC_IDESC = sm100::idesc_mma(128, 64, 1u, 0u);
__device__ int g_tree_tc_timeout;

struct TreeTcArgs {
  const float* w;
  int64_t NB;
  const int32_t* kp;
  int64_t kp_ld;
  const int32_t* kpc;
  int64_t n_cand;
  float* cscore;
  int32_t* cid;
  int64_t ldc;
};

__global__ void __launch_bounds__(128, 1)
    k_tree_child_tc(const __grid_constant__ CUtensorMap tm_split, const __grid_constant__ CUtensorMap tm_q,
                    TreeTcArgs a) {
  using namespace sm100;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* a_s = base;
  unsigned char* q_s = a_s + TC_A_BYTES;
  float* w_s = reinterpret_cast<float*>(q_s + TC_Q_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(w_s + 64);  // [0] loads landed, [1] MMAs complete
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int b = blockIdx.y;
  const int64_t slot0 = 2 * static_cast<int64_t>(blockIdx.x);
  const int64_t nkp = min(static_cast<int64_t>(max(a.kpc[b], 0)), a.kp_ld);
  int par[2];
  #pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t sl = slot0 + i;
    par[i] = (sl < nkp) ? a.kp[static_cast<int64_t>(b) * a.kp_ld + sl] : -1;
    if (par[i] >= 0 && static_cast<int64_t>(par[i]) * TC_F >= a.NB) par[i] = -1;
  }
  if (tid < 64) w_s[tid] = a.w[static_cast<int64_t>(b) * 64 + tid];
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    if (par[0] >= 0 || par[1] >= 0) {
      const uint32_t bytes = TC_Q_BYTES + (par[0] >= 0 ? 6 : 0) * TC_KB_BYTES + (par[1] >= 0 ? 6 : 0) * TC_KB_BYTES;
      mbar_expect_tx(&bars[0], bytes);
      for (int kb = 0; kb < 2; ++kb) tma_load_2d(q_s + kb * TC_KB_BYTES, &tm_q, &bars[0], 64 * kb, b * 64);
      for (int part = 0; part < 3; ++part)
        for (int kb = 0; kb < 2; ++kb)
          for (int i = 0; i < 2; ++i)
            if (par[i] >= 0)
              tma_load_2d(a_s + ((part * 2 + kb) * 2 + i) * TC_KB_BYTES, &tm_split, &bars[0], 64 * kb,
                          static_cast<int>(part * a.NB + static_cast<int64_t>(par[i]) * TC_F));
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const bool any = par[0] >= 0 || par[1] >= 0;
  bool ok = true;
  if (any && tid == 0) {
    ok = mbar_wait(&bars[0], 0);
    if (ok) {
      tc_fence_after();
      const uint64_t ad = desc_sw128(smem_u32(a_s)), qd = desc_sw128(smem_u32(q_s));
      #pragma unroll
      for (int part = 0; part < 3; ++part) {
        #pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem, ad + ((((part * 2 + kb) * 2) * TC_KB_BYTES + kk * 32) >> 4),
                    qd + ((kb * TC_KB_BYTES + kk * 32) >> 4), TC_IDESC, (part | kb | kk) != 0);
        }
      }
      mma_commit(&bars[1]);
    } else {
      atomicExch(&g_tree_tc_timeout, 1);
      mbar_arrive(&bars[1]);  // nothing was issued: release the epilogue's wait
    }
  }
  // epilogue: thread t = TMEM lane t = child (t & 63) of the kept parent in slot slot0 + (t >> 6)
  const bool done = any && __all_sync(0xffffffffu, mbar_wait(&bars[1], 0));
  tc_fence_after();
  float score = -INFINITY;
  if (done) {
    uint32_t r0[32], r1[32];
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    tmem_ld32(taddr, r0);
    tmem_ld32(taddr + 32, r1);
    tmem_ld_wait();
    float acc0 = 0.f, acc1 = 0.f;
    #pragma unroll
    for (int c = 0; c < 32; ++c) {
      acc0 = fmaf(w_s[c], fmaxf(__uint_as_float(r0[c]), 0.f), acc0);
      acc1 = fmaf(w_s[32 + c], fmaxf(__uint_as_float(r1[c]), 0.f), acc1);
    }
    score = acc0 + acc1;
  }
  const int i = tid >> 6, r = tid & 63;
  const int64_t c = (slot0 + i) * TC_F + r;
  const int64_t child = par[i] >= 0 ? static_cast<int64_t>(par[i]) * TC_F + r : -1;
  const bool valid = done && ok && child >= 0 && child < a.NB;
  if (c < a.n_cand) {
    a.cscore[static_cast<int64_t>(b) * a.ldc + c] = valid ? score : -INFINITY;
    a.cid[static_cast<int64_t>(b) * a.ldc + c] = valid ? static_cast<int32_t>(child) : -1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace

int launch_tree_child_score_tc(const void* q, const float* w, int64_t B, const void* split, int64_t NB,
                               const int32_t* kp, int64_t kp_ld, const int32_t* kpc, int64_t n_cand, float* cscore,
                               int32_t* cid, int64_t ldc, cudaStream_t s) {
  if (B == 0 || n_cand == 0) return LSA_OK;
  CUtensorMap tsplit, tq;
  int st = make_map(&tsplit, split, false, 3 * NB, 128, 64, TC_F);
  if (st) return st;
  st = make_map(&tq, q, false, B * 64, 128, 64, 64);
  if (st) return st;
  TreeTcArgs a;
  a.w = w;
  a.NB = NB;
  a.kp = kp;
  a.kp_ld = kp_ld;
  a.kpc = kpc;
  a.n_cand = n_cand;
  a.cscore = cscore;
  a.cid = cid;
  a.ldc = ldc;
  LSA_CUDA_TRY(func_smem_once(reinterpret_cast<const void*>(k_tree_child_tc), TC_SMEM));
  const dim3 grid(static_cast<unsigned>(cdiv(cdiv(n_cand, TC_F), 2)), static_cast<unsigned>(B));
  k_tree_child_tc<<<grid, 128, TC_SMEM, s>>>(tsplit, tq, a);
  return cuda_status(cudaGetLastError());
}

int take_tree_tc_timeout() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tree_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_tree_tc_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

int launch_tree_parents(const float* reps, int64_t NB, int d_I, int F, float* parents, cudaStream_t s) {
  const int64_t NP = cdiv(NB, F);
  if (NP == 0) return LSA_OK;
  const int64_t blocks = std::min<int64_t>(cdiv(NP * d_I, 256), static_cast<int64_t>(sm_count()) * 8);
  k_tree_parents<<<static_cast<unsigned>(blocks), 256, 0, s>>>(reps, NB, d_I, F, NP, parents);
  return cuda_status(cudaGetLastError());
}

int launch_tree_child_score(const void* q, const float* w, int64_t B, int H_I, int d_I, const float* reps, int64_t NB,
                            int F, const int32_t* kp, int64_t kp_ld, const int32_t* kpc, int64_t n_cand,
                            float* cscore, int32_t* cid, int64_t ldc, cudaStream_t s) {
  if (B == 0 || n_cand == 0) return LSA_OK;
  if (H_I > 64 || d_I > 128) return LSA_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(cdiv(n_cand, TS_PER_CTA)), static_cast<unsigned>(B));
  k_tree_child_score<<<grid, TS_THREADS, 0, s>>>(static_cast<const uint16_t*>(q), w, H_I, d_I, reps, NB, F, kp,
                                                  kp_ld, kpc, n_cand, cscore, cid, ldc);
  return cuda_status(cudaGetLastError());
}

int launch_tree_map(const int32_t* kpos, int64_t kpos_ld, const int32_t* kposc, const int32_t* cid, int64_t ldc,
                    int64_t n_cand, int64_t B, int32_t* kept, int64_t kept_ld, int32_t* kcount, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  k_tree_map<<<static_cast<unsigned>(B), 32, 0, s>>>(kpos, kpos_ld, kposc, cid, ldc, n_cand, kept, kept_ld, kcount);
  return cuda_status(cudaGetLastError());
}

}  // namespace lsa
