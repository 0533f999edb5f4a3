// Hierarchical (two-stage) index: page scores from the sub-blocks' mean keys, the top-M pages, and the
// candidate rows their tokens form for the token-level re-rank.
//
// "LongCat Sparse Attention（LSA）完全拆解", section "机制三：层级索引（HI）":
//   I_page(t, p) = sum_j w_{t,j} sum_{n in page p} ReLU(q_{t,j} . kmean_n),  pages of P tokens, sub-blocks of
//   Bsub tokens with cached mean keys; the M best pages are recalled; the token score then runs on the
//   recalled tokens only and the final arg topK is taken there.
// The sum over j and the sum over n commute, so a page score is the sum of its sub-blocks' indexer scores:
// the sub-block scores come from the representative scoring (tensor cores, exact bf16 split), this file
// sums them per page and expands the recalled pages; the token stage is the re-rank of k_refine.cu.
#include "lsa_common.cuh"

namespace lsa {

int sm_count();

namespace {

constexpr int PS_THREADS = 256;
constexpr int PE_THREADS = 1024;
constexpr int GR_THREADS = 1024;

// page[b, p] = sum of the scores of page p's complete sub-blocks that end at or before q_pos (sequential
// fp32 sum, ascending sub-block), for pages that start at or before q_pos; -inf for the others.
__global__ void __launch_bounds__(PS_THREADS) k_page_sum(const float* __restrict__ sub, int64_t sub_ld, int64_t nsub,
                                                         int P, int Bsub, int64_t npages,
                                                         const int64_t* __restrict__ q_pos, float* __restrict__ page,
                                                         int64_t page_ld) {
  const int b = blockIdx.y;
  const int64_t p = static_cast<int64_t>(blockIdx.x) * PS_THREADS + threadIdx.x;
  if (p >= npages) return;
  const int64_t qp = q_pos[b];
  float v = -INFINITY;
  if (p * P <= qp) {
    const int64_t nvis = min(nsub, (qp + 1) / Bsub);  // complete sub-blocks entirely visible
    const int per = P / Bsub;
    const int64_t n0 = p * per, n1 = min(n0 + per, nvis);
    const float* row = sub + static_cast<int64_t>(b) * sub_ld;
    v = 0.f;
    for (int64_t n = n0; n < n1; ++n) v += row[n];
  }
  page[static_cast<int64_t>(b) * page_ld + p] = v;
}

// One CTA per query: the candidate row of the token stage -- sink positions, then the recalled tokens
// outside sink and window in ascending order, then the window positions (the row layout of
// lsa_topk_refine).  kept[b, :kcnt[b]] are the recalled pages in ascending order (a top-K row); pages past
// q_pos (kept only when fewer pages are eligible than M) contribute nothing.  The visible tokens of the
// sub-block holding q_pos that is not entirely visible join after the pages when their page was not kept.
__global__ void __launch_bounds__(PE_THREADS) k_page_expand(const int32_t* __restrict__ kept, int64_t kept_ld,
                                                            const int32_t* __restrict__ kcnt, int P, int Bsub,
                                                            int sink, int window,
                                                            const int64_t* __restrict__ q_pos,
                                                            int32_t* __restrict__ cand, int64_t cand_ld,
                                                            int32_t* __restrict__ ccount) {
  __shared__ uint32_t wsum[PE_THREADS / 32];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qp = static_cast<int>(q_pos[b]);
  const int nsink = min(sink, qp + 1);
  const int wlo = window > 0 ? max(qp - window + 1, nsink) : qp + 1;  // window = [wlo, qp]
  const int dlo = nsink, dhi = max(wlo, nsink);                       // dynamic positions [dlo, dhi)
  const int nk = min(static_cast<int>(kept_ld), kcnt[b]);
  int32_t* row = cand + static_cast<int64_t>(b) * cand_ld;
  // the tail sub-block and whether its page is among the kept ones
  const int tlo = ((qp + 1) / Bsub) * Bsub;
  const int tpage = qp / P;
  // this thread's page range (kept pages: one per thread, nk <= PE_THREADS)
  int lo = 0, hi = 0;
  bool has_tpage = false;
  if (tid < nk) {
    const int p = kept[static_cast<int64_t>(b) * kept_ld + tid];
    lo = max(p * P, dlo);
    hi = min(p * P + P, dhi);
    has_tpage = p == tpage;
  }
  const int len = max(0, hi - lo);
  const bool tail_needed = !__syncthreads_or(has_tpage);
  // exclusive scan of the range lengths (kept pages are ascending, so the ranges are too)
  uint32_t incl = static_cast<uint32_t>(len);
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0, total = 0;
  for (int w = 0; w < PE_THREADS / 32; ++w) {
    const uint32_t x = wsum[w];
    wbase += w < warp ? x : 0u;
    total += x;
  }
  const int off = nsink + static_cast<int>(wbase + incl) - len;
  for (int i = 0; i < len; ++i) row[off + i] = lo + i;
  for (int i = tid; i < nsink; i += PE_THREADS) row[i] = i;
  int ndyn = static_cast<int>(total);
  if (tail_needed) {  // after every kept page: they all lie before the tail's page
    const int t0 = max(tlo, dlo), t1 = min(qp + 1, dhi);
    for (int i = t0 + tid; i < t1; i += PE_THREADS) row[nsink + ndyn + (i - t0)] = i;
    ndyn += max(0, t1 - t0);
  }
  const int nwin = qp + 1 - dhi;
  for (int i = tid; i < nwin; i += PE_THREADS) row[nsink + ndyn + i] = dhi + i;
  if (tid == 0) ccount[b] = nsink + ndyn + nwin;
}

// Group-wise block selection, per query b (one CTA): the entries are every group's kept blocks
// (kept[(b G + g) kept_ld + j], j < kcnt) and the local block (all groups), keyed (block << 8 | group bit).  The
// keys are sorted (bitonic, in shared memory); the first key of each block's run is its head, the run's bits
// OR to the block's group mask, and an ordered scan of the heads gives each distinct block its rank.  The
// blocks, ascending, then expand to their tokens with coalesced writes: every block below the local one is
// complete and entirely visible (offset rank * block), the local block is the last and ends at q_pos.
__global__ void __launch_bounds__(PE_THREADS) k_msa_expand(const int32_t* __restrict__ kept, int64_t kept_ld,
                                                           const int32_t* __restrict__ kcnt, int G, int block,
                                                           const int64_t* __restrict__ q_pos,
                                                           int32_t* __restrict__ idx, uint8_t* __restrict__ gmask,
                                                           int64_t idx_ld, int32_t* __restrict__ count) {
  constexpr uint64_t PAD = ~0ull;
  __shared__ uint64_t key[PE_THREADS];
  __shared__ int32_t dblk[PE_THREADS];
  __shared__ uint8_t dmask[PE_THREADS];
  __shared__ uint32_t wsum[PE_THREADS / 32];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qp = static_cast<int>(q_pos[b]);
  const int lb = qp / block;
  const int kl = static_cast<int>(kept_ld);
  const int n_ent = G * kl + 1;  // <= PE_THREADS (checked by the launcher)
  int np = 32;
  while (np < n_ent) np <<= 1;
  if (tid < np) {
    uint64_t k = PAD;
    if (tid == n_ent - 1) {
      k = (static_cast<uint64_t>(lb) << 8) | ((1u << G) - 1u);
    } else if (tid < n_ent - 1) {
      const int g = tid / kl, j = tid % kl;
      if (j < kcnt[b * G + g])
        k = (static_cast<uint64_t>(kept[(static_cast<int64_t>(b) * G + g) * kept_ld + j]) << 8) | (1u << g);
    }
    key[tid] = k;
  }
  __syncthreads();
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int p = tid ^ stride;
      if (tid < np && p > tid) {
        const uint64_t x = key[tid], y = key[p];
        if ((x > y) == ((tid & size) == 0)) {
          key[tid] = y;
          key[p] = x;
        }
      }
      __syncthreads();
    }
  }
  const uint64_t kt = tid < np ? key[tid] : PAD;
  const uint64_t blk = kt >> 8;
  const bool head = kt != PAD && (tid == 0 || (key[tid - 1] >> 8) != blk);
  uint32_t mask = 0u;
  if (head)  // a run holds at most one entry per group plus the local block's
    for (int p = tid; p < np && key[p] != PAD && (key[p] >> 8) == blk; ++p) mask |= static_cast<uint32_t>(key[p] & 0xFFu);
  const uint32_t bal = __ballot_sync(0xffffffffu, head);
  if (lane == 0) wsum[warp] = __popc(bal);
  __syncthreads();
  int before = 0, nd = 0;
  for (int w = 0; w < PE_THREADS / 32; ++w) {
    before += w < warp ? static_cast<int>(wsum[w]) : 0;
    nd += static_cast<int>(wsum[w]);
  }
  if (head) {
    const int rank = before + __popc(bal & ((1u << lane) - 1u));
    dblk[rank] = static_cast<int32_t>(blk);
    dmask[rank] = static_cast<uint8_t>(mask);
  }
  __syncthreads();
  const int total = (nd - 1) * block + (qp + 1 - lb * block);
  int32_t* row = idx + static_cast<int64_t>(b) * idx_ld;
  uint8_t* mrow = gmask + static_cast<int64_t>(b) * idx_ld;
  for (int t = tid; t < total; t += PE_THREADS) {
    const int r = t / block;
    row[t] = dblk[r] * block + (t - r * block);
    mrow[t] = dmask[r];
  }
  if (tid == 0) count[b] = total;
}

// out[b G + g] = q_pos[b] + delta (the per-(query, group) positions of group-wise selection)
__global__ void k_shift_qpos(const int64_t* __restrict__ q_pos, int64_t n, int G, int64_t delta,
                             int64_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = q_pos[i / G] + delta;
}

// Each group's own rows out of a group-wise selection: grows[(b G + g) idx_ld + i] = the i-th entry of
// idx[b, :count[b]] whose gmask has bit g (ascending, as in the union row); gcount[b G + g] of them.  One
// CTA per (query, group): an ordered block scan of the bit.
__global__ void __launch_bounds__(GR_THREADS) k_msa_group_rows(const int32_t* __restrict__ idx,
                                                               const uint8_t* __restrict__ gmask, int64_t idx_ld,
                                                               const int32_t* __restrict__ count, int G,
                                                               int32_t* __restrict__ grows,
                                                               int32_t* __restrict__ gcount) {
  __shared__ uint32_t wsum[GR_THREADS / 32];
  const int bg = blockIdx.x;
  const int b = bg / G, g = bg % G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = min(static_cast<int64_t>(max(count[b], 0)), idx_ld);
  const int32_t* row = idx + static_cast<int64_t>(b) * idx_ld;
  const uint8_t* mrow = gmask + static_cast<int64_t>(b) * idx_ld;
  int32_t* out = grows + static_cast<int64_t>(bg) * idx_ld;
  uint32_t base = 0;
  for (int i0 = 0; i0 < n; i0 += GR_THREADS) {
    const int i = i0 + tid;
    const bool mine = i < n && ((mrow[i] >> g) & 1u);
    const uint32_t bal = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    uint32_t before = 0, total = 0;
    for (int w = 0; w < GR_THREADS / 32; ++w) {
      before += w < warp ? wsum[w] : 0u;
      total += wsum[w];
    }
    if (mine) out[base + before + __popc(bal & ((1u << lane) - 1u))] = row[i];
    base += total;
    __syncthreads();  // wsum is rewritten by the next step
  }
  if (tid == 0) gcount[bg] = static_cast<int32_t>(base);
}

}  // namespace

int launch_page_sum(const float* sub, int64_t sub_ld, int64_t nsub, int P, int Bsub, int64_t npages, int64_t B,
                    const int64_t* q_pos, float* page, int64_t page_ld, cudaStream_t s) {
  if (B == 0 || npages == 0) return LSA_OK;
  const dim3 grid(static_cast<unsigned>(cdiv(npages, PS_THREADS)), static_cast<unsigned>(B));
  k_page_sum<<<grid, PS_THREADS, 0, s>>>(sub, sub_ld, nsub, P, Bsub, npages, q_pos, page, page_ld);
  return cuda_status(cudaGetLastError());
}

int launch_page_expand(const int32_t* kept, int64_t kept_ld, const int32_t* kcnt, int P, int Bsub, int sink,
                       int window, const int64_t* q_pos, int64_t B, int32_t* cand, int64_t cand_ld,
                       int32_t* ccount, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  if (kept_ld > PE_THREADS) return LSA_ERR_INVALID_ARG;
  k_page_expand<<<static_cast<unsigned>(B), PE_THREADS, 0, s>>>(kept, kept_ld, kcnt, P, Bsub, sink, window, q_pos,
                                                                cand, cand_ld, ccount);
  return cuda_status(cudaGetLastError());
}

int launch_msa_expand(const int32_t* kept, int64_t kept_ld, const int32_t* kcnt, int G, int block,
                      const int64_t* q_pos, int64_t B, int32_t* idx, uint8_t* gmask, int64_t idx_ld, int32_t* count,
                      cudaStream_t s) {
  if (B == 0) return LSA_OK;
  if (G * kept_ld + 1 > PE_THREADS) return LSA_ERR_INVALID_ARG;
  k_msa_expand<<<static_cast<unsigned>(B), PE_THREADS, 0, s>>>(kept, kept_ld, kcnt, G, block, q_pos, idx, gmask,
                                                               idx_ld, count);
  return cuda_status(cudaGetLastError());
}

int launch_shift_qpos(const int64_t* q_pos, int64_t B, int G, int64_t delta, int64_t* out, cudaStream_t s) {
  const int64_t n = B * G;
  if (n == 0) return LSA_OK;
  k_shift_qpos<<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, s>>>(q_pos, n, G, delta, out);
  return cuda_status(cudaGetLastError());
}

int launch_msa_group_rows(const int32_t* idx, const uint8_t* gmask, int64_t idx_ld, const int32_t* count, int64_t B,
                          int G, int32_t* grows, int32_t* gcount, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  k_msa_group_rows<<<static_cast<unsigned>(B * G), GR_THREADS, 0, s>>>(idx, gmask, idx_ld, count, G, grows, gcount);
  return cuda_status(cudaGetLastError());
}

}  // namespace lsa
