// lsa_bucket_select_noalloc: bucket / micro-block selection with library-owned scratch.
//
// lsa_bucket_select needs scratch memory (the per-query representative scores and the kept-bucket
// lists) that its caller allocates.  Some callers cannot allocate device memory at the point of the
// call: a plugin running inside a host framework that owns every device allocation, code running on a
// thread that must not enter the CUDA allocator, or a caller with no spare allocation budget left.
// This entry point uses a fixed scratch area that lives in the library image instead: a file-scope
// __device__ array that the CUDA runtime creates on each GPU when the library's module is loaded
// there, and that stays allocated on that GPU until the process exits.
#include <cstdio>
#include <mutex>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per GPU
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_bucket_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_bucket_scratch on the current device.  The name is only a host-side stand-in:
// the address must come from the runtime, once per device, with that device current.  With lazy module
// loading (the CUDA 12 default) this lookup is also what loads the library's module on the device, so
// the first call on a device is the one that creates the 8 MiB buffer there.  The cached address
// belongs to the device's primary context: after cudaDeviceReset on that device it is stale, and
// calling this entry point on that device again is not supported.
int scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) {
    set_last_error("lsa_bucket_select_noalloc: device ordinal out of range");
    return LSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bucket_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    if (p == nullptr) {
      set_last_error("lsa_bucket_select_noalloc: no device address for the static scratch");
      return LSA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LSA_OK;
}

}  // namespace
}  // namespace lsa

extern "C" {

int lsa_bucket_select_noalloc(const void* q_idx, const float* q_scale, const float* w, int dtype, int64_t B, int H_I,
                              int d_I, const float* centroids, int64_t NB, const int32_t* members, int bsz, int M,
                              int sink, int window, int64_t L, const int64_t* q_pos, int32_t* idx, int64_t idx_ld,
                              int32_t* count, void* stream) {
  // the static buffer serves the CUDA-core scoring (no room reserved for the tensor-core path's split copy of
  // the representatives)
  const size_t need = lsa_workspace_size(LSA_OP_BUCKET_MIN, B, NB, M, 0, 0, 0);
  if (need == static_cast<size_t>(-1)) return LSA_ERR_INVALID_ARG;
  if (need > lsa::kNoAllocScratchBytes) {
    char msg[160];
    std::snprintf(msg, sizeof(msg),
                  "lsa_bucket_select_noalloc: needs %zu scratch bytes (B=%lld, NB=%lld, M=%d); the static buffer "
                  "holds %zu",
                  need, static_cast<long long>(B), static_cast<long long>(NB), M, lsa::kNoAllocScratchBytes);
    lsa::set_last_error(msg);
    return LSA_ERR_WORKSPACE;
  }
  if (B == 0) return LSA_OK;
  void* scratch = nullptr;
  const int st = lsa::scratch_for_current_device(&scratch);
  if (st != LSA_OK) return st;
  // Nothing in this scratch has to start at zero: every byte the selection reads is written first
  // within the same call.  The size passed on is the smaller workspace's, not the whole buffer: given
  // more, lsa_bucket_select would take its tensor-core branch (which stores a split copy of the
  // representatives) for the shapes where that copy fits, and this entry point promises the CUDA-core
  // scoring for every shape.
  return lsa_bucket_select(q_idx, q_scale, w, dtype, B, H_I, d_I, centroids, NB, members, bsz, M, sink, window, L,
                           q_pos, idx, idx_ld, count, scratch, need, stream);
}

}  // extern "C"
