// Mean pooling for callers that cannot allocate device memory.
//
// jepa_b200_op_mean_pool needs a scratch buffer for its partial column sums
// and grows one with cudaMalloc on demand.  Some callers cannot do that:
// serving loops that run under a fixed device-memory budget, code that must
// never stall the device (cudaMalloc may synchronise it), and hosts whose
// device allocator belongs to another framework.  For them this file keeps
// the scratch in a fixed file-scope __device__ array that every GPU loading
// the library holds until the process exits, and exposes
// jepa_b200_op_mean_pool_noalloc, which allocates nothing.
#include <mutex>

#include "internal.h"

namespace {

// Partial sums of at most kNoAllocPoolFloats floats: B * 32 * D <= 2^20,
// i.e. B * D <= 32768 (4 MiB per device).
constexpr int kNoAllocPoolFloats = 1 << 20;

static __device__ __align__(256) float g_noalloc_pool_scratch[kNoAllocPoolFloats];

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array for the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return JEPA_B200_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_pool_scratch) != cudaSuccess || !p) return JEPA_B200_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return JEPA_B200_OK;
}

}  // namespace

extern "C" {

int jepa_b200_op_mean_pool_noalloc(const float* y, int B, int ntok, int D, int first, float* out, void* stream) {
  if (!y || !out) return JEPA_B200_ERR_ARG;
  if (B < 1 || D < 1 || first < 0 || first >= ntok || B > 65535) return JEPA_B200_ERR_SHAPE;
  const long long per_col = jb::mean_pool_partial_floats(1, 1);  // partial sums per (clip, column)
  if (static_cast<long long>(B) * D * per_col > kNoAllocPoolFloats) return JEPA_B200_ERR_SHAPE;
  float* scratch = nullptr;
  const int s = noalloc_scratch(&scratch);
  if (s != JEPA_B200_OK) return s;
  // every partial sum the final kernel reads is written by this call first,
  // so the array's previous contents never matter
  return jb::launch_mean_pool(y, B, ntok, D, first, scratch, out, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
