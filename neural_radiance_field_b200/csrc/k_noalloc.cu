// Occupancy-march compaction that allocates no device memory.
//
// Some callers cannot call cudaMalloc: a host framework that owns all device
// memory through its own allocator (a cudaMalloc would synchronise the device
// and escape its accounting), or a render loop held to a fixed memory budget.
// This entry point needs only its inputs and outputs plus a small scratch array
// that lives in this file as a static device variable, so it allocates nothing.
//
// Scratch: the block partial sums of the exclusive scan over per-ray live
// counts, one int32 per 1024 rays, for at most kNoAllocMaxRays rays (4 KB).
// Every GPU that loads the library holds the array until the process exits.
// All calls share it and it keeps the last call's contents; every entry a call
// reads is written earlier in the same call, so nothing needs clearing. Calls
// whose work overlaps on the GPU (for example on two streams) race on it.
#include <cstdio>
#include <mutex>

#include "nerf_ctx.h"

namespace nerfb {

void set_global_error(const char* msg);

namespace {

constexpr int64_t kNoAllocMaxRays = int64_t(1) << 20;
constexpr int kScanBlock = 1024;

static __device__ __align__(256) int32_t g_noalloc_scan[kNoAllocMaxRays / kScanBlock];

// Device address of g_noalloc_scan on each device, looked up once per device.
std::mutex g_setup_mutex;
int32_t* g_scan_ptr[64] = {};

cudaError_t scratch_for_current_device(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scan_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scan);
    if (e != cudaSuccess) return e;
    g_scan_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scan_ptr[dev];
  return cudaSuccess;
}

// Warp per ray: re-tests every candidate (the same decision as the mask kernel
// that counted them) and writes the live ones, in order, from the ray's offset.
// Writes never pass the next ray's offset.
__global__ void emit_recompute_kernel(const float* __restrict__ o, const float* __restrict__ d,
                                      int64_t R, float near, float step, int K,
                                      const uint32_t* __restrict__ occ,
                                      const int32_t* __restrict__ off,
                                      uint32_t* __restrict__ live) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= R) return;
  int64_t base = off[r];
  const int64_t end = off[r + 1];
  for (int w = 0; w < (K + 31) / 32; ++w) {
    const int k = w * 32 + lane;
    bool is_live = false;
    if (k < K) {
      float x[3], t;
      march_point(o, d, r, near, step, k, x, &t);
      is_live = occupied_at(occ, x[0], x[1], x[2], nullptr);
    }
    const uint32_t m = __ballot_sync(0xffffffffu, is_live);
    const int64_t pos = base + __popc(m & ((1u << lane) - 1u));
    if (is_live && pos < end) live[pos] = ((uint32_t)r << 9) | (uint32_t)k;
    base += __popc(m);
  }
}

nerf_status cuda_error(cudaError_t e, const char* where) {
  char msg[200];
  snprintf(msg, sizeof msg, "nerf_march_compact_noalloc: %s: %s", where, cudaGetErrorString(e));
  set_global_error(msg);
  return NERF_ERR_CUDA;
}

}  // namespace

}  // namespace nerfb

using namespace nerfb;

extern "C" nerf_status nerf_march_compact_noalloc(const float* rays_o, const float* rays_d,
                                                  int64_t n_rays, float near, float step, int K,
                                                  const uint32_t* occupancy, int32_t* out_offsets,
                                                  uint32_t* out_live, void* stream) {
  if (!rays_o || !rays_d || !occupancy || !out_offsets || !out_live || K < 1 || K > 512 ||
      !(step > 0.0f) || n_rays <= 0) {
    set_global_error("nerf_march_compact_noalloc: bad argument");
    return NERF_ERR_INVALID_ARG;
  }
  if (n_rays > kNoAllocMaxRays) {
    // the scan's scratch holds one partial sum per 1024 rays
    char msg[160];
    snprintf(msg, sizeof msg,
             "nerf_march_compact_noalloc: n_rays = %lld exceeds the %lld-ray limit of its "
             "static scratch; split the batch",
             (long long)n_rays, (long long)kNoAllocMaxRays);
    set_global_error(msg);
    return NERF_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)stream;
  int32_t* scan = nullptr;
  cudaError_t e = scratch_for_current_device(&scan);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress of the scratch");
  // The per-ray live counts go into the front of the caller's out_live buffer
  // (it holds n_rays * K >= n_rays entries and is overwritten by the compaction
  // below), are scanned into out_offsets, and the live entries are then written.
  int32_t* counts = reinterpret_cast<int32_t*>(out_live);
  e = launch_march_mask(rays_o, rays_d, n_rays, near, step, K, occupancy, nullptr, counts,
                        nullptr, st);
  if (e != cudaSuccess) return cuda_error(e, "live-count launch");
  e = exclusive_scan(counts, n_rays, out_offsets, scan, st);
  if (e != cudaSuccess) return cuda_error(e, "scan launch");
  emit_recompute_kernel<<<(unsigned)((n_rays + 7) / 8), 256, 0, st>>>(
      rays_o, rays_d, n_rays, near, step, K, occupancy, out_offsets, out_live);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_error(e, "emit launch");
  return NERF_OK;
}
