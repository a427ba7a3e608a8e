// Internal interface of the marching scene functions (k_march.cu).
#pragma once

#include "nerf_internal.cuh"

namespace nerfb {

// ------------------------------------------------------------------ occupancy
// Shared by every kernel that decides whether a march candidate is live, so that
// they all take the same decision.

// Voxel of one coordinate by exact comparison with the boundaries b_v = -1.5 +
// v * 3/128 (exact in fp32): returns -1 outside [-1.5, 1.5).
__device__ __forceinline__ int voxel_axis(float x) {
  if (!(x >= -1.5f) || !(x < 1.5f)) return -1;
  int v = (int)floorf(fmul(fadd(x, 1.5f), 42.666666666666664f));
  v = v < 0 ? 0 : (v > 127 ? 127 : v);
  if (x < fsub(fmul((float)v, 0.0234375f), 1.5f)) --v;
  else if (v < 127 && x >= fsub(fmul((float)(v + 1), 0.0234375f), 1.5f)) ++v;
  return v;
}

__device__ __forceinline__ bool occupied_at(const uint32_t* __restrict__ occ, float x0, float x1,
                                            float x2, int* vox) {
  const int a = voxel_axis(x0), b = voxel_axis(x1), c = voxel_axis(x2);
  if (a < 0 || b < 0 || c < 0) return false;
  const int idx = (a * 128 + b) * 128 + c;
  if (vox) *vox = idx;
  return (__ldg(occ + (idx >> 5)) >> (idx & 31)) & 1u;
}

__device__ __forceinline__ void march_point(const float* o, const float* d, int64_t r, float near,
                                            float step, int k, float* x, float* t) {
  *t = fadd(near, fmul((float)k, step));
#pragma unroll
  for (int c = 0; c < 3; ++c) x[c] = fadd(o[r * 3 + c], fmul(*t, d[r * 3 + c]));
}

// Candidates [*klo, *khi] of ray r that can lie in [-1.5, 1.5)^3; every other
// candidate's point is outside it, so the exact test above would reject it. The
// interval comes from the slabs of the cube expanded by 1e-4 on every side (far
// more than the fp32 error of a point, about 1e-6 here), in fp32, padded by one
// candidate on each end. Empty (klo > khi) when the ray misses the box.
__device__ __forceinline__ void march_window(const float* o, const float* d, int64_t r,
                                             float near, float step, int K, int* klo, int* khi) {
  constexpr float B = 1.5f + 1e-4f;
  float tin = -INFINITY, tout = INFINITY;
  bool miss = false;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const float oc = o[r * 3 + c], dc = d[r * 3 + c];
    if (dc != 0.0f) {
      const float t0 = (-B - oc) / dc, t1 = (B - oc) / dc;
      tin = fmaxf(tin, fminf(t0, t1));
      tout = fminf(tout, fmaxf(t0, t1));
    } else if (!(oc >= -B && oc <= B)) {
      miss = true;
    }
  }
  if (miss || !(tin <= tout)) {
    *klo = K;
    *khi = -1;
    return;
  }
  float a = (tin - near) / step, b = (tout - near) / step;
  a = fminf(fmaxf(a, -2.0f), (float)K + 2.0f);      // also maps +-inf and keeps NaN out
  b = fminf(fmaxf(b, -2.0f), (float)K + 2.0f);
  *klo = max(0, (int)floorf(a) - 1);
  *khi = min(K - 1, (int)ceilf(b) + 1);
}

struct HashGridInfo {
  int res[16];
  int offset[16];
  int direct[16];
  int64_t entries;
};
HashGridInfo hash_grid_info();

struct ShConst { float k[16]; };
ShConst sh_constants();

// Workspace of one ray chunk.
struct MarchWs {
  int64_t cap = 0;            // live-entry capacity
  uint32_t* mask = nullptr;   // [chunk][16]
  int32_t* count = nullptr;   // [chunk]
  int32_t* off = nullptr;     // [chunk + 1]
  int32_t* scan_tmp = nullptr;  // [2048]
  uint32_t* live = nullptr;   // [cap] (ray_in_chunk << 9) | k
  float* val = nullptr;       // [cap][4] activated (r, g, b, sigma)
  int32_t* cell = nullptr;    // [cap]
  int32_t* order = nullptr;   // [cap]
  int32_t* cell_hist = nullptr;  // [4096] followed by cell_fill [4096]
  int32_t* cell_fill = nullptr;
  int32_t* cell_off = nullptr;   // [4097]
  int4* items = nullptr;         // [cap / 128 + 4096]: (cell, first order index, points, 0)
  int32_t* n_items = nullptr;    // [1]
};

struct MarchArgs {
  int model;
  const float* o;
  const float* d;
  int64_t r0, R;              // ray chunk [r0, r0 + R)
  float near, step, ert_T;
  int K;
  const uint32_t* occ;
  const float* cell_w;
  const uint16_t* hash_table;
  const float* hash_mlp;
  ShConst sh;
  float* rgb;
  float* depth;
  float* acc;
  unsigned* flag;
  int num_sms;
  int hash_tc;                // hash model: MLP on the tensor cores (bf16 operands)
  MarchWs ws;
  KernelTimer timer;          // events around each kernel class (timing enabled)
};

cudaError_t march_prepare(cudaStream_t st);
cudaError_t march_render_chunk(const MarchArgs& a, cudaStream_t st);
cudaError_t exclusive_scan(const int32_t* in, int64_t n, int32_t* out, int32_t* tmp,
                           cudaStream_t st);
cudaError_t launch_march_mask(const float* o, const float* d, int64_t R, float near, float step,
                              int K, const uint32_t* occ, uint32_t* mask, int32_t* count,
                              uint8_t* live_u8, cudaStream_t st);
cudaError_t launch_route_points(const float* x, int64_t n, int32_t* cell, int32_t* hist,
                                int32_t* off, int32_t* order, int32_t* fill, int32_t* scan_tmp,
                                unsigned* flag, cudaStream_t st);
cudaError_t launch_hash_encode_backward(const float* x, int64_t n, const float* d_feat,
                                       float* grad, int deterministic, cudaStream_t st);
cudaError_t launch_hash_encode(const float* x, int64_t n, const uint16_t* table, float* feat,
                               int32_t* rows, cudaStream_t st);
cudaError_t launch_sh(const float* d, int64_t n, float* out, cudaStream_t st);

}  // namespace nerfb
