// Internal interface of the marching scene functions (k_march.cu).
#pragma once

#include "nerf_internal.cuh"

namespace nerfb {

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
  cudaEvent_t ev_start = nullptr;   // recorded around the scene-function kernel
  cudaEvent_t ev_stop = nullptr;    // when timing is enabled
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
