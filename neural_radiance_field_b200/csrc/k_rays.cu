// Ray generation, stratified sampling, positional encoding and the per-ray part
// of the direction layer.
#include "nerf_internal.cuh"

namespace nerfb {

struct C2W { float m[12]; };

// get_rays of the NeRF page (Section 2.2): one thread per pixel, row-major.
__global__ void raygen_kernel(int H, int W, float focal, C2W c, float* __restrict__ o,
                              float* __restrict__ d) {
  int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= (int64_t)H * W) return;
  int j = (int)(p / W), i = (int)(p % W);
  float dx = fdiv(fsub((float)i, fmul((float)W, 0.5f)), focal);
  float dy = -fdiv(fsub((float)j, fmul((float)H, 0.5f)), focal);
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    float v = fadd(fadd(fmul(dx, c.m[r * 4 + 0]), fmul(dy, c.m[r * 4 + 1])),
                   fmul(-1.0f, c.m[r * 4 + 2]));
    d[p * 3 + r] = v;
    o[p * 3 + r] = c.m[r * 4 + 3];
  }
}

cudaError_t launch_raygen(int H, int W, float focal, const float* c2w, float* o, float* d,
                          cudaStream_t st) {
  C2W c;
  for (int k = 0; k < 12; ++k) c.m[k] = c2w[k];
  int64_t n = (int64_t)H * W;
  raygen_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(H, W, focal, c, o, d);
  return cudaGetLastError();
}

// Up to RAYGEN_BATCH cameras per launch, passed by value.
constexpr int RAYGEN_BATCH = 32;
struct C2WBatch {
  float m[RAYGEN_BATCH][12];
};

// Rays of several cameras, camera-major: camera c's pixel p lands at
// c * H * W + p, each value computed exactly as raygen_kernel does.
__global__ void raygen_batch_kernel(int H, int W, float focal, int n_cams, C2WBatch cams,
                                    float* __restrict__ o, float* __restrict__ d) {
  const int64_t hw = (int64_t)H * W;
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= hw * n_cams) return;
  const int cam = (int)(q / hw);
  const int64_t p = q % hw;
  const float* m = cams.m[cam];
  int j = (int)(p / W), i = (int)(p % W);
  float dx = fdiv(fsub((float)i, fmul((float)W, 0.5f)), focal);
  float dy = -fdiv(fsub((float)j, fmul((float)H, 0.5f)), focal);
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    float v = fadd(fadd(fmul(dx, m[r * 4 + 0]), fmul(dy, m[r * 4 + 1])), fmul(-1.0f, m[r * 4 + 2]));
    d[q * 3 + r] = v;
    o[q * 3 + r] = m[r * 4 + 3];
  }
}

cudaError_t launch_raygen_batch(int H, int W, float focal, int n_cams, const float* c2w,
                                float* o, float* d, cudaStream_t st) {
  const int64_t hw = (int64_t)H * W;
  for (int c0 = 0; c0 < n_cams; c0 += RAYGEN_BATCH) {
    const int nc = n_cams - c0 < RAYGEN_BATCH ? n_cams - c0 : RAYGEN_BATCH;
    C2WBatch cams;
    for (int c = 0; c < nc; ++c)
      for (int k = 0; k < 12; ++k) cams.m[c][k] = c2w[(int64_t)(c0 + c) * 12 + k];
    const int64_t n = hw * nc;
    raygen_batch_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        H, W, focal, nc, cams, o + c0 * hw * 3, d + c0 * hw * 3);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

__global__ void stratified_kernel(const float* __restrict__ o, const float* __restrict__ d,
                                  int64_t R, float near, float step, int n, uint64_t key,
                                  int perturb, float* __restrict__ out_t,
                                  float* __restrict__ out_x) {
  int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= R * n) return;
  int64_t r = q / n;
  int i = (int)(q % n);
  uint32_t m = perturb ? draw_bits(key, (uint64_t)r, 0, (uint32_t)i) : 0u;
  float t = stratified_t(near, step, i, m, perturb != 0);
  out_t[q] = t;
  if (out_x) {
#pragma unroll
    for (int c = 0; c < 3; ++c) out_x[q * 3 + c] = fadd(o[r * 3 + c], fmul(t, d[r * 3 + c]));
  }
}

cudaError_t launch_stratified(const float* o, const float* d, int64_t R, float near, float far,
                              int n, uint64_t key, int perturb, float* out_t, float* out_x,
                              cudaStream_t st) {
  float step = (float)(far - near);  // fp32 subtraction of fp32 operands
  step = step / (float)n;
  int64_t tot = R * n;
  stratified_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(o, d, R, near, step, n, key,
                                                                    perturb, out_t, out_x);
  return cudaGetLastError();
}

__global__ void pe_kernel(const float* __restrict__ x, int64_t n, int L, float* __restrict__ out) {
  int dim = 3 + 6 * L;
  int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= n * dim) return;
  int64_t p = q / dim;
  int j = (int)(q % dim);
  float v;
  if (j < 3) {
    v = x[p * 3 + j];
  } else {
    int jj = (j - 3) % (3 * L);
    int c = jj / L, k = jj % L;
    float s, co;
    pe_sincos(x[p * 3 + c], k, &s, &co);
    v = (j - 3 < 3 * L) ? s : co;
  }
  out[q] = v;
}

cudaError_t launch_pe(const float* x, int64_t n, int L, float* out, cudaStream_t st) {
  int64_t tot = n * (3 + 6 * L);
  pe_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(x, n, L, out);
  return cudaGetLastError();
}

__device__ __forceinline__ float load_param(const void* blob, int precision, int64_t i) {
  if (precision == NERF_BF16) return __bfloat162float(((const __nv_bfloat16*)blob)[i]);
  return ((const float*)blob)[i];
}

// Thread j (< W/2) keeps row j of the direction layer's gamma(d) columns in
// registers; the block walks over groups of RB rays, encodes their unit
// directions into shared memory and writes RB outputs per thread.
constexpr int DIR_RB = 8;
constexpr int DIR_MAXCH = 27;

__global__ void dir_bias_kernel(const float* __restrict__ d, int64_t R, const void* blob,
                                int precision, int W, int L_dir, int64_t w_off, int64_t b_off,
                                float* __restrict__ out) {
  const int Wh = W / 2;
  const int dir_ch = 3 + 6 * L_dir;
  const int j = threadIdx.x;
  __shared__ float enc[DIR_RB][32];
  const int K = W + dir_ch;
  float w[DIR_MAXCH];
#pragma unroll
  for (int k = 0; k < DIR_MAXCH; ++k)
    w[k] = k < dir_ch ? load_param(blob, precision, w_off + (int64_t)j * K + W + k) : 0.0f;
  const float b = load_param(blob, precision, b_off + j);
  for (int64_t r0 = (int64_t)blockIdx.x * DIR_RB; r0 < R; r0 += (int64_t)gridDim.x * DIR_RB) {
    __syncthreads();
    for (int q = j; q < DIR_RB * dir_ch; q += Wh) {
      const int rr = q / dir_ch, k = q % dir_ch;
      const int64_t r = r0 + rr;
      float v = 0.0f;
      if (r < R) {
        float dx = d[r * 3 + 0], dy = d[r * 3 + 1], dz = d[r * 3 + 2];
        float inv = 1.0f / sqrtf(dx * dx + dy * dy + dz * dz);
        float u[3] = {dx * inv, dy * inv, dz * inv};
        if (k < 3) {
          v = u[k];
        } else {
          int kk = (k - 3) % (3 * L_dir);
          float s, c;
          pe_sincos(u[kk / L_dir], kk % L_dir, &s, &c);
          v = (k - 3 < 3 * L_dir) ? s : c;
        }
      }
      enc[rr][k] = v;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < DIR_RB; ++rr) {
      const int64_t r = r0 + rr;
      if (r >= R) break;
      float acc = b;
#pragma unroll
      for (int k = 0; k < DIR_MAXCH; ++k) acc = fmaf(w[k], enc[rr][k], acc);
      out[r * Wh + j] = acc;
    }
  }
}

cudaError_t launch_dir_bias(const float* d, int64_t R, const void* blob, int precision, int W,
                            int L_dir, int64_t w_off, int64_t b_off, float* out,
                            cudaStream_t st) {
  const int Wh = W / 2;
  if (3 + 6 * L_dir > DIR_MAXCH || Wh < 32 || Wh > 1024) return cudaErrorInvalidValue;
  int64_t groups = (R + DIR_RB - 1) / DIR_RB;
  unsigned blocks = (unsigned)(groups < 148 * 16 ? groups : 148 * 16);
  dir_bias_kernel<<<blocks, Wh, 0, st>>>(d, R, blob, precision, W, L_dir, w_off, b_off, out);
  return cudaGetLastError();
}

}  // namespace nerfb
