// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/nerf.h"

namespace nerfb {

// Device error flag bits (ORed into ctx->d_flag).
enum : unsigned {
  FLAG_BAD_INDEX = 1u,     // an index left its buffer; the access was skipped
  FLAG_TIMEOUT = 2u,       // a bounded wait gave up
};

// ---------------------------------------------------------------------------
// IEEE fp32 helpers without contraction: the CUDA path and the oracle evaluate
// every decision-carrying value (directions, sample positions, points) with the
// same rounded operations in the same order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fadd(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float fsub(float a, float b) { return __fsub_rn(a, b); }
__device__ __forceinline__ float fmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float fdiv(float a, float b) { return __fdiv_rn(a, b); }

// SplitMix64 output function (Steele, Lea and Flood, OOPSLA 2014).
__host__ __device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// 24-bit draw m for (ray, stream, index) under key = sm64_mix(seed).
__device__ __forceinline__ uint32_t draw_bits(uint64_t key, uint64_t ray, uint32_t stream,
                                              uint32_t index) {
  uint64_t ctr = (ray << 20) | ((uint64_t)stream << 16) | (uint64_t)index;
  return (uint32_t)(sm64_mix(key ^ ctr) >> 40);
}

// Stratified sample i of n on [near, far] with 24-bit jitter m (or u = 0.5).
__device__ __forceinline__ float stratified_t(float near, float step, int i, uint32_t m,
                                              bool perturb) {
  float u = perturb ? (float)m * 5.9604644775390625e-08f : 0.5f;
  float s = fadd((float)i, u);
  return fadd(near, fmul(s, step));
}

// Positional encoding value j of coordinate triple x (layout [x, sin block, cos
// block], each block coordinate-major c*L + k): sin/cos(pi * 2^k * x_c).
__device__ __forceinline__ void pe_sincos(float xc, int k, float* s, float* c) {
  sincospif(ldexpf(xc, k), s, c);
}

struct Ctx;

// Kernel classes that nerf_timing_enable times (NERF_TIMED_* of the header).
enum TimedKind : int {
  TK_NETWORK = NERF_TIMED_NETWORK,
  TK_COMPOSITE = NERF_TIMED_COMPOSITE,
  TK_RESAMPLE = NERF_TIMED_RESAMPLE,
  TK_DIR_BIAS = NERF_TIMED_DIR_BIAS,
  TK_MARCH_MASK = NERF_TIMED_MARCH_MASK,
  TK_MARCH_COMPACT = NERF_TIMED_MARCH_COMPACT,
  TK_ROUTER = NERF_TIMED_ROUTER,
  TK_MARCH_COMPOSITE = NERF_TIMED_MARCH_COMPOSITE,
};

// Records a pair of CUDA events on the launching stream around the launches of
// one kernel class; inert when timing is off (ev == nullptr) or the slots are used up.
struct KernelTimer {
  cudaEvent_t* ev = nullptr;   // [2 * cap]
  int* kind = nullptr;         // [cap]
  int* n = nullptr;
  int cap = 0;
  int begin(int k, cudaStream_t st) const {
    if (!ev || *n >= cap) return -1;
    const int s = (*n)++;
    kind[s] = k;
    cudaEventRecord(ev[2 * s], st);
    return s;
  }
  void end(int slot, cudaStream_t st) const {
    if (slot >= 0) cudaEventRecord(ev[2 * slot + 1], st);
  }
};

// Launchers (each returns cudaGetLastError()).
cudaError_t launch_raygen(int H, int W, float focal, const float* c2w, float* o, float* d,
                          cudaStream_t st);
cudaError_t launch_raygen_batch(int H, int W, float focal, int n_cams, const float* c2w,
                                float* o, float* d, cudaStream_t st);
cudaError_t launch_stratified(const float* o, const float* d, int64_t R, float near, float far,
                              int n, uint64_t key, int perturb, float* out_t, float* out_x,
                              cudaStream_t st);
cudaError_t launch_pe(const float* x, int64_t n, int L, float* out, cudaStream_t st);

// Dir-layer per-ray bias: out[r][j] = b_dir[j] + sum_k Wdir[j][W + k] gamma(d_r/|d_r|)[k].
cudaError_t launch_dir_bias(const float* d, int64_t R, const void* blob, int precision, int W,
                            int L_dir, int64_t dir_w_off, int64_t dir_b_off, float* out,
                            cudaStream_t st);

// fp32 weights packed for the CUDA-core MLP (see k_mlp_fp32.cu for the layout).
struct PackedFp32 {
  int D, W, skip, pos_ch;
  int64_t layer_w[8], layer_b[8];
  int64_t sigma_w, sigma_b, feat_w, feat_b, dir_w, rgb_w, rgb_b;
  int64_t total;
};
PackedFp32 plan_fp32(int D, int W, int skip, int pos_ch, int dir_ch);
cudaError_t launch_pack_fp32(const void* blob, int precision, const PackedFp32& p, int dir_ch,
                             float* out, cudaStream_t st);

// Sample sources for the MLP kernels.
enum SampleMode { SAMPLES_STRATIFIED = 0, SAMPLES_GIVEN_T = 1, SAMPLES_GIVEN_X = 2 };
struct SampleSpec {
  int mode;
  int S;            // samples per ray
  float near, step; // stratified
  uint64_t key;
  int perturb;
  const float* t;   // [R][S] when GIVEN_T; points [R*S][3] when GIVEN_X
};

cudaError_t launch_mlp_fp32(const PackedFp32& p, const float* packed, const float* dir_bias,
                            const float* o, const float* d, int64_t R, const SampleSpec& ss,
                            float* raw, cudaStream_t st);

// Compositing of raw [R][S][4]; t from ss (stratified or given).
struct CompositeSpec {
  int last_mode;     // 0: 1e10, 1: to far, 2: march step
  float far, march_step;
  int sigma_act, white;
};
// Training path (k_train.cu).
cudaError_t launch_composite_bw(const float* raw, const SampleSpec& ss, const float* d, int64_t R,
                                const CompositeSpec& cs, const float* target, float inv3n,
                                float* d_raw, float* loss_terms, cudaStream_t st);
// bsplit: scratch of TRAIN_BSPLIT floats (K x n_out x 2 for the widest layer,
// K = 256 + 64, 256 outputs) for the tensor-core row GEMMs' split weights;
// flag: the context's error flag.
constexpr int64_t TRAIN_BSPLIT = (int64_t)320 * 256 * 2;
// ray0: index of the first ray in the whole batch (the stratified draws are
// keyed by it); compact: the store keeps only what the forward needs,
// [gamma(x) 64 | two ping-pong hidden slots W | h_dir W/2] (row stride
// compact_ldc), instead of every layer's output for the backward.
cudaError_t mlp_forward_train_fp32(const PackedFp32& p, const float* packed, const float* dir_bias,
                                   const float* o, const float* d, int64_t R,
                                   const SampleSpec& ss, float* raw, float* save, float* bsplit,
                                   unsigned* flag, cudaStream_t st, int64_t ray0 = 0,
                                   bool compact = false);
inline int64_t compact_ldc(int W) { return 64 + 2 * (int64_t)W + W / 2; }
cudaError_t mlp_backward_fp32(const PackedFp32& p, int L_dir, const float* w, const float* save,
                              int64_t R, int S, const float* d, const float* d_raw,
                              float* grad, float* tmp, float* bsplit, unsigned* flag,
                              cudaStream_t st);
cudaError_t launch_sum(const float* v, int64_t n, float* out, cudaStream_t st);
cudaError_t launch_composite(const float* raw, const SampleSpec& ss, const float* d, int64_t R,
                             const CompositeSpec& cs, float* rgb, float* depth, float* acc,
                             float* weights, cudaStream_t st);

// Optional copies of the resampler's own intermediates (device, NULL = none):
// the coarse weights it composited [R][64], its draws in draw order [R][Nf] and
// their bins [R][Nf].
struct ResampleTrace {
  float* w = nullptr;
  float* t_f = nullptr;
  int32_t* below = nullptr;
};
// Coarse compositing fused with inverse-CDF resampling and the sorted merge:
// raw_c [R][64][4] -> t_all [R][64 + Nf].
cudaError_t launch_coarse_resample(const float* raw_c, const SampleSpec& coarse, const float* d,
                                   int64_t R, const CompositeSpec& cs, int Nf, uint64_t key,
                                   int perturb, float* t_all, cudaStream_t st,
                                   const ResampleTrace& tr = ResampleTrace{});
// Resampling from given coarse t and weights (unit entry point).
cudaError_t launch_sample_pdf(const float* t_c, const float* w, int64_t R, int Nc, int Nf,
                              uint64_t key, int perturb, float* t_f, int32_t* below,
                              float* t_all, cudaStream_t st);

}  // namespace nerfb
