// Marching scene functions: occupancy-grid empty-space skipping, the 3D
// multiresolution hash grid with its small MLP (Instant-NGP notebook, "A shared
// toolkit" and Experiment 1, in 3D; the MLP in fp32 on the CUDA cores or in bf16
// on the tensor cores), the hash encoding's backward, the KiloNeRF grid of tiny
// MLPs with a cell router (KiloNeRF page, abstract), and compositing with early
// termination.
#include <cmath>

#include "tc_ptx.cuh"
#include "nerf_march.cuh"

namespace nerfb {

// ------------------------------------------------------------------ occupancy
// (voxel_axis, occupied_at and march_point: nerf_march.cuh)

// Warp per ray: live bitmask (K <= 512 -> 16 words) and live count.
__global__ void march_mask_kernel(const float* __restrict__ o, const float* __restrict__ d,
                                  int64_t R, float near, float step, int K,
                                  const uint32_t* __restrict__ occ, uint32_t* __restrict__ mask,
                                  int32_t* __restrict__ count, uint8_t* __restrict__ live_u8) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= R) return;
  int klo, khi;                      // only these candidates can be inside the grid
  march_window(o, d, r, near, step, K, &klo, &khi);
  int n = 0;
  for (int w = 0; w < (K + 31) / 32; ++w) {
    const int k = w * 32 + lane;
    bool live = false;
    if (k < K) {
      if (k >= klo && k <= khi) {
        float x[3], t;
        march_point(o, d, r, near, step, k, x, &t);
        live = occupied_at(occ, x[0], x[1], x[2], nullptr);
      }
      if (live_u8) live_u8[r * K + k] = live;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, live);
    if (lane == 0 && mask) mask[r * 16 + w] = m;
    n += __popc(m);
  }
  if (lane == 0) count[r] = n;
}

// Live entries (ray << 9 | k) in ray-major order from the masks and offsets;
// entries past `cap` are dropped and flagged.
__global__ void march_emit_kernel(const uint32_t* __restrict__ mask, const int32_t* __restrict__ off,
                                  int64_t R, int K, uint32_t* __restrict__ live, int64_t cap,
                                  unsigned* flag) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= R) return;
  int64_t base = off[r];
  for (int w = 0; w < (K + 31) / 32; ++w) {
    const uint32_t m = mask[r * 16 + w];
    if ((m >> lane) & 1u) {
      const int64_t pos = base + __popc(m & ((1u << lane) - 1u));
      if (pos < cap) live[pos] = ((uint32_t)r << 9) | (uint32_t)(w * 32 + lane);
      else atomicOr(flag, FLAG_BAD_INDEX);
    }
    base += __popc(m);
  }
}

// ------------------------------------------------------------------ scan

// Exclusive scan of int32 counts (n <= 2048 * 1024) into off[0..n].
__global__ void scan_block_kernel(const int32_t* __restrict__ in, int64_t n,
                                  int32_t* __restrict__ out, int32_t* __restrict__ block_sums) {
  __shared__ int32_t s[1024];
  const int64_t i = (int64_t)blockIdx.x * 1024 + threadIdx.x;
  int v = i < n ? in[i] : 0;
  s[threadIdx.x] = v;
  __syncthreads();
  for (int offs = 1; offs < 1024; offs <<= 1) {
    int a = threadIdx.x >= offs ? s[threadIdx.x - offs] : 0;
    __syncthreads();
    s[threadIdx.x] += a;
    __syncthreads();
  }
  if (i < n) out[i] = s[threadIdx.x] - v;
  if (threadIdx.x == 1023) block_sums[blockIdx.x] = s[1023];
}

__global__ void scan_sums_kernel(int32_t* __restrict__ sums, int nb, int32_t* __restrict__ total) {
  __shared__ int32_t s[2048];
  for (int i = threadIdx.x; i < 2048; i += blockDim.x) s[i] = i < nb ? sums[i] : 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < nb; ++i) { int v = s[i]; s[i] = run; run += v; }
    *total = run;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nb; i += blockDim.x) sums[i] = s[i];
}

__global__ void scan_add_kernel(int32_t* __restrict__ out, int64_t n,
                                const int32_t* __restrict__ block_sums) {
  const int64_t i = (int64_t)blockIdx.x * 1024 + threadIdx.x;
  if (i < n) out[i] += block_sums[blockIdx.x];
}

cudaError_t exclusive_scan(const int32_t* in, int64_t n, int32_t* out, int32_t* tmp,
                           cudaStream_t st) {
  const int64_t nb = (n + 1023) / 1024;
  if (nb > 2048) return cudaErrorInvalidValue;
  scan_block_kernel<<<(unsigned)nb, 1024, 0, st>>>(in, n, out, tmp);
  scan_sums_kernel<<<1, 256, 0, st>>>(tmp, (int)nb, out + n);
  scan_add_kernel<<<(unsigned)nb, 1024, 0, st>>>(out, n, tmp);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ hash grid

__constant__ int c_hres[16];
__constant__ int c_hoff[16];
__constant__ int c_hdirect[16];

HashGridInfo hash_grid_info() {
  HashGridInfo h{};
  const double b = std::exp((std::log(2048.0) - std::log(16.0)) / 15.0);
  int64_t off = 0;
  for (int l = 0; l < 16; ++l) {
    const double v = 16.0 * std::pow(b, l);
    // round half to even, as the resolution schedule specifies
    double fl = std::floor(v);
    int N = (int)fl;
    const double frac = v - fl;
    if (frac > 0.5 || (frac == 0.5 && (N & 1))) N += 1;
    const int64_t cells = (int64_t)(N + 1) * (N + 1) * (N + 1);
    h.res[l] = N;
    h.direct[l] = cells <= (int64_t(1) << 19);
    h.offset[l] = (int)off;
    off += h.direct[l] ? cells : (int64_t(1) << 19);
  }
  h.entries = off;
  return h;
}

cudaError_t upload_hash_grid(const HashGridInfo& h) {
  cudaError_t e = cudaMemcpyToSymbol(c_hres, h.res, sizeof h.res);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(c_hoff, h.offset, sizeof h.offset);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(c_hdirect, h.direct, sizeof h.direct);
  return e;
}

// Encoding of one point; optionally records the corner rows.
// Level l of the encoding of a point with unit-cube coordinates u: the
// trilinear blend of the 8 corner rows, feature pair (a0, a1).
__device__ __forceinline__ void hash_encode_level(const __half2* __restrict__ table, float u0,
                                                  float u1, float u2, int l, int32_t* rows_out,
                                                  float& a0, float& a1) {
  const int N = c_hres[l];
  const float fN = (float)N;
  const float c0 = fmul(u0, fN), c1 = fmul(u1, fN), c2 = fmul(u2, fN);
  const float f0 = floorf(c0), f1 = floorf(c1), f2 = floorf(c2);
  const float w0 = fsub(c0, f0), w1 = fsub(c1, f1), w2 = fsub(c2, f2);
  const int i0 = (int)f0, i1 = (int)f1, i2 = (int)f2;
  a0 = 0.f;
  a1 = 0.f;
#pragma unroll
  for (int corner = 0; corner < 8; ++corner) {
    const int dx = corner >> 2, dy = (corner >> 1) & 1, dz = corner & 1;
    const int ix = min(max(i0 + dx, 0), N), iy = min(max(i1 + dy, 0), N),
              iz = min(max(i2 + dz, 0), N);
    uint32_t idx;
    if (c_hdirect[l]) {
      idx = (uint32_t)((ix * (N + 1) + iy) * (N + 1) + iz);
    } else {
      idx = ((uint32_t)ix ^ ((uint32_t)iy * 2654435761u) ^ ((uint32_t)iz * 805459861u)) &
            ((1u << 19) - 1u);
    }
    const int row = c_hoff[l] + (int)idx;
    if (rows_out) rows_out[l * 8 + corner] = row;
    const float2 f = __half22float2(__ldg(table + row));
    const float wx = dx ? w0 : 1.0f - w0;
    const float wy = dy ? w1 : 1.0f - w1;
    const float wz = dz ? w2 : 1.0f - w2;
    const float wt = wx * wy * wz;
    a0 = fmaf(wt, f.x, a0);
    a1 = fmaf(wt, f.y, a1);
  }
}

__device__ __forceinline__ void hash_unit_coords(float x0, float x1, float x2, float& u0,
                                                 float& u1, float& u2) {
  u0 = fdiv(fadd(x0, 1.5f), 3.0f);
  u1 = fdiv(fadd(x1, 1.5f), 3.0f);
  u2 = fdiv(fadd(x2, 1.5f), 3.0f);
}

__device__ __forceinline__ void hash_encode_point(const __half2* __restrict__ table, float x0,
                                                  float x1, float x2, float* feat,
                                                  int32_t* rows_out) {
  float u0, u1, u2;
  hash_unit_coords(x0, x1, x2, u0, u1, u2);
#pragma unroll 4
  for (int l = 0; l < 16; ++l) hash_encode_level(table, u0, u1, u2, l, rows_out, feat[2 * l], feat[2 * l + 1]);
}

// Backward of the encoding (its adjoint): every point adds, at each level,
// weight * d_feat[level] to each of its 8 corner rows, the same rows and
// trilinear weights as hash_encode_level computes. Two ways to sum:
//   fp32 atomics (fast; the summation order, hence the last bits, varies), or
//   fixed point: each term rounded to a multiple of 2^-E and added as int64 with
//   2's-complement atomics, which are associative, so the result does not
//   depend on the order. E = 62 - ceil(log2(n max|d_feat|)): a row's sum of
//   |weight * g| is at most n max|g| (a point's 8 weights per level sum to 1),
//   so no sum can overflow.
template <bool FIXED>
__device__ __forceinline__ void hash_level_scatter(float u0, float u1, float u2, int l, float g0,
                                                   float g1, float* grad,
                                                   unsigned long long* acc, double scale) {
  const int N = c_hres[l];
  const float fN = (float)N;
  const float c0 = fmul(u0, fN), c1 = fmul(u1, fN), c2 = fmul(u2, fN);
  const float f0 = floorf(c0), f1 = floorf(c1), f2 = floorf(c2);
  const float w0 = fsub(c0, f0), w1 = fsub(c1, f1), w2 = fsub(c2, f2);
  const int i0 = (int)f0, i1 = (int)f1, i2 = (int)f2;
#pragma unroll
  for (int corner = 0; corner < 8; ++corner) {
    const int dx = corner >> 2, dy = (corner >> 1) & 1, dz = corner & 1;
    const int ix = min(max(i0 + dx, 0), N), iy = min(max(i1 + dy, 0), N),
              iz = min(max(i2 + dz, 0), N);
    uint32_t idx;
    if (c_hdirect[l]) {
      idx = (uint32_t)((ix * (N + 1) + iy) * (N + 1) + iz);
    } else {
      idx = ((uint32_t)ix ^ ((uint32_t)iy * 2654435761u) ^ ((uint32_t)iz * 805459861u)) &
            ((1u << 19) - 1u);
    }
    const int64_t row = (int64_t)c_hoff[l] + (int64_t)idx;
    const float wx = dx ? w0 : 1.0f - w0;
    const float wy = dy ? w1 : 1.0f - w1;
    const float wz = dz ? w2 : 1.0f - w2;
    const float wt = wx * wy * wz;
    if (FIXED) {
      atomicAdd(acc + 2 * row, (unsigned long long)__double2ll_rn((double)wt * (double)g0 * scale));
      atomicAdd(acc + 2 * row + 1,
                (unsigned long long)__double2ll_rn((double)wt * (double)g1 * scale));
    } else {
      atomicAdd(grad + 2 * row, wt * g0);
      atomicAdd(grad + 2 * row + 1, wt * g1);
    }
  }
}

__device__ __forceinline__ double hash_fixed_scale(float max_abs, int64_t n) {
  return ldexp(1.0, 62 - (int)ceil(log2((double)n * (double)max_abs)));
}

template <bool FIXED>
__global__ void hash_bw_kernel(const float* __restrict__ x, int64_t n,
                               const float* __restrict__ d_feat, float* __restrict__ grad,
                               unsigned long long* __restrict__ acc,
                               const unsigned* __restrict__ max_bits) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  double scale = 0.0;
  if (FIXED) {
    const float mx = __uint_as_float(*max_bits);
    if (!(mx > 0.0f)) return;
    scale = hash_fixed_scale(mx, n);
  }
  float u0, u1, u2;
  hash_unit_coords(x[i * 3], x[i * 3 + 1], x[i * 3 + 2], u0, u1, u2);
#pragma unroll 2
  for (int l = 0; l < 16; ++l)
    hash_level_scatter<FIXED>(u0, u1, u2, l, d_feat[i * 32 + 2 * l], d_feat[i * 32 + 2 * l + 1],
                              grad, acc, scale);
}

// max |v| over m values, as the bits of a non-negative float (which order like
// unsigned integers), into *out (zeroed by the caller).
__global__ void absmax_kernel(const float* __restrict__ v, int64_t m, unsigned* __restrict__ out) {
  float mx = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < m;
       i += (int64_t)gridDim.x * blockDim.x)
    mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(mx));
}

__global__ void fixed_to_grad_kernel(const unsigned long long* __restrict__ acc, int64_t m,
                                     const unsigned* __restrict__ max_bits, int64_t n,
                                     float* __restrict__ grad) {
  const float mx = __uint_as_float(*max_bits);
  if (!(mx > 0.0f)) return;
  const double inv = 1.0 / hash_fixed_scale(mx, n);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < m;
       i += (int64_t)gridDim.x * blockDim.x)
    grad[i] += (float)((double)(long long)acc[i] * inv);
}

__global__ void hash_encode_kernel(const float* __restrict__ x, int64_t n,
                                   const __half2* __restrict__ table, float* __restrict__ feat,
                                   int32_t* __restrict__ rows) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float f[32];
  hash_encode_point(table, x[i * 3], x[i * 3 + 1], x[i * 3 + 2], f, rows ? rows + i * 128 : nullptr);
#pragma unroll
  for (int j = 0; j < 32; ++j) feat[i * 32 + j] = f[j];
}

// Real SH bands 0..3 of a unit vector, no Condon-Shortley phase; K holds
// sqrt(2) K_l^m (m > 0) or K_l^0 folded with the Legendre leading factors.
__device__ __forceinline__ void sh16(float x, float y, float z, const ShConst& K, float* o) {
  o[0] = K.k[0];
  o[1] = K.k[1] * y;
  o[2] = K.k[2] * z;
  o[3] = K.k[1] * x;
  o[4] = K.k[4] * x * y;
  o[5] = K.k[5] * y * z;
  o[6] = K.k[6] * (3.0f * z * z - 1.0f);
  o[7] = K.k[5] * x * z;
  o[8] = K.k[8] * (x * x - y * y);
  o[9] = K.k[9] * (3.0f * x * x * y - y * y * y);
  o[10] = K.k[10] * x * y * z;
  o[11] = K.k[11] * y * (5.0f * z * z - 1.0f);
  o[12] = K.k[12] * z * (5.0f * z * z - 3.0f);
  o[13] = K.k[11] * x * (5.0f * z * z - 1.0f);
  o[14] = K.k[14] * z * (x * x - y * y);
  o[15] = K.k[9] * (x * x * x - 3.0f * x * y * y);
}

ShConst sh_constants() {
  auto fact = [](int n) { double f = 1; for (int i = 2; i <= n; ++i) f *= i; return f; };
  auto norm = [&](int l, int m) {
    return std::sqrt((2 * l + 1) / (4.0 * M_PI) * fact(l - m) / fact(l + m));
  };
  const double r2 = std::sqrt(2.0);
  ShConst K{};
  // P_l^m (no Condon-Shortley phase) times cos/sin(m phi), written in x, y, z:
  // P_1^1 -> (x, y); P_2^1 = 3z sqrt(1-z^2); P_2^2 = 3(1-z^2); P_2^0 = (3z^2-1)/2;
  // P_3^0 = z(5z^2-3)/2; P_3^1 = 3/2 (5z^2-1) sqrt(1-z^2); P_3^2 = 15 z (1-z^2);
  // P_3^3 = 15 (1-z^2)^(3/2); sin(2 phi) terms carry the factor 2 of 2xy.
  K.k[0] = (float)norm(0, 0);
  K.k[1] = (float)(r2 * norm(1, 1));
  K.k[2] = (float)norm(1, 0);
  K.k[4] = (float)(r2 * norm(2, 2) * 3.0 * 2.0);
  K.k[5] = (float)(r2 * norm(2, 1) * 3.0);
  K.k[6] = (float)(norm(2, 0) * 0.5);
  K.k[8] = (float)(r2 * norm(2, 2) * 3.0);
  K.k[9] = (float)(r2 * norm(3, 3) * 15.0);
  K.k[10] = (float)(r2 * norm(3, 2) * 15.0 * 2.0);
  K.k[11] = (float)(r2 * norm(3, 1) * 1.5);
  K.k[12] = (float)(norm(3, 0) * 0.5);
  K.k[14] = (float)(r2 * norm(3, 2) * 15.0);
  return K;
}

__global__ void sh_kernel(const float* __restrict__ d, int64_t n, ShConst K,
                          float* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float dx = d[i * 3], dy = d[i * 3 + 1], dz = d[i * 3 + 2];
  const float inv = 1.0f / sqrtf(dx * dx + dy * dy + dz * dz);
  float o[16];
  sh16(dx * inv, dy * inv, dz * inv, K, o);
#pragma unroll
  for (int j = 0; j < 16; ++j) out[i * 16 + j] = o[j];
}


// The hash scene function as small fp32 GEMMs over tiles of 128 live points
// (a CTA per SM, persistent): the points' activations sit k-major in shared
// memory, the layer weights transposed (Wt[k][n]) beside them, and each of
// 256 threads accumulates an 8-point x 4-output block, so every k step costs
// three 16-byte shared loads for 32 FMAs. The CTA holds two such groups of 256
// threads, each with its own tile and activations and its own named barrier,
// sharing the weights: one group's table gathers overlap the other's GEMMs. Layers: encoding (32) -> 64 -> 64
// (ReLU) -> sigma = ReLU(w . h + b); [h | SH16(d)] (80) -> 64 -> 64 (ReLU) ->
// rgb = sigmoid(W h + b). All arithmetic is fp32 on the CUDA cores.
constexpr int HASH_NW = 15876;                       // fp32 weights of the ABI blob
#ifndef NERF_HT_P
#define NERF_HT_P 128
#endif
constexpr int HT_P = NERF_HT_P;                      // points per tile (128 or 64)
constexpr int HT_PPT = HT_P / 16;                    // points per thread in the GEMMs
constexpr int HT_TPP = 256 / HT_P;                   // threads per point in the encoding
constexpr int HT_AP = HT_P + 4;                      // padded row of an activation buffer
constexpr int HT_GROUPS = 2;                         // independent tile groups per CTA
constexpr int HT_THREADS = 256 * HT_GROUPS;
constexpr int HT_CTAS_PER_SM = 1;
// shared-memory layout (floats)
constexpr int HT_D0 = 0, HT_D1 = HT_D0 + 32 * 64, HT_C0 = HT_D1 + 64 * 64, HT_C1 = HT_C0 + 80 * 64;
constexpr int HT_VEC = HT_C1 + 64 * 64;              // d0b d1b c0b c1b sw (5 x 64), sb, pad, rw (192), rb
constexpr int HT_GRP = HT_VEC + 5 * 64 + 4 + 192 + 4;  // first group's buffers
// per group: act_a [80][HT_AP], act_b [64][HT_AP], sig [HT_P], rgb [3][HT_P]
constexpr int HT_ACT_A = 0;
constexpr int HT_ACT_B = HT_ACT_A + 80 * HT_AP;
constexpr int HT_SIG = HT_ACT_B + 64 * HT_AP;
constexpr int HT_RGB = HT_SIG + HT_P;
constexpr int HT_GRP_FLOATS = HT_RGB + 3 * HT_P;
constexpr int HT_FLOATS = HT_GRP + HT_GROUPS * HT_GRP_FLOATS;
constexpr size_t HT_SMEM = HT_FLOATS * sizeof(float);
static_assert(HT_GRP % 4 == 0 && HT_ACT_B % 4 == 0 && HT_GRP_FLOATS % 4 == 0 && HT_AP % 4 == 0,
              "float4 alignment");

// Barrier of one 256-thread group (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

// The staged weights and biases keep output n in column perm64(n), so that
// thread tx's four columns 4 tx .. 4 tx + 3 hold outputs tx, tx + 16, tx + 32,
// tx + 48: its epilogue then stores four feature rows 16 apart, which fall in
// distinct shared-memory banks across the warp.
__device__ __forceinline__ int perm64(int n) { return 4 * (n & 15) + (n >> 4); }

// out[n][p] = act(b[n] + sum_k W[n][k] in[k][p]) for the tile, N = 64; the
// operands of step k + 1 are loaded while step k computes.
template <int K>
__device__ __forceinline__ void tile_dense64(const float* __restrict__ Wt, const float* __restrict__ b,
                                             const float* in, float* out, int lt) {
  const int tx = lt & 15, ty = lt >> 4;
  const int n0 = 4 * tx, p0 = HT_PPT * ty;
  static_assert(HT_PPT == 8, "two float4 of points per thread");
  float acc[HT_PPT][4];
  const float4 bb = *reinterpret_cast<const float4*>(b + n0);
#pragma unroll
  for (int i = 0; i < HT_PPT; ++i) { acc[i][0] = bb.x; acc[i][1] = bb.y; acc[i][2] = bb.z; acc[i][3] = bb.w; }
  float4 a0 = *reinterpret_cast<const float4*>(in + p0);
  float4 a1 = *reinterpret_cast<const float4*>(in + p0 + 4);
  float4 w = *reinterpret_cast<const float4*>(Wt + n0);
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    const float a[HT_PPT] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float4 wc = w;
    if (k + 1 < K) {
      a0 = *reinterpret_cast<const float4*>(in + (k + 1) * HT_AP + p0);
      a1 = *reinterpret_cast<const float4*>(in + (k + 1) * HT_AP + p0 + 4);
      w = *reinterpret_cast<const float4*>(Wt + (k + 1) * 64 + n0);
    }
#pragma unroll
    for (int i = 0; i < HT_PPT; ++i) {
      acc[i][0] = fmaf(wc.x, a[i], acc[i][0]);
      acc[i][1] = fmaf(wc.y, a[i], acc[i][1]);
      acc[i][2] = fmaf(wc.z, a[i], acc[i][2]);
      acc[i][3] = fmaf(wc.w, a[i], acc[i][3]);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float* o = out + (tx + 16 * j) * HT_AP + p0;
#pragma unroll
    for (int v = 0; v < HT_PPT / 4; ++v)
      *reinterpret_cast<float4*>(o + 4 * v) =
          make_float4(fmaxf(acc[4 * v][j], 0.f), fmaxf(acc[4 * v + 1][j], 0.f),
                      fmaxf(acc[4 * v + 2][j], 0.f), fmaxf(acc[4 * v + 3][j], 0.f));
  }
}

__global__ void __launch_bounds__(HT_THREADS, HT_CTAS_PER_SM)
hash_eval_kernel(const float* __restrict__ o, const float* __restrict__ d, int64_t r0,
                 float near, float step, const uint32_t* __restrict__ live,
                 const int32_t* __restrict__ total, const __half2* __restrict__ table,
                 const float* __restrict__ mlp, ShConst K, float* __restrict__ out) {
  extern __shared__ __align__(16) float hs[];
  float* d0t = hs + HT_D0;
  float* d1t = hs + HT_D1;
  float* c0t = hs + HT_C0;
  float* c1t = hs + HT_C1;
  float* d0b = hs + HT_VEC;
  float* d1b = d0b + 64;
  float* c0b = d1b + 64;
  float* c1b = c0b + 64;
  float* sw = c1b + 64;
  float* sb = sw + 64;                 // [1] + pad
  float* rw = sb + 4;                  // [3][64]
  float* rb = rw + 192;                // [3]
  const int grp = threadIdx.x >> 8, lt = threadIdx.x & 255;
  float* gb = hs + HT_GRP + grp * HT_GRP_FLOATS;
  float* act_a = gb + HT_ACT_A;        // [80][HT_AP]: encoding, then h2 | SH, then the last h
  float* act_b = gb + HT_ACT_B;        // [64][HT_AP]
  float* sig = gb + HT_SIG;
  float* rgbv = gb + HT_RGB;           // [3][HT_P]
  // weights of the ABI blob (row-major W[n][k]) -> transposed Wt[k][n]
  for (int q = threadIdx.x; q < HASH_NW; q += HT_THREADS) {
    const float v = mlp[q];
    if (q < 2048) { d0t[(q % 32) * 64 + perm64(q / 32)] = v; }
    else if (q < 2112) { d0b[perm64(q - 2048)] = v; }
    else if (q < 6208) { const int z = q - 2112; d1t[(z % 64) * 64 + perm64(z / 64)] = v; }
    else if (q < 6272) { d1b[perm64(q - 6208)] = v; }
    else if (q < 6336) { sw[q - 6272] = v; }
    else if (q < 6337) { sb[0] = v; }
    else if (q < 11457) { const int z = q - 6337; c0t[(z % 80) * 64 + perm64(z / 80)] = v; }
    else if (q < 11521) { c0b[perm64(q - 11457)] = v; }
    else if (q < 15617) { const int z = q - 11521; c1t[(z % 64) * 64 + perm64(z / 64)] = v; }
    else if (q < 15681) { c1b[perm64(q - 15617)] = v; }
    else if (q < 15873) { rw[q - 15681] = v; }
    else { rb[q - 15873] = v; }
  }
  __syncthreads();       // the weights are staged
  const int64_t P = *total;
  const int p = lt & (HT_P - 1);
  const int part = lt / HT_P;                   // 0 .. HT_TPP - 1
  for (int64_t i0 = ((int64_t)blockIdx.x * HT_GROUPS + grp) * HT_P; i0 < P;
       i0 += (int64_t)gridDim.x * HT_GROUPS * HT_P) {
    const int n = (int)min((int64_t)HT_P, P - i0);
    group_sync(grp);     // the group's previous tile's last reads are over
    // encoding: HT_TPP threads per point, each 16 / HT_TPP of the levels; the
    // last also writes SH16 of the unit direction into rows 64..79
    {
      float x[3] = {0.f, 0.f, 0.f}, t;
      int64_t r = 0;
      if (p < n) {
        const uint32_t e = live[i0 + p];
        r = r0 + (e >> 9);
        march_point(o, d, r, near, step, (int)(e & 511u), x, &t);
      }
      float u0, u1, u2;
      hash_unit_coords(x[0], x[1], x[2], u0, u1, u2);
      constexpr int LPT = 16 / HT_TPP;
#pragma unroll 2
      for (int l = LPT * part; l < LPT * part + LPT; ++l) {
        float a0 = 0.f, a1 = 0.f;
        if (p < n) hash_encode_level(table, u0, u1, u2, l, nullptr, a0, a1);
        act_a[(2 * l) * HT_AP + p] = a0;
        act_a[(2 * l + 1) * HT_AP + p] = a1;
      }
      if (part == HT_TPP - 1) {
        float sh[16];
        const float dx = d[r * 3], dy = d[r * 3 + 1], dz = d[r * 3 + 2];
        const float inv = 1.0f / sqrtf(dx * dx + dy * dy + dz * dz);
        sh16(dx * inv, dy * inv, dz * inv, K, sh);
#pragma unroll
        for (int j = 0; j < 16; ++j) act_a[(64 + j) * HT_AP + p] = p < n ? sh[j] : 0.f;
      }
    }
    group_sync(grp);
    tile_dense64<32>(d0t, d0b, act_a, act_b, lt);          // 32 -> 64
    group_sync(grp);
    tile_dense64<64>(d1t, d1b, act_b, act_a, lt);          // 64 -> 64: h2 in rows 0..63
    group_sync(grp);
    if (part == 0) {                                   // sigma = ReLU(sw . h2 + sb)
      float s = sb[0];
#pragma unroll 8
      for (int j = 0; j < 64; ++j) s = fmaf(sw[j], act_a[j * HT_AP + p], s);
      sig[p] = fmaxf(s, 0.0f);
    }
    tile_dense64<80>(c0t, c0b, act_a, act_b, lt);          // [h2 | SH16] -> 64
    group_sync(grp);
    tile_dense64<64>(c1t, c1b, act_b, act_a, lt);          // 64 -> 64
    group_sync(grp);
    for (int q = lt; q < 3 * HT_P; q += 256) {   // rgb head
      const int c = q / HT_P, pp = q % HT_P;
      float v = rb[c];
#pragma unroll 8
      for (int j = 0; j < 64; ++j) v = fmaf(rw[c * 64 + j], act_a[j * HT_AP + pp], v);
      rgbv[c * HT_P + pp] = 1.0f / (1.0f + expf(-v));
    }
    group_sync(grp);
    if (part == 0 && p < n)
      reinterpret_cast<float4*>(out)[i0 + p] =
          make_float4(rgbv[p], rgbv[HT_P + p], rgbv[2 * HT_P + p], sig[p]);
  }
}

// The hash scene function with its MLP on the tensor cores (bf16 operands,
// fp32 accumulation in tensor memory): the reading of the Instant-NGP pages'
// tiny MLP as an optional bf16 path. The encoding and the heads stay fp32; the
// 32 encoded features, SH16(d) and the hidden activations are rounded to bf16
// as the MMAs' A operand, and the weights to bf16 when staged.
//
// One CTA per SM: warp 0 issues the MMAs (one elected thread), and six groups
// of four warps each own a tile of 128 live points (thread = point = TMEM lane);
// six groups keep more table gathers in flight than four (4 % faster, measured).
// A group encodes its tile into a bf16 operand buffer in shared memory ([enc (32)
// | h (64, overwriting enc) | SH16 at K 64..79]), then drains its 64 TMEM
// columns after each layer (+ bias, ReLU, bf16 back into the buffer). Layers:
// 32 -> 64 -> 64 (sigma head), [h | SH16] (80) -> 64 -> 64 (rgb head). The MMA
// thread interleaves the tiles layer by layer (M = 128, N = 64, K = 16
// steps), so that one tile's epilogue overlaps the others' MMAs and encodings.
constexpr int HC_GROUPS = 6;                               // tiles in flight per SM
constexpr int HC_TMEM_COLS = 512;                           // 64 per tile, allocated as a power of 2
constexpr int HC_P = 128;                                   // points per tile
constexpr int HC_THREADS = 32 + HC_GROUPS * HC_P;
constexpr int HC_W1 = 0;                                    // bf16 weights, bytes
constexpr int HC_W2 = HC_W1 + 64 * 32 * 2;
constexpr int HC_W3 = HC_W2 + 64 * 64 * 2;
constexpr int HC_W4 = HC_W3 + 64 * 80 * 2;
constexpr int HC_VEC = HC_W4 + 64 * 64 * 2;                 // fp32: b1..b4, ws, bs, rw, rb
constexpr int HC_NV = 4 * 64 + 64 + 4 + 3 * 64 + 4;
constexpr int HC_A = (HC_VEC + HC_NV * 4 + 1023) / 1024 * 1024;   // per group 128 x 80 bf16
constexpr int HC_A_BYTES = HC_P * 80 * 2;
constexpr int HC_BARS = HC_A + HC_GROUPS * HC_A_BYTES;
constexpr size_t HC_SMEM = HC_BARS + (2 * HC_GROUPS + 1) * 8 + 16;
static_assert(HC_A % 128 == 0 && HC_VEC % 16 == 0, "operand alignment");

// Byte offset of K-group kg (8 bf16) of row r in a 128-row operand buffer, and of
// output n, K-group kg in a 64-row weight matrix.
__device__ __forceinline__ uint32_t hc_a_off(int r, int kg) {
  return (uint32_t)(kg * (HC_P * 16) + (r >> 3) * 128 + (r & 7) * 16);
}
__device__ __forceinline__ uint32_t hc_w_off(int n, int k) {
  return (uint32_t)((k >> 3) * (64 * 16) + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

// The MMAs of one layer for one tile: KS steps of K = 16 into 64 TMEM columns.
template <int KS>
__device__ __forceinline__ void hc_layer_mma(uint32_t d, uint64_t a, uint64_t b) {
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) |
                             ((uint32_t)(HC_P >> 4) << 24);     // M = 128, N = 64
#pragma unroll
  for (int s = 0; s < KS; ++s)
    tcx::mma_bf16(d, a + (uint64_t)((s * 2 * HC_P * 16) >> 4), b + (uint64_t)((s * 2 * 64 * 16) >> 4),
                  idesc, s != 0);
}

__global__ void __launch_bounds__(HC_THREADS, 1)
hash_tc_kernel(const float* __restrict__ o, const float* __restrict__ d, int64_t r0, float near,
               float step, const uint32_t* __restrict__ live, const int32_t* __restrict__ total,
               const __half2* __restrict__ table, const float* __restrict__ mlp, ShConst K,
               float* __restrict__ out, unsigned* flag) {
  extern __shared__ __align__(1024) uint8_t hsm[];
  float* vec = reinterpret_cast<float*>(hsm + HC_VEC);
  float* b1 = vec;
  float* ws = vec + 4 * 64;
  float* rw = ws + 68;                                      // [3][64]
  uint64_t* a_ready = reinterpret_cast<uint64_t*>(hsm + HC_BARS);   // [groups]
  uint64_t* mma_done = a_ready + HC_GROUPS;                          // [groups]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + HC_GROUPS + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  constexpr uint64_t kLimit = 2000000000ull;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // weights of the blob (row-major W[n][k], layer order d0, d1, sigma, c0, c1, rgb)
  // -> bf16 core-matrix operands; biases and head weights stay fp32
  for (int q = threadIdx.x; q < HASH_NW; q += HC_THREADS) {
    const float v = mlp[q];
    auto wput = [&](int base, int K_, int z) {
      const int n = z / K_, k = z % K_;
      *reinterpret_cast<__nv_bfloat16*>(hsm + base + hc_w_off(n, k)) = __float2bfloat16_rn(v);
    };
    if (q < 2048) wput(HC_W1, 32, q);
    else if (q < 2112) b1[q - 2048] = v;
    else if (q < 6208) wput(HC_W2, 64, q - 2112);
    else if (q < 6272) b1[64 + q - 6208] = v;
    else if (q < 6336) ws[q - 6272] = v;
    else if (q < 6337) ws[64] = v;
    else if (q < 11457) wput(HC_W3, 80, q - 6337);
    else if (q < 11521) b1[128 + q - 11457] = v;
    else if (q < 15617) wput(HC_W4, 64, q - 11521);
    else if (q < 15681) b1[192 + q - 15617] = v;
    else if (q < 15873) rw[q - 15681] = v;
    else rw[192 + q - 15873] = v;
  }
  if (threadIdx.x == 0) {
    for (int g = 0; g < HC_GROUPS; ++g) {
      tcx::mbar_init(&a_ready[g], 4);          // one arrival per warp of the group
      tcx::mbar_init(&mma_done[g], 1);
    }
    tcx::mbar_init(&mma_done[HC_GROUPS], 1);   // final drain
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tcx::smem_u32(tmem_holder)), "r"(HC_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tcx::fence_async_smem();                     // the staged weights, for the tensor cores
  tcx::fence_before();
  __syncthreads();
  tcx::fence_after();
  const uint32_t tmem = *tmem_holder;
  const int64_t P = *total;
  // tile (round k, group g): points [T * 128, T * 128 + 128), T = (k * grid + block) * groups + g
  auto tile_of = [&](int64_t k, int g) {
    return (k * gridDim.x + blockIdx.x) * HC_GROUPS + g;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t ph[HC_GROUPS] = {};
      const uint32_t a0 = tcx::smem_u32(hsm + HC_A);
      const uint32_t wb = tcx::smem_u32(hsm);
      bool ok = true;
      for (int64_t k = 0; ok; ++k) {
        int active = 0;
        while (active < HC_GROUPS && tile_of(k, active) * HC_P < P) ++active;
        if (active == 0) break;
        for (int l = 0; l < 4 && ok; ++l) {
          for (int g = 0; g < active; ++g) {
            if (!tcx::mbar_wait(&a_ready[g], ph[g], abort_flag, flag, kLimit)) { ok = false; break; }
            ph[g] ^= 1;
            tcx::fence_after();
            const uint64_t a = tcx::sdesc(a0 + g * HC_A_BYTES, HC_P * 16, 128);
            const uint32_t dt = tmem + 64 * g;
            if (l == 0) hc_layer_mma<2>(dt, a, tcx::sdesc(wb + HC_W1, 64 * 16, 128));
            else if (l == 1) hc_layer_mma<4>(dt, a, tcx::sdesc(wb + HC_W2, 64 * 16, 128));
            else if (l == 2) hc_layer_mma<5>(dt, a, tcx::sdesc(wb + HC_W3, 64 * 16, 128));
            else hc_layer_mma<4>(dt, a, tcx::sdesc(wb + HC_W4, 64 * 16, 128));
            tcx::mma_commit(&mma_done[g]);
          }
        }
      }
      // drain before TMEM is freed (not stopped by an abort: the MMAs already
      // issued must land first); running out is reported like any other wait
      uint64_t* fin = mma_done + HC_GROUPS;
      tcx::mma_commit(fin);
      const uint64_t t0 = tcx::globaltimer();
      bool drained = tcx::mbar_try(fin, 0);
      while (!drained && tcx::globaltimer() - t0 < kLimit) drained = tcx::mbar_try(fin, 0);
      if (!drained) {
        atomicOr(flag, FLAG_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else {
    const int g = (warp - 1) >> 2;
    const int r = (warp & 3) * 32 + lane;                  // TMEM lane = row of the tile
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t abase = tcx::smem_u32(hsm + HC_A + g * HC_A_BYTES);
    uint32_t pd = 0;
    for (int64_t k = 0;; ++k) {
      const int64_t T = tile_of(k, g);
      if (T * HC_P >= P) break;
      const int64_t i = T * HC_P + r;
      const bool valid = i < P;
      // encoding: 16 levels x 2 features and SH16 of the unit direction, bf16
      {
        float x[3] = {0.f, 0.f, 0.f}, t;
        int64_t ray = r0;
        if (valid) {
          const uint32_t e = live[i];
          ray = r0 + (e >> 9);
          march_point(o, d, ray, near, step, (int)(e & 511u), x, &t);
        }
        float u0, u1, u2;
        hash_unit_coords(x[0], x[1], x[2], u0, u1, u2);
#pragma unroll 1
        for (int l2 = 0; l2 < 16; l2 += 4) {
          float f[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            f[2 * j] = 0.f;
            f[2 * j + 1] = 0.f;
            if (valid) hash_encode_level(table, u0, u1, u2, l2 + j, nullptr, f[2 * j], f[2 * j + 1]);
          }
          tcx::st_shared_v4(abase + hc_a_off(r, l2 / 4), tcx::pack_bf16(f[0], f[1]),
                            tcx::pack_bf16(f[2], f[3]), tcx::pack_bf16(f[4], f[5]),
                            tcx::pack_bf16(f[6], f[7]));
        }
        float sh[16];
        const float dx = d[ray * 3], dy = d[ray * 3 + 1], dz = d[ray * 3 + 2];
        const float inv = 1.0f / sqrtf(dx * dx + dy * dy + dz * dz);
        sh16(dx * inv, dy * inv, dz * inv, K, sh);
#pragma unroll
        for (int j = 0; j < 2; ++j)
          tcx::st_shared_v4(abase + hc_a_off(r, 8 + j), tcx::pack_bf16(sh[8 * j], sh[8 * j + 1]),
                            tcx::pack_bf16(sh[8 * j + 2], sh[8 * j + 3]),
                            tcx::pack_bf16(sh[8 * j + 4], sh[8 * j + 5]),
                            tcx::pack_bf16(sh[8 * j + 6], sh[8 * j + 7]));
        tcx::fence_async_smem();
        __syncwarp();
        if (lane == 0) tcx::mbar_arrive(&a_ready[g]);
      }
      float sig = 0.f, c0 = 0.f, c1 = 0.f, c2 = 0.f;
      bool ok = true;
      for (int l = 0; l < 4; ++l) {
        if (!tcx::mbar_wait(&mma_done[g], pd, abort_flag, flag, kLimit)) { ok = false; break; }
        pd ^= 1;
        tcx::fence_after();
        const float* bias = b1 + 64 * l;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t u[32];
          tcx::tmem_ld32(tmem + lane_base + 64 * g + 32 * half, u);
          tcx::tmem_ld_wait(u);
#pragma unroll
          for (int j = 0; j < 4; ++j) {                   // 8 columns: one K-group
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int n = 32 * half + 8 * j + e;
              v[e] = fmaxf(__uint_as_float(u[8 * j + e]) + bias[n], 0.f);
              if (l == 1) sig = fmaf(v[e], ws[n], sig);
              if (l == 3) {
                c0 = fmaf(v[e], rw[n], c0);
                c1 = fmaf(v[e], rw[64 + n], c1);
                c2 = fmaf(v[e], rw[128 + n], c2);
              }
            }
            if (l < 3)
              tcx::st_shared_v4(abase + hc_a_off(r, 4 * half + j), tcx::pack_bf16(v[0], v[1]),
                                tcx::pack_bf16(v[2], v[3]), tcx::pack_bf16(v[4], v[5]),
                                tcx::pack_bf16(v[6], v[7]));
          }
        }
        tcx::fence_before();
        if (l < 3) {
          tcx::fence_async_smem();
          __syncwarp();
          if (lane == 0) tcx::mbar_arrive(&a_ready[g]);
        }
      }
      if (!ok) break;
      if (valid)
        reinterpret_cast<float4*>(out)[i] =
            make_float4(1.0f / (1.0f + expf(-(c0 + rw[192]))), 1.0f / (1.0f + expf(-(c1 + rw[193]))),
                        1.0f / (1.0f + expf(-(c2 + rw[194]))), fmaxf(sig + ws[64], 0.0f));
    }
  }
  tcx::fence_before();
  __syncthreads();
  if (warp == 0) {
    tcx::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(HC_TMEM_COLS));
  }
}

// ------------------------------------------------------------------ KiloNeRF

// The cell routing counts and scatters with one atomic per distinct cell among
// a warp's 32 points (__match_any_sync): consecutive live entries lie along one
// ray and share few cells, so hot cells see far fewer contended atomics. The
// loops step by whole warps so that every lane takes part in the match.
__device__ __forceinline__ void warp_hist_add(int32_t* hist, int id, int lane) {
  const unsigned peers = __match_any_sync(0xffffffffu, id);
  if (id >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[id], __popc(peers));
}

__global__ void cell_hist_kernel(const float* __restrict__ o, const float* __restrict__ d,
                                 int64_t r0, float near, float step,
                                 const uint32_t* __restrict__ live, const int32_t* __restrict__ total,
                                 int32_t* __restrict__ cell, int32_t* __restrict__ hist) {
  const int64_t P = *total;
  const int lane = threadIdx.x & 31;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); i0 < P;
       i0 += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = i0 + lane;
    int id = -1;
    if (i < P) {
      const uint32_t e = live[i];
      float x[3], t;
      march_point(o, d, r0 + (e >> 9), near, step, (int)(e & 511u), x, &t);
      const int a = voxel_axis(x[0]), b = voxel_axis(x[1]), c = voxel_axis(x[2]);
      id = ((a >> 3) * 16 + (b >> 3)) * 16 + (c >> 3);
      cell[i] = id;
    }
    warp_hist_add(hist, id, lane);
  }
}

__global__ void cell_hist_points_kernel(const float* __restrict__ x, int64_t n,
                                        int32_t* __restrict__ cell, int32_t* __restrict__ hist,
                                        unsigned* flag) {
  const int lane = threadIdx.x & 31;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  if (i0 >= n) return;                         // whole warps only
  const int64_t i = i0 + lane;
  int id = -1;
  if (i < n) {
    const int a = voxel_axis(x[i * 3]), b = voxel_axis(x[i * 3 + 1]), c = voxel_axis(x[i * 3 + 2]);
    if (a < 0 || b < 0 || c < 0) {
      atomicOr(flag, FLAG_BAD_INDEX);
    } else {
      id = ((a >> 3) * 16 + (b >> 3)) * 16 + (c >> 3);
    }
    cell[i] = id;
  }
  warp_hist_add(hist, id, lane);
}

__global__ void cell_scatter_kernel(const int32_t* __restrict__ cell, const int32_t* __restrict__ total,
                                    int64_t n_fixed, const int32_t* __restrict__ cell_off,
                                    int32_t* __restrict__ fill, int32_t* __restrict__ order) {
  const int64_t P = total ? (int64_t)*total : n_fixed;
  const int lane = threadIdx.x & 31;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); i0 < P;
       i0 += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = i0 + lane;
    const int c = i < P ? cell[i] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    const int leader = __ffs(peers) - 1;
    int base = 0;
    if (c >= 0 && lane == leader) base = atomicAdd(&fill[c], __popc(peers));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (c >= 0) order[cell_off[c] + base + __popc(peers & ((1u << lane) - 1u))] = (int32_t)i;
  }
}

constexpr int KILO_NP = 3317;

// Work items of the per-cell evaluation: every cell's run of the cell-grouped
// order split into tiles of at most KT_P points. One CTA of 1024 threads, four
// cells per thread, a block scan of the tile counts.
constexpr int KT_P = 128;
__global__ void __launch_bounds__(1024)
kilo_items_kernel(const int32_t* __restrict__ hist, const int32_t* __restrict__ cell_off,
                  int4* __restrict__ items, int32_t* __restrict__ n_items) {
  __shared__ int32_t sums[1024];
  const int t = threadIdx.x;
  int cnt[4], tot = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    cnt[j] = (hist[4 * t + j] + KT_P - 1) / KT_P;
    tot += cnt[j];
  }
  sums[t] = tot;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = t >= off ? sums[t - off] : 0;
    __syncthreads();
    sums[t] += v;
    __syncthreads();
  }
  int pos = sums[t] - tot;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = 4 * t + j, h = hist[c], base = cell_off[c];
    for (int q = 0; q < cnt[j]; ++q)
      items[pos++] = make_int4(c, base + q * KT_P, min(KT_P, h - q * KT_P), 0);
  }
  if (t == 1023) *n_items = sums[1023];
}

// The per-cell tiny MLPs, their two 32-wide layers on the tensor cores. A CTA
// runs a tile of up to 128 points of one cell at a time (consecutive items
// mostly share a cell, whose weights then stay staged):
//   gamma(x) (63 -> K 64) -> 32 -> 32 : tcgen05.mma kind::tf32, M = 128, N = 32,
//   the heads sigma (32 -> 1) and rgb ([h2, gamma(d)] 59 -> 3) : fp32 CUDA cores.
// fp32-level accuracy from tf32 operands: every operand value v is split into
// hi = v rounded to tf32 and lo = v - hi (exact in fp32), and a product of two
// operands is accumulated as hi*hi + hi*lo + lo*hi (the dropped lo*lo term is
// below 2^-22 of it; the tensor core reads lo at tf32 precision, 2^-11 of lo).
// The accumulation runs in fp32 in tensor memory; the bias and ReLU are applied
// by the epilogue in fp32.
constexpr int KT_AP = KT_P + 4;
constexpr int KT_THREADS = 256;
// shared memory, bytes: operands in the no-swizzle K-major core-matrix layout
// (8 rows x 16 bytes: 4 tf32 elements of K per row)
constexpr int KC_B1 = 0;                               // W1 hi, lo: 32 x 64 x 4 B each
constexpr int KC_B2 = KC_B1 + 2 * 32 * 64 * 4;         // W2 hi, lo: 32 x 32 x 4 B each
constexpr int KC_VEC = KC_B2 + 2 * 32 * 32 * 4;        // fp32: b1, b2, ws, bs, wc, bc
constexpr int KC_NV = 32 + 32 + 32 + 1 + 3 * 59 + 3;
constexpr int KC_A = (KC_VEC + KC_NV * 4 + 1023) / 1024 * 1024;  // A hi, lo: 128 x 64 x 4 B each
constexpr int KC_A_HALF = KT_P * 64 * 4;               // one of A hi / lo (32 KB)
constexpr int KC_DPE = KC_A + 2 * KC_A_HALF;           // [27][KT_AP] fp32: gamma(unit d)
constexpr int KC_SIG = KC_DPE + 27 * KT_AP * 4;        // [KT_P]
constexpr int KC_RGB = KC_SIG + KT_P * 4;              // [3][KT_P]
constexpr int KC_BAR = KC_RGB + 3 * KT_P * 4;
constexpr size_t KT_SMEM = KC_BAR + 16 + 16;
static_assert(KC_A % 1024 == 0 && KC_B2 % 16 == 0 && KC_DPE % 16 == 0, "operand alignment");
static_assert(32 * KT_AP * 4 <= 2 * KC_A_HALF, "h2 fits in the A operand area");
static_assert(2 * KT_THREADS - 3 * KT_P == KT_P, "the heads' second round leaves KT_P threads for sigma");

// Byte offset of element (r, k) in an operand of R rows, K-major core matrices.
__device__ __forceinline__ uint32_t kc_off(int r, int k, int R) {
  return (uint32_t)((k >> 2) * (R * 16) + (r >> 3) * 128 + (r & 7) * 16 + (k & 3) * 4);
}
// v = hi + lo with hi rounded to tf32 (nearest, ties away from zero) and lo exact.
__device__ __forceinline__ void tf32_split(float v, float& hi, float& lo) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(v));
  hi = __uint_as_float(h);
  lo = __fsub_rn(v, hi);
}
__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
// One 32-wide layer: D[128 x 32] = A[128 x K] B[32 x K]^T in three tf32 passes
// per K-step of 8 (issued by one thread).
template <int K>
__device__ __forceinline__ void kilo_layer_mma(uint32_t tmem, uint32_t a_hi, uint32_t b_hi,
                                               int b_half_bytes) {
  constexpr uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((32u >> 3) << 17) |
                             ((uint32_t)(KT_P >> 4) << 24);   // f32 <- tf32 x tf32, N 32, M 128
  const uint64_t ah = tcx::sdesc(a_hi, KT_P * 16, 128), al = tcx::sdesc(a_hi + KC_A_HALF, KT_P * 16, 128);
  const uint64_t bh = tcx::sdesc(b_hi, 32 * 16, 128), bl = tcx::sdesc(b_hi + b_half_bytes, 32 * 16, 128);
#pragma unroll
  for (int s = 0; s < K / 8; ++s) {
    const uint64_t da = (uint64_t)((s * 2 * KT_P * 16) >> 4), db = (uint64_t)((s * 2 * 32 * 16) >> 4);
    mma_tf32(tmem, ah + da, bh + db, idesc, s != 0);
    mma_tf32(tmem, ah + da, bl + db, idesc, 1);
    mma_tf32(tmem, al + da, bh + db, idesc, 1);
  }
}

__global__ void __launch_bounds__(KT_THREADS, 2)
kilo_eval_kernel(const float* __restrict__ o, const float* __restrict__ d, int64_t r0, float near,
                 float step, const uint32_t* __restrict__ live, const int32_t* __restrict__ order,
                 const int4* __restrict__ items, const int32_t* __restrict__ n_items,
                 const float* __restrict__ cell_w, float* __restrict__ out, unsigned* flag) {
  extern __shared__ __align__(1024) uint8_t ksm[];
  float* vecs = reinterpret_cast<float*>(ksm + KC_VEC);
  const float* b1 = vecs;
  const float* b2 = vecs + 32;
  const float* ws = vecs + 64;
  const float* bs = vecs + 96;
  const float* wc = vecs + 97;                         // [3][59]
  const float* bc = vecs + 97 + 3 * 59;
  float* stage = reinterpret_cast<float*>(ksm + KC_A); // gamma(x) [64][KT_P] fp32, before the split
  float* h2 = reinterpret_cast<float*>(ksm + KC_A);    // [32][KT_AP], after the second layer
  float* dpe = reinterpret_cast<float*>(ksm + KC_DPE);
  float* sig = reinterpret_cast<float*>(ksm + KC_SIG);
  float* rgbv = reinterpret_cast<float*>(ksm + KC_RGB);
  uint64_t* bar = reinterpret_cast<uint64_t*>(ksm + KC_BAR);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ksm + KC_BAR + 8);
  const uint32_t a_hi = tcx::smem_u32(ksm + KC_A);
  const int warp = threadIdx.x >> 5;
  const int p = threadIdx.x & (KT_P - 1);
  const int part = threadIdx.x / KT_P;          // 0: position encoding, 1: the rest of it and gamma(d)
  constexpr uint64_t kLimit = 2000000000ull;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    tcx::mbar_init(bar, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tcx::smem_u32(tmem_holder)), "r"(32));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tcx::fence_before();
  __syncthreads();
  tcx::fence_after();
  const uint32_t tmem = *tmem_holder;
  uint32_t phase = 0;
  // one thread issues a layer's MMAs and commits them; every thread waits and
  // all take the same decision on a timeout
  auto run_layer = [&](bool second) -> bool {
    tcx::fence_async_smem();
    tcx::fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tcx::fence_after();
      if (second) kilo_layer_mma<32>(tmem, a_hi, tcx::smem_u32(ksm + KC_B2), 32 * 32 * 4);
      else kilo_layer_mma<64>(tmem, a_hi, tcx::smem_u32(ksm + KC_B1), 32 * 64 * 4);
      tcx::mma_commit(bar);
    }
    const bool ok = tcx::mbar_wait(bar, phase, &abort_s, flag, kLimit);
    phase ^= 1;
    tcx::fence_after();
    return __syncthreads_and(ok) != 0;
  };
  // a contiguous run of items per CTA: the items are in cell order, so
  // consecutive items mostly share a cell and its weights stay staged
  const int NI = *n_items;
  const int per = (NI + (int)gridDim.x - 1) / (int)gridDim.x;
  const int it0 = (int)blockIdx.x * per;
  const int it1 = min(NI, it0 + per);
  int staged = -1;
  bool pending = false;          // a layer's wait gave up with its MMAs still in flight
  for (int it = it0; it < it1; ++it) {
    const int4 item = items[it];
    const int n = item.z;
    __syncthreads();     // the previous item's last reads are over
    if (item.x != staged) {
      // this cell's weights: W1 [32][63] and W2 [32][32] (row-major in the blob)
      // as tf32 hi / lo operands, K-major (W1's K padded to 64 with zeros); the
      // vectors in fp32
      staged = item.x;
      const float* W = cell_w + (int64_t)item.x * KILO_NP;
      for (int q = threadIdx.x; q < 32 * 64; q += KT_THREADS) {
        const int nn = q >> 6, k = q & 63;
        float hi, lo;
        tf32_split(k < 63 ? __ldg(W + nn * 63 + k) : 0.0f, hi, lo);
        *reinterpret_cast<float*>(ksm + KC_B1 + kc_off(nn, k, 32)) = hi;
        *reinterpret_cast<float*>(ksm + KC_B1 + 32 * 64 * 4 + kc_off(nn, k, 32)) = lo;
      }
      for (int q = threadIdx.x; q < 32 * 32; q += KT_THREADS) {
        const int nn = q >> 5, k = q & 31;
        float hi, lo;
        tf32_split(__ldg(W + 63 * 32 + 32 + q), hi, lo);
        *reinterpret_cast<float*>(ksm + KC_B2 + kc_off(nn, k, 32)) = hi;
        *reinterpret_cast<float*>(ksm + KC_B2 + 32 * 32 * 4 + kc_off(nn, k, 32)) = lo;
      }
      // blob order after W1: b1 (32), W2 (1024), b2 (32), ws (32), bs (1), wc (177), bc (3)
      for (int q = threadIdx.x; q < KC_NV; q += KT_THREADS)
        vecs[q] = __ldg(W + (q < 32 ? 63 * 32 + q : 63 * 32 + 32 + 32 * 32 + (q - 32)));
    }
    int64_t i = 0;
    if (p < n) i = order[item.y + p];
    {
      float x[3] = {0.f, 0.f, 0.f}, t;
      int64_t r = 0;
      if (p < n) {
        const uint32_t e = live[i];
        r = r0 + (e >> 9);
        march_point(o, d, r, near, step, (int)(e & 511u), x, &t);
      }
      // gamma(x) in fp32, k-major; the 42 sin/cos pairs split about evenly:
      // part 0 takes position coordinates 0 and 1 (20), part 1 coordinate 2
      // and the direction (10 + 12)
      if (part == 0) {
        stage[0 * KT_P + p] = x[0];
        stage[1 * KT_P + p] = x[1];
        stage[2 * KT_P + p] = x[2];
        stage[63 * KT_P + p] = 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int k = 0; k < 10; ++k) {
            float sn, cs;
            pe_sincos(x[c], k, &sn, &cs);
            stage[(3 + c * 10 + k) * KT_P + p] = sn;
            stage[(33 + c * 10 + k) * KT_P + p] = cs;
          }
      } else {
#pragma unroll
        for (int k = 0; k < 10; ++k) {
          float sn, cs;
          pe_sincos(x[2], k, &sn, &cs);
          stage[(3 + 20 + k) * KT_P + p] = sn;
          stage[(33 + 20 + k) * KT_P + p] = cs;
        }
        const float dx = d[r * 3], dy = d[r * 3 + 1], dz = d[r * 3 + 2];
        const float inv = 1.0f / sqrtf(dx * dx + dy * dy + dz * dz);
        const float u[3] = {dx * inv, dy * inv, dz * inv};
        dpe[0 * KT_AP + p] = u[0];
        dpe[1 * KT_AP + p] = u[1];
        dpe[2 * KT_AP + p] = u[2];
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float sn, cs;
            pe_sincos(u[c], k, &sn, &cs);
            dpe[(3 + c * 4 + k) * KT_AP + p] = sn;
            dpe[(15 + c * 4 + k) * KT_AP + p] = cs;
          }
      }
    }
    // the A operand of the first layer: this thread's point, K columns
    // [32 part, 32 part + 32), read from the staging area (which the operand
    // then overwrites), split into tf32 hi / lo, four columns per 16-byte store
    {
      __syncthreads();
      float g[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) g[k] = stage[(32 * part + k) * KT_P + p];
      __syncthreads();
#pragma unroll
      for (int kg = 0; kg < 8; ++kg) {
        float hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) tf32_split(g[4 * kg + j], hi[j], lo[j]);
        const uint32_t off = kc_off(p, 32 * part + 4 * kg, KT_P);
        tcx::st_shared_v4(a_hi + off, __float_as_uint(hi[0]), __float_as_uint(hi[1]),
                          __float_as_uint(hi[2]), __float_as_uint(hi[3]));
        tcx::st_shared_v4(a_hi + KC_A_HALF + off, __float_as_uint(lo[0]), __float_as_uint(lo[1]),
                          __float_as_uint(lo[2]), __float_as_uint(lo[3]));
      }
    }
    if (!run_layer(false)) { pending = true; break; }
    // h1 = ReLU(b1 + acc) as the second layer's A operand (tf32 hi / lo): warps
    // 0-3 read their TMEM lane quarter, 32 columns each
    if (warp < 4) {
      uint32_t u[32];
      tcx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), u);
      tcx::tmem_ld_wait(u);
#pragma unroll
      for (int kg = 0; kg < 8; ++kg) {
        float hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tf32_split(fmaxf(__fadd_rn(b1[4 * kg + j], __uint_as_float(u[4 * kg + j])), 0.0f), hi[j], lo[j]);
        const uint32_t off = kc_off(p, 4 * kg, KT_P);
        tcx::st_shared_v4(a_hi + off, __float_as_uint(hi[0]), __float_as_uint(hi[1]),
                          __float_as_uint(hi[2]), __float_as_uint(hi[3]));
        tcx::st_shared_v4(a_hi + KC_A_HALF + off, __float_as_uint(lo[0]), __float_as_uint(lo[1]),
                          __float_as_uint(lo[2]), __float_as_uint(lo[3]));
      }
    }
    if (!run_layer(true)) { pending = true; break; }
    // h2 = ReLU(b2 + acc), fp32, k-major for the heads
    if (warp < 4) {
      uint32_t u[32];
      tcx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), u);
      tcx::tmem_ld_wait(u);
#pragma unroll
      for (int k = 0; k < 32; ++k) h2[k * KT_AP + p] = fmaxf(__fadd_rn(b2[k], __uint_as_float(u[k])), 0.0f);
    }
    tcx::fence_before();
    __syncthreads();
    // heads: 3 KT_P rgb items and KT_P sigma items over two rounds of the 256
    // threads (sigma on the threads the rgb items leave idle in the second round)
    if (threadIdx.x >= 3 * KT_P - KT_THREADS) {
      const int pp = threadIdx.x - (3 * KT_P - KT_THREADS);
      float s = bs[0];
#pragma unroll 8
      for (int k = 0; k < 32; ++k) s = fmaf(ws[k], h2[k * KT_AP + pp], s);
      sig[pp] = fmaxf(s, 0.0f);
    }
    for (int q = threadIdx.x; q < 3 * KT_P; q += KT_THREADS) {
      const int c = q / KT_P, pp = q % KT_P;
      float v = bc[c];
#pragma unroll 8
      for (int k = 0; k < 32; ++k) v = fmaf(wc[c * 59 + k], h2[k * KT_AP + pp], v);
#pragma unroll
      for (int k = 0; k < 27; ++k) v = fmaf(wc[c * 59 + 32 + k], dpe[k * KT_AP + pp], v);
      rgbv[c * KT_P + pp] = 1.0f / (1.0f + expf(-v));
    }
    __syncthreads();
    if (part == 0 && p < n)
      reinterpret_cast<float4*>(out)[i] =
          make_float4(rgbv[p], rgbv[KT_P + p], rgbv[2 * KT_P + p], sig[p]);
  }
  // the MMAs this CTA issued complete before TMEM is freed: every layer was
  // waited for, or a wait gave up (raising the timeout flag) and the pending
  // MMAs get one more bounded wait here
  if (pending && threadIdx.x == 0) {
    const uint64_t t0 = tcx::globaltimer();
    while (!tcx::mbar_try(bar, phase ^ 1) && tcx::globaltimer() - t0 < kLimit) {
    }
  }
  tcx::fence_before();
  __syncthreads();
  if (warp == 0) {
    tcx::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(32));
  }
}

// ------------------------------------------------------------------ compositing

// Warp per ray over its live entries (already activated sigma, rgb); every
// live sample has delta = step * |d|. Early termination: stop before the first
// live sample whose transmittance (fp32) is below ert_T.
__global__ void march_composite_kernel(const float* __restrict__ d, int64_t r0, int64_t R,
                                       float near, float step, float ert_T,
                                       const int32_t* __restrict__ off,
                                       const uint32_t* __restrict__ live,
                                       const float* __restrict__ val, float* __restrict__ rgb,
                                       float* __restrict__ depth, float* __restrict__ acc_out) {
  const int lane = threadIdx.x & 31;
  const int64_t rl = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (rl >= R) return;
  const int64_t r = r0 + rl;
  const float dx = d[r * 3], dy = d[r * 3 + 1], dz = d[r * 3 + 2];
  const float delta = step * sqrtf(dx * dx + dy * dy + dz * dz);
  const int64_t b = off[rl], e = off[rl + 1];
  float S = 0.0f, cr = 0.f, cg = 0.f, cb = 0.f, dep = 0.f, acc = 0.f;
  bool done = false;
  for (int64_t s0 = b; s0 < e && !done; s0 += 32) {
    const int64_t i = s0 + lane;
    const bool in = i < e;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    float t = 0.0f;
    if (in) {
      v = reinterpret_cast<const float4*>(val)[i];
      t = fadd(near, fmul((float)(live[i] & 511u), step));
    }
    const float tau = in ? v.w * delta : 0.0f;
    float incl = tau;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      float q = __shfl_up_sync(0xffffffffu, incl, o2);
      if (lane >= o2) incl += q;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0f;
    const float T = expf(-(S + excl));
    bool keep = in;
    if (ert_T > 0.0f) {
      const uint32_t stop = __ballot_sync(0xffffffffu, in && T < ert_T);
      if (stop) {
        const int first = __ffs(stop) - 1;
        keep = in && lane < first;
        done = true;
      }
    }
    if (keep) {
      const float w = T * (-expm1f(-tau));
      cr += w * v.x; cg += w * v.y; cb += w * v.z;
      dep += w * t;
      acc += w;
    }
    S += __shfl_sync(0xffffffffu, incl, 31);
  }
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) {
    cr += __shfl_xor_sync(0xffffffffu, cr, o2);
    cg += __shfl_xor_sync(0xffffffffu, cg, o2);
    cb += __shfl_xor_sync(0xffffffffu, cb, o2);
    dep += __shfl_xor_sync(0xffffffffu, dep, o2);
    acc += __shfl_xor_sync(0xffffffffu, acc, o2);
  }
  if (lane == 0) {
    rgb[r * 3] = cr; rgb[r * 3 + 1] = cg; rgb[r * 3 + 2] = cb;
    depth[r] = dep;
    acc_out[r] = acc;
  }
}

// ------------------------------------------------------------------ launchers

static unsigned grid_for(int64_t work, int block, int max_blocks) {
  int64_t b = (work + block - 1) / block;
  if (b < 1) b = 1;
  return (unsigned)(b < max_blocks ? b : max_blocks);
}

cudaError_t launch_march_mask(const float* o, const float* d, int64_t R, float near, float step,
                              int K, const uint32_t* occ, uint32_t* mask, int32_t* count,
                              uint8_t* live_u8, cudaStream_t st) {
  if (K < 1 || K > 512) return cudaErrorInvalidValue;
  march_mask_kernel<<<(unsigned)((R + 7) / 8), 256, 0, st>>>(o, d, R, near, step, K, occ, mask,
                                                              count, live_u8);
  return cudaGetLastError();
}

cudaError_t march_render_chunk(const MarchArgs& a, cudaStream_t st) {
  const int64_t R = a.R;
  const KernelTimer& tm = a.timer;
  int slot = tm.begin(TK_MARCH_MASK, st);
  cudaError_t e = launch_march_mask(a.o + a.r0 * 3, a.d + a.r0 * 3, R, a.near, a.step, a.K, a.occ,
                                    a.ws.mask, a.ws.count, nullptr, st);
  tm.end(slot, st);
  if (e != cudaSuccess) return e;
  slot = tm.begin(TK_MARCH_COMPACT, st);
  e = exclusive_scan(a.ws.count, R, a.ws.off, a.ws.scan_tmp, st);
  if (e != cudaSuccess) return e;
  march_emit_kernel<<<(unsigned)((R + 7) / 8), 256, 0, st>>>(a.ws.mask, a.ws.off, R, a.K,
                                                             a.ws.live, a.ws.cap, a.flag);
  tm.end(slot, st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int32_t* total = a.ws.off + R;
  const unsigned g = (unsigned)(a.num_sms * 8);
  if (a.model == NERF_MODEL_HASHGRID) {
    slot = tm.begin(TK_NETWORK, st);
    if (a.hash_tc)
      hash_tc_kernel<<<(unsigned)a.num_sms, HC_THREADS, HC_SMEM, st>>>(
          a.o, a.d, a.r0, a.near, a.step, a.ws.live, total,
          reinterpret_cast<const __half2*>(a.hash_table), a.hash_mlp, a.sh, a.ws.val, a.flag);
    else
      hash_eval_kernel<<<(unsigned)(a.num_sms * HT_CTAS_PER_SM), HT_THREADS, HT_SMEM, st>>>(
          a.o, a.d, a.r0, a.near, a.step, a.ws.live, total,
          reinterpret_cast<const __half2*>(a.hash_table), a.hash_mlp, a.sh, a.ws.val);
    tm.end(slot, st);
  } else {
    slot = tm.begin(TK_ROUTER, st);
    cudaMemsetAsync(a.ws.cell_hist, 0, 2 * 4096 * sizeof(int32_t), st);
    cell_hist_kernel<<<g, 256, 0, st>>>(a.o, a.d, a.r0, a.near, a.step, a.ws.live, total,
                                        a.ws.cell, a.ws.cell_hist);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = exclusive_scan(a.ws.cell_hist, 4096, a.ws.cell_off, a.ws.scan_tmp, st);
    if (e != cudaSuccess) return e;
    cell_scatter_kernel<<<g, 256, 0, st>>>(a.ws.cell, total, 0, a.ws.cell_off, a.ws.cell_fill,
                                           a.ws.order);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kilo_items_kernel<<<1, 1024, 0, st>>>(a.ws.cell_hist, a.ws.cell_off, a.ws.items,
                                          a.ws.n_items);
    tm.end(slot, st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    slot = tm.begin(TK_NETWORK, st);
    kilo_eval_kernel<<<(unsigned)(a.num_sms * 2), KT_THREADS, KT_SMEM, st>>>(
        a.o, a.d, a.r0, a.near, a.step, a.ws.live, a.ws.order, a.ws.items, a.ws.n_items,
        a.cell_w, a.ws.val, a.flag);
    tm.end(slot, st);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  slot = tm.begin(TK_MARCH_COMPOSITE, st);
  march_composite_kernel<<<(unsigned)((R + 7) / 8), 256, 0, st>>>(
      a.d, a.r0, R, a.near, a.step, a.ert_T, a.ws.off, a.ws.live, a.ws.val, a.rgb, a.depth, a.acc);
  tm.end(slot, st);
  return cudaGetLastError();
}

cudaError_t launch_route_points(const float* x, int64_t n, int32_t* cell, int32_t* hist,
                                int32_t* off, int32_t* order, int32_t* fill, int32_t* scan_tmp,
                                unsigned* flag, cudaStream_t st) {
  cudaMemsetAsync(hist, 0, 4096 * sizeof(int32_t), st);
  cell_hist_points_kernel<<<grid_for(n, 256, 1 << 20), 256, 0, st>>>(x, n, cell, hist, flag);
  cudaError_t e = exclusive_scan(hist, 4096, off, scan_tmp, st);
  if (e != cudaSuccess || !order) return e == cudaSuccess ? cudaGetLastError() : e;
  cudaMemsetAsync(fill, 0, 4096 * sizeof(int32_t), st);
  cell_scatter_kernel<<<grid_for(n, 256, 4096), 256, 0, st>>>(cell, nullptr, n, off, fill, order);
  return cudaGetLastError();
}

cudaError_t launch_hash_encode(const float* x, int64_t n, const uint16_t* table, float* feat,
                               int32_t* rows, cudaStream_t st) {
  hash_encode_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(
      x, n, reinterpret_cast<const __half2*>(table), feat, rows);
  return cudaGetLastError();
}

cudaError_t launch_hash_encode_backward(const float* x, int64_t n, const float* d_feat,
                                       float* grad, int deterministic, cudaStream_t st) {
  const unsigned blocks = (unsigned)((n + 127) / 128);
  if (!deterministic) {
    hash_bw_kernel<false><<<blocks, 128, 0, st>>>(x, n, d_feat, grad, nullptr, nullptr);
    return cudaGetLastError();
  }
  const int64_t m = 2 * hash_grid_info().entries;
  unsigned long long* acc = nullptr;
  unsigned* mx = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&acc, m * sizeof(unsigned long long), st);
  if (e == cudaSuccess) e = cudaMallocAsync((void**)&mx, sizeof(unsigned), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(acc, 0, m * sizeof(unsigned long long), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(mx, 0, sizeof(unsigned), st);
  if (e == cudaSuccess) {
    absmax_kernel<<<1024, 256, 0, st>>>(d_feat, n * 32, mx);
    hash_bw_kernel<true><<<blocks, 128, 0, st>>>(x, n, d_feat, nullptr, acc, mx);
    fixed_to_grad_kernel<<<2048, 256, 0, st>>>(acc, m, mx, n, grad);
    e = cudaGetLastError();
  }
  if (acc) cudaFreeAsync(acc, st);
  if (mx) cudaFreeAsync(mx, st);
  return e;
}

cudaError_t launch_sh(const float* d, int64_t n, float* out, cudaStream_t st) {
  sh_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(d, n, sh_constants(), out);
  return cudaGetLastError();
}

cudaError_t march_prepare(cudaStream_t st) {
  (void)st;
  cudaError_t e = upload_hash_grid(hash_grid_info());
  if (e != cudaSuccess) return e;
  cudaError_t e2 = cudaFuncSetAttribute(hash_eval_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)HT_SMEM);
  if (e2 != cudaSuccess) return e2;
  e2 = cudaFuncSetAttribute(hash_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)HC_SMEM);
  if (e2 != cudaSuccess) return e2;
  return cudaFuncSetAttribute(kilo_eval_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)KT_SMEM);
}

}  // namespace nerfb
