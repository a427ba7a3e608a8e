// fp32 CUDA-core evaluation of the NeRF scene MLP (NeRF page, Section 2.4),
// fused with sample placement and positional encoding.
//
// One CTA of 2 W threads owns 128 consecutive rows (samples); their activations
// stay in shared memory for the whole network, feature-major, so every layer is a
// register-blocked product (8 x 8 outputs per thread) whose left operand is read
// straight from the activations and whose weights (packed K-major) stream
// through a shared-memory double buffer.
#include "nerf_internal.cuh"

namespace nerfb {

namespace {
struct PackSeg {
  int64_t src_off, dst_off;
  int N, K_take, K_pad, stride, transpose;
};
struct PackTable { PackSeg s[24]; int n; };

__global__ void pack_kernel(const void* __restrict__ src, int precision, PackTable tab,
                            float* __restrict__ dst) {
  const PackSeg sg = tab.s[blockIdx.y];
  int64_t total = sg.transpose ? (int64_t)sg.K_pad * sg.N : sg.N;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (int64_t)gridDim.x * blockDim.x) {
    float v;
    if (sg.transpose) {
      int k = (int)(q / sg.N), n = (int)(q % sg.N);
      int64_t i = sg.src_off + (int64_t)n * sg.stride + k;
      v = k < sg.K_take ? (precision == NERF_BF16
                               ? __bfloat162float(((const __nv_bfloat16*)src)[i])
                               : ((const float*)src)[i])
                        : 0.0f;
    } else {
      int64_t i = sg.src_off + q;
      v = precision == NERF_BF16 ? __bfloat162float(((const __nv_bfloat16*)src)[i])
                                 : ((const float*)src)[i];
    }
    dst[sg.dst_off + q] = v;
  }
}

}  // namespace

PackedFp32 plan_fp32(int D, int W, int skip, int pos_ch, int dir_ch) {
  (void)dir_ch;
  PackedFp32 p{};
  p.D = D; p.W = W; p.skip = skip; p.pos_ch = pos_ch;
  int64_t off = 0;
  auto a4 = [](int64_t x) { return (x + 3) & ~int64_t(3); };
  for (int l = 0; l < D; ++l) {
    int kpad = (l == 0) ? 64 : (l == skip + 1 ? W + 64 : W);
    p.layer_w[l] = off; off = a4(off + (int64_t)kpad * W);
    p.layer_b[l] = off; off = a4(off + W);
  }
  p.sigma_w = off; off = a4(off + W);
  p.sigma_b = off; off = a4(off + 1);
  p.feat_w = off; off = a4(off + (int64_t)W * W);
  p.feat_b = off; off = a4(off + W);
  p.dir_w = off; off = a4(off + (int64_t)W * (W / 2));
  p.rgb_w = off; off = a4(off + 3 * (W / 2));
  p.rgb_b = off; off = a4(off + 3);
  p.total = off;
  return p;
}

cudaError_t launch_pack_fp32(const void* blob, int precision, const PackedFp32& p, int dir_ch,
                             float* out, cudaStream_t st) {
  PackTable t{};
  int64_t so = 0;  // offset in the source blob (layer order of the ABI)
  const int W = p.W;
  for (int l = 0; l < p.D; ++l) {
    int k = (l == 0) ? p.pos_ch : (l == p.skip + 1 ? W + p.pos_ch : W);
    int kpad = (l == 0) ? 64 : (l == p.skip + 1 ? W + 64 : W);
    t.s[t.n++] = {so, p.layer_w[l], W, k, kpad, k, 1};
    so += (int64_t)W * k;
    t.s[t.n++] = {so, p.layer_b[l], W, 0, 0, 0, 0};
    so += W;
  }
  t.s[t.n++] = {so, p.sigma_w, W, 0, 0, 0, 0}; so += W;           // [1][W] row = vector
  t.s[t.n++] = {so, p.sigma_b, 1, 0, 0, 0, 0}; so += 1;
  t.s[t.n++] = {so, p.feat_w, W, W, W, W, 1}; so += (int64_t)W * W;
  t.s[t.n++] = {so, p.feat_b, W, 0, 0, 0, 0}; so += W;
  t.s[t.n++] = {so, p.dir_w, W / 2, W, W, W + dir_ch, 1};
  so += (int64_t)(W / 2) * (W + dir_ch) + W / 2;
  // rgb [3][W/2] kept row-major, then its bias
  if (t.n + 2 > 24) return cudaErrorInvalidValue;
  t.s[t.n++] = {so, p.rgb_w, 3 * (W / 2), 0, 0, 0, 0}; so += 3 * (W / 2);
  t.s[t.n++] = {so, p.rgb_b, 3, 0, 0, 0, 0};
  dim3 grid(64, t.n);
  pack_kernel<<<grid, 256, 0, st>>>(blob, precision, t, out);
  return cudaGetLastError();
}

namespace {

// Geometry for width W: a CTA of 2 W threads owns BM = 128 rows; thread (ty, tx)
// holds 8 x 8 outputs of a layer of N columns (N = W, or W / 2 for the direction
// layer): rows {4 ty + i, 64 + 4 ty + i} and columns {4 tx + j, N / 2 + 4 tx + j},
// i, j < 4, for tx < N / 8. A warp covers 2 (W >= 128) or 4 (W = 64) values of ty.
template <int W>
struct Cfg {
  static constexpr int BM = 128;
  static constexpr int NTH = 2 * W;
  static constexpr int BK = 8;                     // weight rows per staged slice
  static constexpr int LDA = BM + 4;               // one feature's BM row values
  static constexpr int LDB = W + 4;
  static constexpr int MIN_CTAS = W == 256 ? 1 : W == 128 ? 2 : 3;
  static constexpr int TXW = W / 8 < 16 ? W / 8 : 16;   // tx values per warp
};

// The activations are stored feature-major: actT[f][r] is feature f of row r,
// features [h (W) | gamma(x) (63) | 0], so the skip layer's input [h, gamma(x)]
// is features 0 .. W + 63 and layer 0's input is features W .. W + 63.
template <int W>
struct Smem {
  float actT[W + 64][Cfg<W>::LDA];
  float wb[2][Cfg<W>::BK][Cfg<W>::LDB];
  float sig[Cfg<W>::BM];
  float x[Cfg<W>::BM][3];
  int64_t ray[Cfg<W>::BM];
};

// One dense layer on the tile: out[r][n] = act(sum_k actT[f0 + k][r] Wt[k][n] + bias),
// Wt K-major [K][N] (K a multiple of BK), staged through shared memory in slices
// of BK rows with a register prefetch of the next slice; then written back as
// features 0 .. N - 1. bias[n], or row_bias[ray(r) * N + n] when given.
template <int W>
__device__ __forceinline__ void tile_layer(Smem<W>& sm, const float* __restrict__ Wt,
                                           const float* __restrict__ bias,
                                           const float* __restrict__ row_bias, int K, int f0,
                                           int N, bool relu, int ty, int tx) {
  using C = Cfg<W>;
  constexpr int PF = C::BK / 8;                 // float4 fetches per thread per slice
  const int tid = threadIdx.x;
  const int n4 = N / 4;
  const bool active = tx < N / 8;
  float4 pre[PF];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int i = 0; i < PF; ++i) {
      const int q = tid + i * C::NTH;
      const int k = q / n4, c = 4 * (q % n4);
      pre[i] = q < C::BK * n4 ? __ldg(reinterpret_cast<const float4*>(Wt + (int64_t)(k0 + k) * N + c))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto put = [&](int buf) {
#pragma unroll
    for (int i = 0; i < PF; ++i) {
      const int q = tid + i * C::NTH;
      if (q < C::BK * n4)
        *reinterpret_cast<float4*>(&sm.wb[buf][q / n4][4 * (q % n4)]) = pre[i];
    }
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  fetch(0);
  put(0);
  __syncthreads();
  const int steps = K / C::BK;
  const int c1 = N / 2 + 4 * tx;
  for (int s = 0; s < steps; ++s) {
    const int cur = s & 1;
    if (s + 1 < steps) fetch((s + 1) * C::BK);
    if (active) {
      const int fb = f0 + s * C::BK;
#pragma unroll
      for (int k = 0; k < C::BK; ++k) {
        const float4 a0 = *reinterpret_cast<const float4*>(&sm.actT[fb + k][4 * ty]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sm.actT[fb + k][64 + 4 * ty]);
        const float4 b0 = *reinterpret_cast<const float4*>(&sm.wb[cur][k][4 * tx]);
        const float4 b1 = *reinterpret_cast<const float4*>(&sm.wb[cur][k][c1]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
    }
    if (s + 1 < steps) put(cur ^ 1);
    __syncthreads();   // the last one also ends every read of the input features
  }
  if (active) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = j < 4 ? 4 * tx + j : c1 + j - 4;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r0 = 64 * h + 4 * ty;
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float b = row_bias ? row_bias[sm.ray[r0 + i] * N + c] : __ldg(bias + c);
          v[i] = acc[4 * h + i][j] + b;
          if (relu) v[i] = fmaxf(v[i], 0.0f);
        }
        *reinterpret_cast<float4*>(&sm.actT[c][r0]) = make_float4(v[0], v[1], v[2], v[3]);
      }
    }
  }
  __syncthreads();
}

template <int W>
__global__ void __launch_bounds__(Cfg<W>::NTH, Cfg<W>::MIN_CTAS)
mlp_fp32_kernel(PackedFp32 p, const float* __restrict__ pk, const float* __restrict__ dir_bias,
                const float* __restrict__ o, const float* __restrict__ d, int64_t R,
                SampleSpec ss, float* __restrict__ raw) {
  using C = Cfg<W>;
  constexpr int BM = C::BM;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<W>& sm = *reinterpret_cast<Smem<W>*>(smem_raw);
  const int64_t rows = R * ss.S;
  const int64_t row0 = (int64_t)blockIdx.x * BM;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int NBLK = (W / 8) / C::TXW;       // warps across the columns
  const int ty = (warp / NBLK) * (32 / C::TXW) + lane / C::TXW;
  const int tx = (warp % NBLK) * C::TXW + lane % C::TXW;

  // sample positions and points (fp32, same rounded ops as the oracle)
  if (tid < BM) {
    int64_t row = row0 + tid;
    float x0 = 0.f, x1 = 0.f, x2 = 0.f;
    int64_t ray = 0;
    if (row < rows) {
      ray = row / ss.S;
      int s = (int)(row % ss.S);
      if (ss.mode == SAMPLES_GIVEN_X) {
        x0 = ss.t[row * 3 + 0]; x1 = ss.t[row * 3 + 1]; x2 = ss.t[row * 3 + 2];
      } else {
        float t;
        if (ss.mode == SAMPLES_STRATIFIED) {
          uint32_t m = ss.perturb ? draw_bits(ss.key, (uint64_t)ray, 0, (uint32_t)s) : 0u;
          t = stratified_t(ss.near, ss.step, s, m, ss.perturb != 0);
        } else {
          t = ss.t[row];
        }
        x0 = fadd(o[ray * 3 + 0], fmul(t, d[ray * 3 + 0]));
        x1 = fadd(o[ray * 3 + 1], fmul(t, d[ray * 3 + 1]));
        x2 = fadd(o[ray * 3 + 2], fmul(t, d[ray * 3 + 2]));
      }
    }
    sm.x[tid][0] = x0; sm.x[tid][1] = x1; sm.x[tid][2] = x2;
    sm.ray[tid] = ray;
  }
  __syncthreads();
  // gamma(x) into features W .. W + 63 (the last one zero), one row per lane
  for (int q = tid; q < BM * 64; q += C::NTH) {
    const int r = q % BM, j = q / BM;
    float v = 0.0f;
    if (j < 3) {
      v = sm.x[r][j];
    } else if (j < 63) {
      const int jj = (j - 3) % 30;
      float sn, cs;
      pe_sincos(sm.x[r][jj / 10], jj % 10, &sn, &cs);
      v = (j - 3 < 30) ? sn : cs;
    }
    sm.actT[W + j][r] = v;
  }
  __syncthreads();

  for (int l = 0; l < p.D; ++l) {
    const int K = (l == 0) ? 64 : (l == p.skip + 1 ? W + 64 : W);
    tile_layer<W>(sm, pk + p.layer_w[l], pk + p.layer_b[l], nullptr, K, l == 0 ? W : 0, W, true,
                  ty, tx);
  }
  // sigma head from h_{D-1}
  if (tid < BM) {
    float a = 0.0f;
    for (int k = 0; k < W; ++k) a = fmaf(sm.actT[k][tid], __ldg(pk + p.sigma_w + k), a);
    sm.sig[tid] = a + __ldg(pk + p.sigma_b);
  }
  // (the feature layer's first barrier orders these reads before its writes)
  tile_layer<W>(sm, pk + p.feat_w, pk + p.feat_b, nullptr, W, 0, W, false, ty, tx);
  tile_layer<W>(sm, pk + p.dir_w, nullptr, dir_bias, W, 0, W / 2, true, ty, tx);
  // rgb head and output
  for (int q = tid; q < BM * 3; q += C::NTH) {
    const int r = q / 3, c = q % 3;
    const float* w = pk + p.rgb_w + c * (W / 2);
    float a = __ldg(pk + p.rgb_b + c);
    for (int k = 0; k < W / 2; ++k) a = fmaf(sm.actT[k][r], __ldg(w + k), a);
    const int64_t row = row0 + r;
    if (row < rows) raw[row * 4 + c] = a;
  }
  if (tid < BM) {
    const int64_t row = row0 + tid;
    if (row < rows) raw[row * 4 + 3] = sm.sig[tid];
  }
}

}  // namespace

cudaError_t launch_mlp_fp32(const PackedFp32& p, const float* packed, const float* dir_bias,
                            const float* o, const float* d, int64_t R, const SampleSpec& ss,
                            float* raw, cudaStream_t st) {
  const int64_t rows = R * ss.S;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 127) / 128);
  cudaError_t e = cudaErrorInvalidValue;
  auto go = [&](auto kern, int nth, size_t sh) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    if (e != cudaSuccess) return;
    kern<<<blocks, nth, sh, st>>>(p, packed, dir_bias, o, d, R, ss, raw);
    e = cudaGetLastError();
  };
  if (p.W == 256) go(mlp_fp32_kernel<256>, Cfg<256>::NTH, sizeof(Smem<256>));
  else if (p.W == 128) go(mlp_fp32_kernel<128>, Cfg<128>::NTH, sizeof(Smem<128>));
  else if (p.W == 64) go(mlp_fp32_kernel<64>, Cfg<64>::NTH, sizeof(Smem<64>));
  return e;
}

}  // namespace nerfb
