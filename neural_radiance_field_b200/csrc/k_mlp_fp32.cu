// fp32 CUDA-core evaluation of the NeRF scene MLP (NeRF page, Section 2.4),
// fused with sample placement and positional encoding.
//
// One CTA of 256 threads owns BM = 64 consecutive rows (samples); their
// activations stay in shared memory for the whole network as fp32 rows of
// [h (W columns) | gamma(x) (63 columns + 1 zero pad)], so the skip layer's input
// [h, gamma(x)] is simply the first W + 64 columns. Each layer is a register-
// blocked product with the packed, K-major weights read through L1.
#include "nerf_internal.cuh"

namespace nerfb {

namespace {
constexpr int BM = 64;
constexpr int NT = 256;

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

// Rows r = blockIdx.x * BM + i; sample s of ray r / S.
template <int W>
struct Smem {
  static constexpr int LD = W + 64;  // fp32 row stride of the activation tile
  float act[BM][LD];
  float sig[BM];
  float x[BM][3];
  int64_t ray[BM];
};

// One dense layer on the tile: out[:, out_col + n] = act(act[:, in_col:in_col+K] Wt + b),
// Wt K-major [K][N]. Thread (tx, ty) owns columns tx*8..tx*8+7 and RPT rows.
template <int W, int N>
__device__ __forceinline__ void tile_layer(Smem<W>& sm, const float* __restrict__ Wt,
                                           const float* __restrict__ bias,
                                           const float* __restrict__ row_bias, int K,
                                           int in_col, int out_col, bool relu) {
  constexpr int TPC = N / 8;          // threads across the columns
  constexpr int RG = NT / TPC;        // row groups
  constexpr int RPT = BM / RG;        // rows per thread
  static_assert(RPT >= 1 && BM % RG == 0, "tile shape");
  const int tx = threadIdx.x % TPC, ty = threadIdx.x / TPC;
  const int c0 = tx * 8;
  float acc[RPT][8];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int k = 0; k < K; k += 4) {
    float4 a[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      a[i] = *reinterpret_cast<const float4*>(&sm.act[ty * RPT + i][in_col + k]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float4 w0 = __ldg(reinterpret_cast<const float4*>(Wt + (int64_t)(k + kk) * N + c0));
      const float4 w1 =
          __ldg(reinterpret_cast<const float4*>(Wt + (int64_t)(k + kk) * N + c0 + 4));
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const float av = kk == 0 ? a[i].x : kk == 1 ? a[i].y : kk == 2 ? a[i].z : a[i].w;
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av, wv[j], acc[i][j]);
      }
    }
  }
  __syncthreads();  // every read of the input columns is done
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = ty * RPT + i;
    const float* rb = row_bias ? row_bias + sm.ray[r] * N : nullptr;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float b = rb ? rb[c0 + j] : __ldg(bias + c0 + j);
      v[j] = acc[i][j] + b;
      if (relu) v[j] = fmaxf(v[j], 0.0f);
    }
    *reinterpret_cast<float4*>(&sm.act[r][out_col + c0]) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(&sm.act[r][out_col + c0 + 4]) =
        make_float4(v[4], v[5], v[6], v[7]);
  }
  __syncthreads();
}

// Copies columns [src, src + n) of the tile's activations to columns
// [dst, dst + n) of the training path's activation store (row-major, ld floats
// per row; n a multiple of 4).
template <int W>
__device__ __forceinline__ void store_cols(const Smem<W>& sm, float* save, int64_t ld,
                                           int64_t row0, int64_t rows, int src, int64_t dst,
                                           int n) {
  const int n4 = n / 4;
  for (int q = threadIdx.x; q < BM * n4; q += NT) {
    const int r = q / n4, c = 4 * (q % n4);
    const int64_t row = row0 + r;
    if (row < rows)
      *reinterpret_cast<float4*>(save + row * ld + dst + c) =
          *reinterpret_cast<const float4*>(&sm.act[r][src + c]);
  }
}

template <int W>
__global__ void __launch_bounds__(NT, 1)
mlp_fp32_kernel(PackedFp32 p, const float* __restrict__ pk, const float* __restrict__ dir_bias,
                const float* __restrict__ o, const float* __restrict__ d, int64_t R,
                SampleSpec ss, float* __restrict__ raw, float* __restrict__ save) {
  // save (training path, else NULL): per row [gamma(x) (64) | h_0 .. h_{D-1} |
  // feature | h_dir], the layers' post-activation outputs
  const int64_t ldc = 64 + (int64_t)(p.D + 1) * W + W / 2;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<W>& sm = *reinterpret_cast<Smem<W>*>(smem_raw);
  const int64_t rows = R * ss.S;
  const int64_t row0 = (int64_t)blockIdx.x * BM;
  const int tid = threadIdx.x;

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
  // gamma(x) into columns W .. W+63 (last one zero)
  for (int q = tid; q < BM * 64; q += NT) {
    int r = q / 64, j = q % 64;
    float v = 0.0f;
    if (j < 3) {
      v = sm.x[r][j];
    } else if (j < 63) {
      int jj = (j - 3) % 30;
      float s, c;
      pe_sincos(sm.x[r][jj / 10], jj % 10, &s, &c);
      v = (j - 3 < 30) ? s : c;
    }
    sm.act[r][W + j] = v;
  }
  __syncthreads();
  if (save) store_cols<W>(sm, save, ldc, row0, rows, W, 0, 64);

  for (int l = 0; l < p.D; ++l) {
    int K = (l == 0) ? 64 : (l == p.skip + 1 ? W + 64 : W);
    int in_col = (l == 0) ? W : 0;
    tile_layer<W, W>(sm, pk + p.layer_w[l], pk + p.layer_b[l], nullptr, K, in_col, 0, true);
    if (save) store_cols<W>(sm, save, ldc, row0, rows, 0, 64 + (int64_t)l * W, W);
  }
  // sigma head from h (4 threads per row)
  {
    int r = tid / 4, part = tid % 4;
    float a = 0.0f;
    for (int k = part; k < W; k += 4) a = fmaf(sm.act[r][k], __ldg(pk + p.sigma_w + k), a);
    a += __shfl_xor_sync(0xffffffffu, a, 1);
    a += __shfl_xor_sync(0xffffffffu, a, 2);
    if (part == 0) sm.sig[r] = a + __ldg(pk + p.sigma_b);
  }
  // feature layer (no activation), then the direction layer with its per-ray bias
  tile_layer<W, W>(sm, pk + p.feat_w, pk + p.feat_b, nullptr, W, 0, 0, false);
  if (save) store_cols<W>(sm, save, ldc, row0, rows, 0, 64 + (int64_t)p.D * W, W);
  tile_layer<W, W / 2>(sm, pk + p.dir_w, nullptr, dir_bias, W, 0, 0, true);
  if (save) store_cols<W>(sm, save, ldc, row0, rows, 0, 64 + (int64_t)(p.D + 1) * W, W / 2);
  // rgb head and output
  if (tid < BM * 3) {
    int r = tid / 3, c = tid % 3;
    const float* w = pk + p.rgb_w + c * (W / 2);
    float a = __ldg(pk + p.rgb_b + c);
    for (int k = 0; k < W / 2; ++k) a = fmaf(sm.act[r][k], __ldg(w + k), a);
    int64_t row = row0 + r;
    if (row < rows) raw[row * 4 + c] = a;
  }
  if (tid < BM) {
    int64_t row = row0 + tid;
    if (row < rows) raw[row * 4 + 3] = sm.sig[tid];
  }
}

}  // namespace

cudaError_t launch_mlp_fp32(const PackedFp32& p, const float* packed, const float* dir_bias,
                            const float* o, const float* d, int64_t R, const SampleSpec& ss,
                            float* raw, cudaStream_t st, float* save) {
  int64_t rows = R * ss.S;
  unsigned blocks = (unsigned)((rows + BM - 1) / BM);
  if (p.W == 256) {
    size_t sh = sizeof(Smem<256>);
    cudaFuncSetAttribute(mlp_fp32_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    mlp_fp32_kernel<256><<<blocks, NT, sh, st>>>(p, packed, dir_bias, o, d, R, ss, raw, save);
  } else if (p.W == 128) {
    size_t sh = sizeof(Smem<128>);
    cudaFuncSetAttribute(mlp_fp32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    mlp_fp32_kernel<128><<<blocks, NT, sh, st>>>(p, packed, dir_bias, o, d, R, ss, raw, save);
  } else if (p.W == 64) {
    size_t sh = sizeof(Smem<64>);
    cudaFuncSetAttribute(mlp_fp32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    mlp_fp32_kernel<64><<<blocks, NT, sh, st>>>(p, packed, dir_bias, o, d, R, ss, raw, save);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace nerfb
