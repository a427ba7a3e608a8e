// The training step's backward (NeRF page, "7. Training loop": loss =
// mse(rgb_coarse, target) + mse(rgb_fine, target); the coarse weights are
// detached before resampling, "6. Hierarchical sampling", so every pass has
// fixed sample positions). fp32 on the CUDA cores.
//
// Per pass (rows = rays x samples), with the forward's activations stored
// row-major as [gamma(x) (64) | h_0 .. h_{D-1} | feature | h_dir]:
//   composite_bw_kernel  d raw (rgb, sigma) per sample and the per-ray loss term
//   head_bw_kernel       d h_dir through the rgb head, masked by h_dir > 0
//   in_bw_kernel         d input = d out x W (tiled), + a rank-1 term, masked by
//                        the ReLU of the layer below
//   wgrad_kernel         dW = sum over rows of d out^T x input, and db, as a
//                        split-row tiled reduction added atomically into the
//                        gradient blob (fp32 atomics: the summation order, not
//                        the terms, varies between runs)
#include "nerf_internal.cuh"

namespace nerfb {

namespace {

constexpr int CB_WARPS = 4;
constexpr int CB_SMAX = 256;     // samples per ray on the training path

__device__ __forceinline__ float sigmoid_(float r) { return 1.0f / (1.0f + expf(-r)); }

__device__ __forceinline__ float sample_t_(const SampleSpec& ss, int64_t ray, int i) {
  if (ss.mode == SAMPLES_STRATIFIED) {
    uint32_t m = ss.perturb ? draw_bits(ss.key, (uint64_t)ray, 0, (uint32_t)i) : 0u;
    return stratified_t(ss.near, ss.step, i, m, ss.perturb != 0);
  }
  return ss.t[ray * ss.S + i];
}

// One warp per ray. Forward: T_i, w_i, rgb (as the compositing kernel computes
// them); the ray's loss term sum_k (rgb_k - y_k)^2 / (3 n_total); then the
// backward of sum_k d_k rgb_k with d_k = 2 (rgb_k - y_k) / (3 n_total):
//   d tau_i = sum_k d_k (T_{i+1} s_ik - sum_{j>i} w_j s_jk)
//             [- (T_{i+1} - sum_{j>i} w_j) sum_k d_k on a white background],
//   d sigma_raw_i = d tau_i delta_i act'(sigma_raw_i), d c_ik = d_k w_i s_ik (1 - s_ik).
// The suffix sums come from a reverse scan (no cancellation against the total).
__global__ void __launch_bounds__(CB_WARPS * 32)
composite_bw_kernel(const float* __restrict__ raw, SampleSpec ss, const float* __restrict__ d,
                    int64_t R, CompositeSpec cs, const float* __restrict__ target,
                    float inv3n, float* __restrict__ d_raw, float* __restrict__ loss_terms) {
  __shared__ float sm_w[CB_WARPS][CB_SMAX], sm_tn[CB_WARPS][CB_SMAX], sm_dl[CB_WARPS][CB_SMAX];
  __shared__ float sm_s[CB_WARPS][CB_SMAX][3];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ray = (int64_t)blockIdx.x * CB_WARPS + wid;
  if (ray >= R) return;
  const int S = ss.S;
  const float dx = d[ray * 3], dy = d[ray * 3 + 1], dz = d[ray * 3 + 2];
  const float dnorm = sqrtf(dx * dx + dy * dy + dz * dz);
  float carry = 0.0f, r = 0.f, g = 0.f, b = 0.f, acc = 0.f;
  for (int c0 = 0; c0 < S; c0 += 32) {
    const int i = c0 + lane;
    float tau = 0.0f, delta = 0.0f;
    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < S) {
      const float t = sample_t_(ss, ray, i);
      if (i + 1 < S) delta = (sample_t_(ss, ray, i + 1) - t) * dnorm;
      else delta = cs.last_mode == NERF_LAST_1E10 ? 1e10f * dnorm : (cs.far - t) * dnorm;
      q = *reinterpret_cast<const float4*>(raw + (ray * S + i) * 4);
      const float sigma = cs.sigma_act == NERF_SIGMA_SOFTPLUS
                              ? (q.w > 30.0f ? q.w : log1pf(expf(q.w))) : fmaxf(q.w, 0.0f);
      tau = sigma * delta;
    }
    float incl = tau;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0f;
    excl += carry;
    carry += __shfl_sync(0xffffffffu, incl, 31);
    if (i < S) {
      const float T = expf(-excl);
      const float w = T * (-expm1f(-tau));
      const float s0 = sigmoid_(q.x), s1 = sigmoid_(q.y), s2 = sigmoid_(q.z);
      sm_w[wid][i] = w;
      sm_tn[wid][i] = T * expf(-tau);
      sm_dl[wid][i] = delta;
      sm_s[wid][i][0] = s0; sm_s[wid][i][1] = s1; sm_s[wid][i][2] = s2;
      r += w * s0; g += w * s1; b += w * s2; acc += w;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    r += __shfl_xor_sync(0xffffffffu, r, off);
    g += __shfl_xor_sync(0xffffffffu, g, off);
    b += __shfl_xor_sync(0xffffffffu, b, off);
    acc += __shfl_xor_sync(0xffffffffu, acc, off);
  }
  if (cs.white) { r += 1.0f - acc; g += 1.0f - acc; b += 1.0f - acc; }
  const float e0 = r - target[ray * 3], e1 = g - target[ray * 3 + 1], e2 = b - target[ray * 3 + 2];
  if (lane == 0) loss_terms[ray] = (e0 * e0 + e1 * e1 + e2 * e2) * inv3n;
  const float d0 = 2.0f * e0 * inv3n, d1 = 2.0f * e1 * inv3n, d2 = 2.0f * e2 * inv3n;
  const float dsum = d0 + d1 + d2;
  __syncwarp();
  // backward, chunks from the last to the first
  float cw = 0.f, c0s = 0.f, c1s = 0.f, c2s = 0.f;   // sums over the later chunks
  const int last_chunk = ((S - 1) / 32) * 32;
  for (int c0 = last_chunk; c0 >= 0; c0 -= 32) {
    const int i = c0 + lane;
    float w = 0.f, s0 = 0.f, s1 = 0.f, s2 = 0.f;
    if (i < S) {
      w = sm_w[wid][i];
      s0 = sm_s[wid][i][0]; s1 = sm_s[wid][i][1]; s2 = sm_s[wid][i][2];
    }
    // inclusive suffix scans within the chunk (lane L sums lanes L..31)
    float aw = w, a0 = w * s0, a1 = w * s1, a2 = w * s2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float vw = __shfl_down_sync(0xffffffffu, aw, off);
      const float v0 = __shfl_down_sync(0xffffffffu, a0, off);
      const float v1 = __shfl_down_sync(0xffffffffu, a1, off);
      const float v2 = __shfl_down_sync(0xffffffffu, a2, off);
      if (lane + off < 32) { aw += vw; a0 += v0; a1 += v1; a2 += v2; }
    }
    // exclusive (j > i) = the next lane's inclusive suffix + the later chunks
    float nw = __shfl_down_sync(0xffffffffu, aw, 1), n0 = __shfl_down_sync(0xffffffffu, a0, 1);
    float n1 = __shfl_down_sync(0xffffffffu, a1, 1), n2 = __shfl_down_sync(0xffffffffu, a2, 1);
    if (lane == 31) { nw = 0.f; n0 = 0.f; n1 = 0.f; n2 = 0.f; }
    const float after_w = nw + cw, after0 = n0 + c0s, after1 = n1 + c1s, after2 = n2 + c2s;
    cw += __shfl_sync(0xffffffffu, aw, 0);
    c0s += __shfl_sync(0xffffffffu, a0, 0);
    c1s += __shfl_sync(0xffffffffu, a1, 0);
    c2s += __shfl_sync(0xffffffffu, a2, 0);
    if (i < S) {
      const float tn = sm_tn[wid][i];
      float dtau = d0 * (tn * s0 - after0) + d1 * (tn * s1 - after1) + d2 * (tn * s2 - after2);
      if (cs.white) dtau -= (tn - after_w) * dsum;
      const float4 q = *reinterpret_cast<const float4*>(raw + (ray * S + i) * 4);
      const float dact = cs.sigma_act == NERF_SIGMA_SOFTPLUS ? sigmoid_(q.w)
                                                             : (q.w > 0.0f ? 1.0f : 0.0f);
      const float dsig = dtau * sm_dl[wid][i] * dact;
      *reinterpret_cast<float4*>(d_raw + (ray * S + i) * 4) =
          make_float4(d0 * w * s0 * (1.0f - s0), d1 * w * s1 * (1.0f - s1),
                      d2 * w * s2 * (1.0f - s2), dsig);
    }
  }
}

// dz_dir[row][j] = (sum_c d_rgb[row][c] Wr[c][j]) * (h_dir[row][j] > 0).
__global__ void head_bw_kernel(const float* __restrict__ d_raw, const float* __restrict__ wr,
                               const float* __restrict__ save, int64_t ldc, int hcol, int64_t rows,
                               int Wh, float* __restrict__ dz) {
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= rows * Wh) return;
  const int64_t row = q / Wh;
  const int j = (int)(q % Wh);
  const float v = d_raw[row * 4] * __ldg(wr + j) + d_raw[row * 4 + 1] * __ldg(wr + Wh + j) +
                  d_raw[row * 4 + 2] * __ldg(wr + 2 * Wh + j);
  dz[q] = save[row * ldc + hcol + j] > 0.0f ? v : 0.0f;
}

// out[r][k] = (sum_n A[r][n] B[n][k] + ea[r] ev[k]) * (mask: save[r][mcol + k] > 0),
// k < Kout (a multiple of 64), n < N (a multiple of 16). 64 x 64 tiles, 4 x 4 per thread.
__global__ void __launch_bounds__(256)
in_bw_kernel(const float* __restrict__ A, int64_t lda, const float* __restrict__ B, int64_t ldb,
             int N, int Kout, int64_t rows, const float* __restrict__ ea, int64_t ldea,
             const float* __restrict__ ev, const float* __restrict__ save, int64_t ldc, int mcol,
             float* __restrict__ out, int64_t ldo) {
  __shared__ __align__(16) float As[16][64 + 4];   // [n][row]
  __shared__ __align__(16) float Bs[16][64];       // [n][k]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t r0 = (int64_t)blockIdx.x * 64;
  const int k0 = blockIdx.y * 64;
  float acc[4][4] = {};
  for (int n0 = 0; n0 < N; n0 += 16) {
    for (int q = threadIdx.x; q < 64 * 16; q += 256) {     // A tile, transposed into As[n][row]
      const int rr = q / 16, nn = q % 16;
      const int64_t row = r0 + rr;
      As[nn][rr] = row < rows ? A[row * lda + n0 + nn] : 0.0f;
    }
    for (int q = threadIdx.x; q < 16 * 64; q += 256) {
      const int nn = q / 64, kk = q % 64;
      Bs[nn][kk] = __ldg(B + (int64_t)(n0 + nn) * ldb + k0 + kk);
    }
    __syncthreads();
#pragma unroll
    for (int nn = 0; nn < 16; ++nn) {
      const float4 a = *reinterpret_cast<const float4*>(&As[nn][4 * ty]);
      const float4 w = *reinterpret_cast<const float4*>(&Bs[nn][4 * tx]);
      const float av[4] = {a.x, a.y, a.z, a.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = r0 + 4 * ty + i;
    if (row >= rows) continue;
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + 4 * tx + j;
      float x = acc[i][j];
      if (ea) x = fmaf(ea[row * ldea], __ldg(ev + k), x);
      if (save) x = save[row * ldc + mcol + k] > 0.0f ? x : 0.0f;
      v[j] = x;
    }
    *reinterpret_cast<float4*>(out + row * ldo + k0 + 4 * tx) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// G[n][k] += sum_r A[r][n] X(r, k) for n < N, k < K, and db[n] += sum_r A[r][n]
// (the virtual column k = K of ones). X(r, k) = X[r * ldx + c0 + k] for k < split,
// X[r * ldx + c1 + k - split] otherwise. Rows are cut into slices of WG_SLICE.
constexpr int WG_SLICE = 4096;
__global__ void __launch_bounds__(256)
wgrad_kernel(const float* __restrict__ A, int64_t lda, int N, const float* __restrict__ X,
             int64_t ldx, int c0, int split, int c1, int K, int64_t rows,
             float* __restrict__ G, int64_t ldg, float* __restrict__ db) {
  __shared__ __align__(16) float As[16][64];
  __shared__ __align__(16) float Xs[16][64];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int nb = blockIdx.x * 64, kb = blockIdx.y * 64;
  const int64_t rs = (int64_t)blockIdx.z * WG_SLICE;
  const int64_t re = rs + WG_SLICE < rows ? rs + WG_SLICE : rows;
  float acc[4][4] = {};
  for (int64_t r0 = rs; r0 < re; r0 += 16) {
    for (int q = threadIdx.x; q < 16 * 64; q += 256) {
      const int rr = q / 64, cc = q % 64;
      const int64_t row = r0 + rr;
      const int n = nb + cc, k = kb + cc;
      As[rr][cc] = (row < re && n < N) ? A[row * lda + n] : 0.0f;
      float xv = 0.0f;
      if (row < re) {
        if (k < K) xv = X[row * ldx + (k < split ? c0 + k : c1 + k - split)];
        else if (k == K) xv = 1.0f;
      }
      Xs[rr][cc] = xv;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
      const float4 a = *reinterpret_cast<const float4*>(&As[rr][4 * ty]);
      const float4 x = *reinterpret_cast<const float4*>(&Xs[rr][4 * tx]);
      const float av[4] = {a.x, a.y, a.z, a.w}, xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], xv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = nb + 4 * ty + i;
    if (n >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = kb + 4 * tx + j;
      if (k < K) atomicAdd(G + (int64_t)n * ldg + k, acc[i][j]);
      else if (k == K && db) atomicAdd(db + n, acc[i][j]);
    }
  }
}

// dz_ray[ray][j] = sum over the ray's samples of dz[ray * S + s][j].
__global__ void ray_sum_kernel(const float* __restrict__ dz, int64_t R, int S, int Wh,
                               float* __restrict__ out) {
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= R * Wh) return;
  const int64_t ray = q / Wh;
  const int j = (int)(q % Wh);
  float s = 0.0f;
  for (int i = 0; i < S; ++i) s += dz[(ray * S + i) * Wh + j];
  out[q] = s;
}

// gamma(d / |d|) per ray, the direction encoding of the forward (27 values).
__global__ void dir_enc_kernel(const float* __restrict__ d, int64_t R, int L_dir,
                               float* __restrict__ out) {
  const int64_t ray = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (ray >= R) return;
  const float dx = d[ray * 3], dy = d[ray * 3 + 1], dz = d[ray * 3 + 2];
  const float inv = 1.0f / sqrtf(dx * dx + dy * dy + dz * dz);
  const float u[3] = {dx * inv, dy * inv, dz * inv};
  const int ch = 3 + 6 * L_dir;
  float* o = out + ray * ch;
  o[0] = u[0]; o[1] = u[1]; o[2] = u[2];
  for (int c = 0; c < 3; ++c)
    for (int k = 0; k < L_dir; ++k) {
      float s, co;
      pe_sincos(u[c], k, &s, &co);
      o[3 + c * L_dir + k] = s;
      o[3 + 3 * L_dir + c * L_dir + k] = co;
    }
}

// out[0] = sum of n terms (one CTA; a fixed summation order).
__global__ void sum_kernel(const float* __restrict__ v, int64_t n, float* __restrict__ out) {
  __shared__ float part[256];
  float s = 0.0f;
  for (int64_t i = threadIdx.x; i < n; i += 256) s += v[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {
    if ((int)threadIdx.x < off) part[threadIdx.x] += part[threadIdx.x + off];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[0] = part[0];
}

unsigned blocks_for(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t launch_composite_bw(const float* raw, const SampleSpec& ss, const float* d, int64_t R,
                                const CompositeSpec& cs, const float* target, float inv3n,
                                float* d_raw, float* loss_terms, cudaStream_t st) {
  if (ss.S > CB_SMAX) return cudaErrorInvalidValue;
  composite_bw_kernel<<<blocks_for(R, CB_WARPS), CB_WARPS * 32, 0, st>>>(raw, ss, d, R, cs, target,
                                                                        inv3n, d_raw, loss_terms);
  return cudaGetLastError();
}

// Backward of one network over rows = R * S, given d_raw [rows][4] and the
// forward's activation store. Adds into grad (the flat gradient blob, zeroed
// by the caller). w: the network's fp32 blob. tmp: 2 * rows * W + R * (W/2 + 27)
// floats of scratch.
cudaError_t mlp_backward_fp32(const PackedFp32& p, int L_dir, const float* w, const float* save,
                              int64_t R, int S, const float* d, const float* d_raw,
                              float* grad, float* tmp, cudaStream_t st) {
  const int D = p.D, W = p.W, Wh = W / 2, skip = p.skip;
  const int dir_ch = 3 + 6 * L_dir;
  const int64_t rows = R * S;
  const int64_t ldc = 64 + (int64_t)(D + 1) * W + Wh;
  const int feat_col = 64 + D * W, hdir_col = 64 + (D + 1) * W;
  auto hcol = [&](int l) { return 64 + l * W; };
  // blob offsets (layer order: pts0..pts{D-1}, sigma, feature, dir, rgb; W then b)
  int64_t off = 0;
  int64_t wo[8], bo[8], Kl[8];
  for (int l = 0; l < D; ++l) {
    Kl[l] = l == 0 ? 63 : (l == skip + 1 ? W + 63 : W);
    wo[l] = off; off += W * Kl[l];
    bo[l] = off; off += W;
  }
  const int64_t sig_w = off, sig_b = off + W; off += W + 1;
  const int64_t feat_w = off, feat_b = off + (int64_t)W * W; off += (int64_t)W * W + W;
  const int64_t dir_w = off, dir_b = off + (int64_t)Wh * (W + dir_ch);
  off += (int64_t)Wh * (W + dir_ch) + Wh;
  const int64_t rgb_w = off, rgb_b = off + 3 * Wh;
  float* bufA = tmp;
  float* bufB = tmp + rows * W;
  float* dz_ray = bufB + rows * W;
  float* denc = dz_ray + R * Wh;
  const unsigned zs = blocks_for(rows, WG_SLICE);
  cudaError_t e;
#define NERF_WG(A, lda, N, X, ldx, c0, split, c1, K, nrows, G, ldg, db)                         \
  wgrad_kernel<<<dim3(blocks_for(N, 64), blocks_for((K) + 1, 64), blocks_for(nrows, WG_SLICE)), \
                 256, 0, st>>>(A, lda, N, X, ldx, c0, split, c1, K, nrows, G, ldg, db);          \
  if ((e = cudaGetLastError()) != cudaSuccess) return e
  (void)zs;
  // rgb head: dz_dir = (d_rgb x Wr) masked by h_dir > 0; dWr, dbr
  head_bw_kernel<<<blocks_for(rows * Wh, 256), 256, 0, st>>>(d_raw, w + rgb_w, save, ldc, hdir_col,
                                                             rows, Wh, bufA);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  NERF_WG(d_raw, 4, 3, save, ldc, hdir_col, Wh, 0, Wh, rows, grad + rgb_w, Wh, grad + rgb_b);
  // direction layer: input [feature | gamma(d)]; the gamma(d) part per ray
  NERF_WG(bufA, Wh, Wh, save, ldc, feat_col, W, 0, W, rows, grad + dir_w, W + dir_ch,
          grad + dir_b);
  ray_sum_kernel<<<blocks_for(R * Wh, 256), 256, 0, st>>>(bufA, R, S, Wh, dz_ray);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dir_enc_kernel<<<blocks_for(R, 128), 128, 0, st>>>(d, R, L_dir, denc);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  NERF_WG(dz_ray, Wh, Wh, denc, dir_ch, 0, dir_ch, 0, dir_ch, R, grad + dir_w + W, W + dir_ch,
          (float*)nullptr);
  // d feature = dz_dir x Wd[:, :W] (no activation on the feature layer)
  in_bw_kernel<<<dim3(blocks_for(rows, 64), W / 64), 256, 0, st>>>(
      bufA, Wh, w + dir_w, W + dir_ch, Wh, W, rows, nullptr, 0, nullptr, nullptr, 0, 0, bufB, W);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // feature and sigma heads, both reading h_{D-1}
  NERF_WG(bufB, W, W, save, ldc, hcol(D - 1), W, 0, W, rows, grad + feat_w, W, grad + feat_b);
  NERF_WG(d_raw + 3, 4, 1, save, ldc, hcol(D - 1), W, 0, W, rows, grad + sig_w, W, grad + sig_b);
  // d h_{D-1} = d feature x Wf + d sigma x ws, masked by h_{D-1} > 0
  in_bw_kernel<<<dim3(blocks_for(rows, 64), W / 64), 256, 0, st>>>(
      bufB, W, w + feat_w, W, W, W, rows, d_raw + 3, 4, w + sig_w, save, ldc, hcol(D - 1), bufA, W);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the trunk, top down: bufA holds dz of layer l
  for (int l = D - 1; l >= 0; --l) {
    if (l == 0) {
      NERF_WG(bufA, W, W, save, ldc, 0, 63, 0, 63, rows, grad + wo[0], Kl[0], grad + bo[0]);
    } else if (l == skip + 1) {
      NERF_WG(bufA, W, W, save, ldc, hcol(l - 1), W, 0, W + 63, rows, grad + wo[l], Kl[l],
              grad + bo[l]);
    } else {
      NERF_WG(bufA, W, W, save, ldc, hcol(l - 1), W, 0, W, rows, grad + wo[l], Kl[l], grad + bo[l]);
    }
    if (l > 0) {
      in_bw_kernel<<<dim3(blocks_for(rows, 64), W / 64), 256, 0, st>>>(
          bufA, W, w + wo[l], Kl[l], W, W, rows, nullptr, 0, nullptr, save, ldc, hcol(l - 1), bufB,
          W);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      float* t = bufA; bufA = bufB; bufB = t;
    }
  }
#undef NERF_WG
  return cudaSuccess;
}

cudaError_t launch_sum(const float* v, int64_t n, float* out, cudaStream_t st) {
  sum_kernel<<<1, 256, 0, st>>>(v, n, out);
  return cudaGetLastError();
}

}  // namespace nerfb
