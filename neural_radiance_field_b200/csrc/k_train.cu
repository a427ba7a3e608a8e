// The training step (NeRF page, "7. Training loop": loss =
// mse(rgb_coarse, target) + mse(rgb_fine, target); the coarse weights are
// detached before resampling, "6. Hierarchical sampling", so every pass has
// fixed sample positions), at fp32-level accuracy: the layer GEMMs run on the
// tensor cores as three tf32 products per fp32 product (hi*hi + hi*lo + lo*hi),
// the rest in fp32 on the CUDA cores. The same forward, with a compact store,
// is precision TF32's render.
//
// Per pass (rows = rays x samples), the forward writes every layer's output to
// an activation store, row-major [gamma(x) (64) | h_0 .. h_{D-1} | feature | h_dir]:
//   encode_store_kernel   sample points and gamma(x)
//   row GEMM              one launch per layer, reading the previous layer's
//                         columns: row_gemm_pair_kernel (2-SM pairs, 256 rows or
//                         more), row_gemm_tc_kernel (one CTA), row_gemm_kernel
//                         (CUDA cores: 64 outputs, other K)
//   heads_fwd_kernel      sigma and rgb (raw outputs)
// and the backward reads it:
//   composite_bw_kernel   d raw (rgb, sigma) per sample and the per-ray loss term
//   head_bw_kernel        d h_dir through the rgb head, masked by h_dir > 0
//   row GEMM              d input = d out x W, + a rank-1 term, masked by the ReLU
//                         of the layer below
//   wgrad_tc_kernel       dW = sum over rows of d out^T x input, and db (the rows as
//                         the MMA's K; partial tiles added with fp32 atomics: the
//                         summation order, not the terms, varies between runs);
//                         wgrad_gemm_kernel on the CUDA cores for other shapes,
//                         wgrad_head_kernel for the 1- and 3-output heads
#include <algorithm>

#include <cuda.h>

#include "nerf_internal.cuh"
#include "tc_ptx.cuh"

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

// ---------------------------------------------------------------------------
// Register-blocked fp32 GEMM core. A CTA of 256 threads computes a 128 x 128
// output tile; thread (ty, tx) = (tid / 16, tid % 16) owns rows
// {4 ty + i, 64 + 4 ty + i} and columns {4 tx + j, 64 + 4 tx + j}, i, j < 4 (8 x 8
// accumulators). The reduction runs in steps of 8 through a shared-memory
// double buffer: the next step's operands are fetched into registers while the
// current step computes, so a step costs one barrier. Each output accumulates
// its terms in reduction order with fmaf.
// ---------------------------------------------------------------------------
constexpr int GT = 128;          // tile edge
constexpr int GK = 16;           // reduction step (two fetch rounds of 8)
constexpr int GLD = GT + 4;      // padded row of a shared operand tile

struct GemmSmem {
  float a[2][GK][GLD];   // [step][reduction index][tile row]
  float b[2][GK][GLD];   // [step][reduction index][tile column]
};

__device__ __forceinline__ void gemm_step(const float (&a)[GK][GLD], const float (&b)[GK][GLD],
                                          float (&acc)[8][8], int ty, int tx) {
#pragma unroll
  for (int k = 0; k < GK; ++k) {
    const float4 a0 = *reinterpret_cast<const float4*>(&a[k][4 * ty]);
    const float4 a1 = *reinterpret_cast<const float4*>(&a[k][64 + 4 * ty]);
    const float4 b0 = *reinterpret_cast<const float4*>(&b[k][4 * tx]);
    const float4 b1 = *reinterpret_cast<const float4*>(&b[k][64 + 4 * tx]);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// Four consecutive floats of a row: p[0..3] with element e valid when ok[e].
__device__ __forceinline__ float4 load4(const float* p, bool vec, bool ok0, bool ok1, bool ok2,
                                        bool ok3) {
  if (vec && ok3) return __ldg(reinterpret_cast<const float4*>(p));
  return make_float4(ok0 ? __ldg(p) : 0.f, ok1 ? __ldg(p + 1) : 0.f, ok2 ? __ldg(p + 2) : 0.f,
                     ok3 ? __ldg(p + 3) : 0.f);
}

// out[r][c] = epi( sum_k A(r, k) B[k][c] ) for r < rows, c < n_out, where
// A(r, k) = A[r * lda + a0 + k] for k < a_split, A[r * lda + a1 + k - a_split]
// otherwise (a row made of two column ranges, as the skip layer's [h, gamma(x)]),
// K a multiple of 8 with a_split a multiple of 8. The epilogue, in this order:
// + bias[c]; + row_bias[(r / rb_div) * n_out + c]; + ea[r * ldea] ev[c] (fmaf);
// ReLU; zero where mask[r * ldm + c] <= 0.
struct RowGemm {
  const float* A; int64_t lda; int a0, a_split, a1;
  const float* B; int64_t ldb;
  int K, n_out; int64_t rows;
  const float* bias;
  const float* row_bias; int rb_div;
  const float* ea; int64_t ldea; const float* ev;
  int relu;
  const float* mask; int64_t ldm;
  float* out; int64_t ldo;
  int a_vec, b_vec;
  float* bsplit;   // scratch for the tensor-core path's split weights (K x n_out x 2 floats)
  unsigned* flag;  // the context's error flag (bounded waits of the tensor-core path)
};

__global__ void __launch_bounds__(256, 2) row_gemm_kernel(RowGemm g) {
  __shared__ __align__(16) GemmSmem sm;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.x * GT;
  const int n0 = blockIdx.y * GT;
  // operand fetch roles: A row (tid / 2), reduction offset 4 (tid % 2); B reduction
  // index tid / 32, columns 4 (tid % 32)
  const int64_t ar = m0 + (tid >> 1);
  const int ak = (tid & 1) * 4;
  const bool a_row_ok = ar < g.rows;
  const int bk = tid >> 5, bc = n0 + (tid & 31) * 4;
  auto fetch_a = [&](int k0) -> float4 {
    const int k = k0 + ak;
    const int col = k < g.a_split ? g.a0 + k : g.a1 + k - g.a_split;
    return a_row_ok ? load4(g.A + ar * g.lda + col, g.a_vec, true, true, true, true)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto fetch_b = [&](int k0) -> float4 {
    const float* p = g.B + (int64_t)(k0 + bk) * g.ldb + bc;
    return load4(p, g.b_vec, bc < g.n_out, bc + 1 < g.n_out, bc + 2 < g.n_out, bc + 3 < g.n_out);
  };
  auto put = [&](int buf, int kh, float4 va, float4 vb) {
    sm.a[buf][kh + ak + 0][tid >> 1] = va.x;
    sm.a[buf][kh + ak + 1][tid >> 1] = va.y;
    sm.a[buf][kh + ak + 2][tid >> 1] = va.z;
    sm.a[buf][kh + ak + 3][tid >> 1] = va.w;
    *reinterpret_cast<float4*>(&sm.b[buf][kh + bk][(tid & 31) * 4]) = vb;
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  put(0, 0, fetch_a(0), fetch_b(0));
  put(0, 8, fetch_a(8), fetch_b(8));
  __syncthreads();
  const int steps = g.K / GK;
  for (int s = 0; s < steps; ++s) {
    const int cur = s & 1;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 na0 = z, nb0 = z, na1 = z, nb1 = z;
    if (s + 1 < steps) {
      na0 = fetch_a((s + 1) * GK); nb0 = fetch_b((s + 1) * GK);
      na1 = fetch_a((s + 1) * GK + 8); nb1 = fetch_b((s + 1) * GK + 8);
    }
    gemm_step(sm.a[cur], sm.b[cur], acc, ty, tx);
    if (s + 1 < steps) { put(cur ^ 1, 0, na0, nb0); put(cur ^ 1, 8, na1, nb1); }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = m0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
    if (row >= g.rows) continue;
    const float* rb = g.row_bias ? g.row_bias + (row / g.rb_div) * g.n_out : nullptr;
    const float e = g.ea ? g.ea[row * g.ldea] : 0.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = n0 + 64 * h + 4 * tx;
      if (c >= g.n_out) continue;
      float v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float x = acc[i][4 * h + j];
        if (g.bias) x += __ldg(g.bias + c + j);
        if (rb) x += rb[c + j];
        if (g.ea) x = fmaf(e, __ldg(g.ev + c + j), x);
        if (g.relu) x = fmaxf(x, 0.0f);
        if (g.mask) x = g.mask[row * g.ldm + c + j] > 0.0f ? x : 0.0f;
        v[j] = x;
      }
      *reinterpret_cast<float4*>(g.out + row * g.ldo + c) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

// The same row GEMM on the tensor cores (tcgen05.mma kind::tf32, M = 128 rows
// per CTA, N = n_out, 128 or 256), with fp32-level accuracy: every operand
// value v is split into hi = v rounded to tf32 and lo = v - hi (exact in
// fp32), and each product accumulates hi*hi + hi*lo + lo*hi in fp32 in tensor
// memory (the dropped lo*lo term is below 2^-22 of it). The weights B are split
// once per call by split_b_kernel into K chunks of 32 in the MMA's K-major
// core-matrix layout, and a chunk's split weights (hi then lo, contiguous)
// arrive by one bulk copy; the CTA splits its A rows chunk by chunk into shared
// memory, double-buffered against the MMAs of the previous chunk. The epilogue
// applies row_gemm_kernel's steps in the same order. Accumulation runs in the
// tensor core's order, so results differ from the CUDA-core kernel's in the
// last bits.
constexpr int TG_M = 128;                              // rows per tile
constexpr int TG_KC = 16;                              // K per chunk
constexpr int TG_A_HALF = TG_M * TG_KC * 4;            // A hi or lo of a chunk, 8 KB
constexpr int TG_B_HALF = 256 * TG_KC * 4;             // B hi or lo of a chunk (N <= 256), 16 KB
constexpr int TG_STAGE = 2 * TG_A_HALF + 2 * TG_B_HALF;
constexpr int TG_WORKERS = 256;                         // the weight gradient's staging threads
constexpr int TG_THREADS = TG_WORKERS + 32;             // + its issuer warp
// Named barrier 1 over the worker threads; the second form returns whether any passed true.
__device__ __forceinline__ void workers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(TG_WORKERS) : "memory");
}
__device__ __forceinline__ bool __syncthreads_or_workers(bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
               "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((uint32_t)v), "n"(TG_WORKERS) : "memory");
  return r != 0;
}

// Byte offset of element (r, k) of an R-row operand chunk, K-major core matrices
// (8 rows x 16 bytes: 4 tf32 elements of K per row).
__device__ __forceinline__ uint32_t tg_off(int r, int k, int R) {
  return (uint32_t)((k >> 2) * (R * 16) + (r >> 3) * 128 + (r & 7) * 16 + (k & 3) * 4);
}
__device__ __forceinline__ void tg_split(float v, float& hi, float& lo) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(v));
  hi = __uint_as_float(h);
  lo = __fsub_rn(v, hi);
}

// B[k][c] (k < K, c < N) -> chunks of 32 K: [chunk][hi | lo][N rows x 32 K].
__global__ void split_b_kernel(const float* __restrict__ B, int64_t ldb, int K, int N,
                               float* __restrict__ out) {
  const int64_t total = (int64_t)K * N;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int k = (int)(q / N), c = (int)(q % N);
    float hi, lo;
    tg_split(__ldg(B + (int64_t)k * ldb + c), hi, lo);
    float* ch = out + (int64_t)(k / TG_KC) * 2 * N * TG_KC;
    const uint32_t o = tg_off(c, k % TG_KC, N) >> 2;
    ch[o] = hi;
    ch[N * TG_KC + o] = lo;
  }
}

__device__ __forceinline__ void tg_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}

// Roles of the row GEMM's CTA (16 warps):
//   warps 0-3    epilogue: warp w reads TMEM lane quarter w (one accumulator row
//                per lane), 32 columns at a time, finishes the values in
//                registers and writes the 32 x 32 block to one of its two
//                shared-memory tiles (128-byte swizzle: conflict-free), which
//                lane 0 stores with one 2-D tensor copy: a store instruction
//                costs about 64 cycles of the SM's store path whatever its
//                width (measured), so the block leaves in one request instead
//                of eight uncoalesced or thirty-two coalesced ones;
//   warps 4-11   split the raw A rows into the operand stages;
//   warp 12      issues the MMAs: one barrier wait per chunk, six MMAs, a commit;
//   warp 13      streams the raw A rows by 2-D tensor copies (16 K-columns x
//                128 rows per chunk) into a 4-slot ring;
//   warps 14-15  copy the split weights of the even / odd chunks (one bulk copy
//                each; a copy takes the issuing thread about 600 cycles, so two
//                threads share the chunk stream).
// The operand stages are triple-buffered; a stage is full when the eight
// staging warps and the weight copy have arrived. The accumulator is double-
// buffered in tensor memory (2 N columns), so a tile's epilogue overlaps the
// next tile's MMAs.
constexpr int RG_EPI = 128;
constexpr int RG_STG = 256;
constexpr int RG_THREADS = RG_EPI + RG_STG + 128;
constexpr int RG_NSTAGE = 3;
constexpr int RG_RAW = TG_M * TG_KC * 4;                // one raw A chunk, 8 KB
constexpr int RG_NRAW = 4;
constexpr int RG_OUTB = 32 * 32 * 4;                    // an epilogue warp's 32 x 32 output block
constexpr int RG_OUT = RG_NSTAGE * TG_STAGE + RG_NRAW * RG_RAW;   // 4 warps x 2 blocks, 1024-aligned
constexpr int RG_BAR = RG_OUT + 4 * 2 * RG_OUTB;
constexpr size_t RG_SMEM = (size_t)RG_BAR + 256;

template <int N>
__global__ void __launch_bounds__(RG_THREADS, 1) row_gemm_tc_kernel(RowGemm g,
                                                                    const __grid_constant__ CUtensorMap amap,
                                                                    const __grid_constant__ CUtensorMap omap) {
  unsigned* flag = g.flag;
  extern __shared__ __align__(1024) uint8_t tsm[];
  uint64_t* done = reinterpret_cast<uint64_t*>(tsm + RG_BAR);   // [3] MMAs of a stage done
  uint64_t* full = done + RG_NSTAGE;                             // [3] stage staged (A and B)
  uint64_t* accf = full + RG_NSTAGE;                             // [2] accumulator ready
  uint64_t* acce = accf + 2;                                     // [2] accumulator read out
  uint64_t* rfull = acce + 2;                                    // [4] raw A chunk landed
  uint64_t* rempty = rfull + RG_NRAW;                            // [4] raw A chunk read
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(rempty + RG_NRAW);
  __shared__ int abort_s;
  __shared__ __align__(16) float s_bias[N], s_ev[N];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = tcx::smem_u32(tsm);
  const uint32_t rawbase = sbase + RG_NSTAGE * TG_STAGE;
  constexpr uint64_t kLimit = 2000000000ull;
  if (tid == 0) {
    for (int i = 0; i < RG_NSTAGE; ++i) {
      tcx::mbar_init(&done[i], 1);
      tcx::mbar_init(&full[i], RG_STG / 32 + 1);   // the staging warps and the weight copy
    }
    for (int i = 0; i < 2; ++i) {
      tcx::mbar_init(&accf[i], 1);
      tcx::mbar_init(&acce[i], RG_EPI / 32);       // one arrival per epilogue warp
    }
    for (int i = 0; i < RG_NRAW; ++i) {
      tcx::mbar_init(&rfull[i], 1);
      tcx::mbar_init(&rempty[i], RG_STG / 32);
    }
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < N; i += RG_THREADS) {
    s_bias[i] = g.bias ? g.bias[i] : 0.0f;
    s_ev[i] = g.ea ? g.ev[i] : 0.0f;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tcx::smem_u32(tmem_holder)), "r"(2 * N));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tcx::fence_before();
  __syncthreads();
  tcx::fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nch = g.K / TG_KC;
  const int64_t ntiles = (g.rows + TG_M - 1) / TG_M;
  // this CTA's tiles: blockIdx.x, + gridDim.x, ...; chunk G of the CTA is chunk
  // G % nch of its tile G / nch, uses operand stage G % 3 (barrier parity
  // (G / 3) % 2) and raw slot G % 4 (parity (G / 4) % 2); tile i uses
  // accumulator i % 2 (parity (i / 2) % 2)
  // the swizzled output tiles must sit on 1024-byte boundaries: otherwise no
  // role runs (the error flag says why) rather than stores of permuted tiles
  const int n_my = (blockIdx.x < ntiles && ((sbase + RG_OUT) & 1023u) == 0)
                       ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  if (tid == 0 && ((sbase + RG_OUT) & 1023u) != 0) atomicOr(flag, FLAG_BAD_INDEX);
  const int64_t total = (int64_t)n_my * nch;
  bool ok = true;
  constexpr int W_ISSUE = (RG_EPI + RG_STG) / 32, W_APROD = W_ISSUE + 1, W_BPROD = W_ISSUE + 2;
  if (warp == W_ISSUE) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
                                 ((uint32_t)(TG_M >> 4) << 24);   // f32 <- tf32 x tf32, M 128
      int64_t G = 0, issued = -1;
      for (int it = 0; it < n_my && ok; ++it) {
        const int b = it & 1;
        if (it >= 2 && !tcx::mbar_wait(&acce[b], (uint32_t)(((it >> 1) - 1) & 1), &abort_s, flag, kLimit)) {
          ok = false;
          break;
        }
        const uint32_t acc = tmem + (uint32_t)(b * N);
        for (int c = 0; c < nch; ++c, ++G) {
          const int stage = (int)(G % RG_NSTAGE);
          if (!tcx::mbar_wait(&full[stage], (uint32_t)((G / RG_NSTAGE) & 1), &abort_s, flag, kLimit)) {
            ok = false;
            break;
          }
          tcx::fence_after();
          const uint32_t sa = sbase + stage * TG_STAGE;
          const uint64_t ah = tcx::sdesc(sa, TG_M * 16, 128), al = tcx::sdesc(sa + TG_A_HALF, TG_M * 16, 128);
          const uint64_t bh = tcx::sdesc(sa + 2 * TG_A_HALF, N * 16, 128);
          const uint64_t bl = tcx::sdesc(sa + 2 * TG_A_HALF + N * TG_KC * 4, N * 16, 128);
#pragma unroll
          for (int s = 0; s < TG_KC / 8; ++s) {
            const uint64_t da = (uint64_t)((s * 2 * TG_M * 16) >> 4), db = (uint64_t)((s * 2 * N * 16) >> 4);
            tg_mma(acc, ah + da, bh + db, idesc, (c | s) != 0);
            tg_mma(acc, ah + da, bl + db, idesc, 1);
            tg_mma(acc, al + da, bh + db, idesc, 1);
          }
          tcx::mma_commit(&done[stage]);
          if (c == nch - 1) tcx::mma_commit(&accf[b]);
          issued = G;
        }
      }
      // the MMAs already issued land before TMEM is freed, abort or not
      if (issued >= 0)
        tcx::mbar_drain(&done[issued % RG_NSTAGE], (uint32_t)((issued / RG_NSTAGE) & 1), flag,
                        tcx::globaltimer(), kLimit);
    }
    __syncwarp();
  } else if (warp >= W_BPROD) {
    // ------------------------------------------------------------- weight copies
    // warp W_BPROD + q copies the weights of chunks G = q, q + 2, ... into stage
    // G % 3 once chunk G - 3's MMAs have read it
    if (lane == 0) {
      constexpr uint32_t bytes = 2 * N * TG_KC * 4;
      int64_t copied = -1;
      for (int64_t G = warp - W_BPROD; G < total; G += 2) {
        const int stage = (int)(G % RG_NSTAGE), c = (int)(G % nch);
        if (G >= RG_NSTAGE &&
            !tcx::mbar_wait(&done[stage], (uint32_t)((G / RG_NSTAGE - 1) & 1), &abort_s, flag, kLimit))
          break;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                     ::"r"(tcx::smem_u32(&full[stage])), "r"(bytes) : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
            ::"r"(sbase + stage * TG_STAGE + 2 * TG_A_HALF),
              "l"(g.bsplit + (int64_t)c * 2 * N * TG_KC), "r"(bytes),
              "r"(tcx::smem_u32(&full[stage]))
            : "memory");
        copied = G;
      }
      // the last copy lands before shared memory is given up: it has arrived on
      // full[] once that phase completes, or, after an abort, once its bytes did
      // (the staging warps may not have arrived); wait on the copy's bytes by
      // the phase, bounded either way
      const uint64_t t0 = tcx::globaltimer();
      bool landed = copied < 0;
      while (!landed && !abort_s) {
        landed = tcx::mbar_try(&full[copied % RG_NSTAGE], (uint32_t)((copied / RG_NSTAGE) & 1));
        if (!landed && tcx::globaltimer() - t0 > kLimit) {
          atomicOr(flag, FLAG_TIMEOUT);
          abort_s = 1;
        }
      }
      if (!landed) {
        const uint64_t t1 = tcx::globaltimer();
        while (tcx::globaltimer() - t1 < 20000) {   // an aborted launch: give the copy 20 us
        }
      }
    }
    __syncwarp();
  } else if (warp == W_APROD) {
    // ------------------------------------------------------------- raw A producer
    if (lane == 0) {
      int64_t loaded = -1;
      for (int64_t G = 0; G < total && ok; ++G) {
        const int slot = (int)(G % RG_NRAW);
        if (G >= RG_NRAW &&
            !tcx::mbar_wait(&rempty[slot], (uint32_t)((G / RG_NRAW - 1) & 1), &abort_s, flag, kLimit)) {
          ok = false;
          break;
        }
        const int64_t it = G / nch;
        const int c = (int)(G - it * nch);
        const int k = c * TG_KC;
        const int col = k < g.a_split ? g.a0 + k : g.a1 + k - g.a_split;
        const int row = (int)((blockIdx.x + it * gridDim.x) * TG_M);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                     ::"r"(tcx::smem_u32(&rfull[slot])), "r"(RG_RAW) : "memory");
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
            ::"r"(rawbase + slot * RG_RAW), "l"(reinterpret_cast<uint64_t>(&amap)), "r"(col), "r"(row),
              "r"(tcx::smem_u32(&rfull[slot]))
            : "memory");
        loaded = G;
      }
      // the copies in flight land before shared memory is given up
      const uint64_t t0 = tcx::globaltimer();
      for (int64_t q = loaded; q >= 0 && q > loaded - RG_NRAW; --q)
        if (!tcx::mbar_drain(&rfull[q % RG_NRAW], (uint32_t)((q / RG_NRAW) & 1), flag, t0, kLimit)) break;
    }
    __syncwarp();
  } else if (warp >= RG_EPI / 32) {
    // ------------------------------------------------------------- staging warps
    // per chunk, thread st reads the 16-byte pieces i = st and st + 256 of the
    // raw chunk (row i / 4, K columns 4 (i % 4) ..), so that a warp reads 512
    // contiguous bytes. A shuffle then hands lane l the piece of row
    // 8 (warp) + l % 8, K group l / 8: each quarter-warp (the unit in which
    // 16-byte shared accesses are served) stores one 128-byte core-matrix row
    // without bank conflicts. A warp that broke out on an abort never arrives
    // again, so the other roles' waits end by the abort word.
    const int st = tid - RG_EPI;
    const int src = ((lane & 7) << 2) | (lane >> 3);
    const int srow = 8 * (st >> 5) + (lane & 7), skq = lane >> 3;
    for (int64_t G = 0; G < total && ok; ++G) {
      const int slot = (int)(G % RG_NRAW), stage = (int)(G % RG_NSTAGE);
      bool w = tcx::mbar_wait(&rfull[slot], (uint32_t)((G / RG_NRAW) & 1), &abort_s, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      const float* raw = reinterpret_cast<const float*>(tsm + RG_NSTAGE * TG_STAGE + slot * RG_RAW);
      const float4 r0 = *reinterpret_cast<const float4*>(raw + 4 * st);
      const float4 r1 = *reinterpret_cast<const float4*>(raw + 4 * (st + 256));
      const float4 v0 = make_float4(__shfl_sync(0xffffffffu, r0.x, src), __shfl_sync(0xffffffffu, r0.y, src),
                                    __shfl_sync(0xffffffffu, r0.z, src), __shfl_sync(0xffffffffu, r0.w, src));
      const float4 v1 = make_float4(__shfl_sync(0xffffffffu, r1.x, src), __shfl_sync(0xffffffffu, r1.y, src),
                                    __shfl_sync(0xffffffffu, r1.z, src), __shfl_sync(0xffffffffu, r1.w, src));
      w = G < RG_NSTAGE || tcx::mbar_wait(&done[stage], (uint32_t)((G / RG_NSTAGE - 1) & 1), &abort_s, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      const uint32_t sa = sbase + stage * TG_STAGE;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 v = h ? v1 : v0;
        float hi[4], lo[4];
        tg_split(v.x, hi[0], lo[0]);
        tg_split(v.y, hi[1], lo[1]);
        tg_split(v.z, hi[2], lo[2]);
        tg_split(v.w, hi[3], lo[3]);
        const uint32_t o = tg_off(srow + 64 * h, 4 * skq, TG_M);
        tcx::st_shared_v4(sa + o, __float_as_uint(hi[0]), __float_as_uint(hi[1]),
                          __float_as_uint(hi[2]), __float_as_uint(hi[3]));
        tcx::st_shared_v4(sa + TG_A_HALF + o, __float_as_uint(lo[0]), __float_as_uint(lo[1]),
                          __float_as_uint(lo[2]), __float_as_uint(lo[3]));
      }
      tcx::fence_async_smem();
      __syncwarp();
      // the raw slot is released only now: every lane's stores above consumed
      // its loads of the slot, so the next tensor copy into it cannot overtake
      // a read still in flight
      if (lane == 0) {
        tcx::mbar_arrive(&full[stage]);
        tcx::mbar_arrive(&rempty[slot]);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue warps
    // thread = accumulator row warp * 32 + lane; 32 columns per TMEM load; the
    // next block's side input (the mask or the row biases: a launch has at most
    // one) is loaded while the current block is finished; chunk j (columns
    // 4j..4j+3) of row r sits at r * 128 + ((j ^ (r % 8)) * 16) in the tile,
    // the layout the tensor map's 128-byte swizzle reads
    const uint32_t obase = sbase + RG_OUT + warp * 2 * RG_OUTB;
    int nstore = 0;
    for (int it = 0; it < n_my && ok; ++it) {
      const int b = it & 1;
      const bool w = tcx::mbar_wait(&accf[b], (uint32_t)((it >> 1) & 1), &abort_s, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tcx::fence_after();
      const int64_t row0 = (blockIdx.x + (int64_t)it * gridDim.x) * TG_M + warp * 32;
      const int64_t row = row0 + lane;
      const bool live = row < g.rows;
      const float eav = (g.ea && live) ? g.ea[row * g.ldea] : 0.0f;
      const float* mrow = (g.mask && live) ? g.mask + row * g.ldm : nullptr;
      const float* rrow = (g.row_bias && live) ? g.row_bias + (row / g.rb_div) * g.n_out : nullptr;
      const float* srow = mrow ? mrow : rrow;
      float4 sd[8];
      auto load_side = [&](int cb, float4 (&m)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          m[j] = srow ? *reinterpret_cast<const float4*>(srow + cb + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
      };
      load_side(0, sd);
#pragma unroll 1
      for (int cb = 0; cb < N; cb += 32, ++nstore) {
        uint32_t u[32];
        tcx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * N + cb), u);
        float4 sd2[8];
        if (cb + 32 < N) load_side(cb + 32, sd2);
        // the tile written two blocks ago has been read by its store
        if (lane == 0 && nstore >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
        const uint32_t ob = obase + (uint32_t)(nstore & 1) * RG_OUTB + (uint32_t)lane * 128;
        tcx::tmem_ld_wait(u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 bv = *reinterpret_cast<const float4*>(s_bias + cb + 4 * j);
          const float4 ev = *reinterpret_cast<const float4*>(s_ev + cb + 4 * j);
          float x[4] = {__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                        __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3])};
          const float bb[4] = {bv.x, bv.y, bv.z, bv.w}, ee[4] = {ev.x, ev.y, ev.z, ev.w};
          const float sv[4] = {sd[j].x, sd[j].y, sd[j].z, sd[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v = x[e];
            if (g.bias) v += bb[e];
            if (g.row_bias) v += sv[e];
            if (g.ea) v = fmaf(eav, ee[e], v);
            if (g.relu) v = fmaxf(v, 0.0f);
            if (g.mask) v = sv[e] > 0.0f ? v : 0.0f;
            x[e] = v;
          }
          tcx::st_shared_v4(ob + (uint32_t)((j ^ (lane & 7)) * 16), __float_as_uint(x[0]),
                            __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
        }
        tcx::fence_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < g.rows) {
          // rows past the end of the matrix are clipped by the tensor map
          asm volatile(
              "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
              ::"l"(reinterpret_cast<uint64_t>(&omap)), "r"(cb), "r"((int)row0),
                "r"(obase + (uint32_t)(nstore & 1) * RG_OUTB)
              : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (cb + 32 < N) {
#pragma unroll
          for (int j = 0; j < 8; ++j) sd[j] = sd2[j];
        }
      }
      // this warp's rows of the accumulator are read out
      tcx::fence_before();
      __syncwarp();
      if (lane == 0) tcx::mbar_arrive(&acce[b]);
    }
    // every store has read its tile before the CTA gives up shared memory, and
    // has written global memory before the kernel ends
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }
  tcx::fence_before();
  __syncthreads();
  if (warp == 0) {
    tcx::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * N));
  }
}

// ---------------------------------------------------------------------------
// The same row GEMM on CTA pairs: a cluster of two CTAs on two SMs runs
// tcgen05.mma.cta_group::2 (M = 256: rows [0, 128) of a 256-row tile in CTA 0,
// [128, 256) in CTA 1). Each CTA stages its own 128 A rows and holds half of
// the split weights (N / 2 rows of B), and CTA 0 issues the MMAs for both, so
// per MMA each SM reads 4 KB of A and 4 KB of B from its shared memory instead
// of 4 + 8 KB, each CTA copies half the weights, and one MMA instruction does
// the work of two. The halved weight stages make room for 32-K chunks in two
// 64 KB stages (twelve MMAs per barrier wait and commit); the raw A chunks
// arrive under the 128-byte swizzle, read conflict-free by the staging warps.
// The roles per CTA are the single-CTA kernel's; a stage is full on CTA 0's
// barrier when the sixteen staging warps of both CTAs and the two weight
// copies (counted by CTA 0's expect) have arrived, an accumulator is free on
// CTA 0's barrier when the eight epilogue warps of both CTAs have read it, and
// the commits arrive on both CTAs.
constexpr int RP_KC = 32;                                          // K per chunk
constexpr int RP_A_HALF = TG_M * RP_KC * 4;                        // A hi or lo of a chunk: 16 KB
constexpr int RP_NSTAGE = 2;
constexpr int RP_STAGE = 2 * RP_A_HALF + 2 * (128 * RP_KC * 4);    // A hi, lo; B half hi, lo: 64 KB
constexpr int RP_RAW = TG_M * RP_KC * 4;                           // one raw A chunk, 16 KB
constexpr int RP_NRAW = 4;
constexpr int RP_OUT = RP_NSTAGE * RP_STAGE + RP_NRAW * RP_RAW;    // 1024-aligned
constexpr int RP_VEC = RP_OUT + 4 * 2 * RG_OUTB;
constexpr int RP_BAR = RP_VEC + 2 * 256 * 4;
constexpr size_t RP_SMEM = (size_t)RP_BAR + 256;

__device__ __forceinline__ uint32_t rp_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t rp_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t rp_nclusters() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void rp_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// try_wait with cluster-scope acquire: the phase may be completed from the peer CTA
__device__ __forceinline__ bool rp_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(tcx::smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded, as tcx::mbar_wait
__device__ __forceinline__ bool rp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                        unsigned* flag, uint64_t limit_ns) {
  if (rp_try(bar, parity)) return true;
  const uint64_t t0 = tcx::globaltimer();
  while (!rp_try(bar, parity)) {
    if (*abort) return false;
    if (tcx::globaltimer() - t0 > limit_ns) {
      atomicOr(flag, FLAG_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
  return true;
}
// Arrive on CTA 0's barrier at this barrier's offset, releasing this CTA's
// shared-memory writes at cluster scope (a release fence restricted to
// shared::cta operations, then a relaxed remote arrive).
__device__ __forceinline__ void rp_arrive_cta0(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, 0;\n\t"
      "fence.release.sync_restrict::shared::cta.cluster;\n\t"
      "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}"
      ::"r"(tcx::smem_u32(bar))
      : "memory");
}
// 2-D tensor load into this CTA's shared memory counted on CTA 0's barrier
// (the barrier's shared address with the peer bit cleared); no multicast.
__device__ __forceinline__ void rp_load_pair(uint32_t dst, const void* tmap, int x, int y,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tmap)),
        "r"(tcx::smem_u32(bar) & 0xFEFFFFFFu), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void rp_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
// arrive (once each) on this barrier's offset in both CTAs once every MMA
// issued so far by the calling thread has completed
__device__ __forceinline__ void rp_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;"
      ::"r"(tcx::smem_u32(bar)), "h"((uint16_t)3)
      : "memory");
}

// B[k][c] -> chunks of RP_KC K, each [half h][hi | lo][N/2 rows x RP_KC K] (K-major
// core matrices of N/2 rows): the half a CTA of the pair holds is one contiguous run.
__global__ void split_b_pair_kernel(const float* __restrict__ B, int64_t ldb, int K, int N,
                                    float* __restrict__ out) {
  const int64_t total = (int64_t)K * N;
  const int Nh = N / 2;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int k = (int)(q / N), c = (int)(q % N);
    const int h = c / Nh, cl = c - h * Nh;
    float hi, lo;
    tg_split(__ldg(B + (int64_t)k * ldb + c), hi, lo);
    float* ch = out + (int64_t)(k / RP_KC) * 2 * N * RP_KC + (int64_t)h * N * RP_KC;
    const uint32_t o = tg_off(cl, k % RP_KC, Nh) >> 2;
    ch[o] = hi;
    ch[Nh * RP_KC + o] = lo;
  }
}

template <int N>
__global__ void __launch_bounds__(RG_THREADS, 1) row_gemm_pair_kernel(RowGemm g,
                                                                      const __grid_constant__ CUtensorMap amap,
                                                                      const __grid_constant__ CUtensorMap bmap,
                                                                      const __grid_constant__ CUtensorMap omap) {
  constexpr int Nh = N / 2;
  constexpr uint32_t BH = Nh * RP_KC * 4;        // B half, hi or lo, of a chunk
  unsigned* flag = g.flag;
  extern __shared__ __align__(1024) uint8_t tsm[];
  float* s_bias = reinterpret_cast<float*>(tsm + RP_VEC);
  float* s_ev = s_bias + 256;
  uint64_t* done = reinterpret_cast<uint64_t*>(tsm + RP_BAR);   // [4] MMAs of a stage done (both CTAs)
  uint64_t* full = done + RP_NSTAGE;                             // [4] stage staged (CTA 0's)
  uint64_t* accf = full + RP_NSTAGE;                             // [2] accumulator ready (both CTAs)
  uint64_t* acce = accf + 2;                                     // [2] accumulator read out (CTA 0's)
  uint64_t* rfull = acce + 2;                                    // [4] raw A chunk landed
  uint64_t* rempty = rfull + RP_NRAW;                            // [4] raw A chunk read
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(rempty + RP_NRAW);
  volatile int* abort_p = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = (int)rp_rank();
  const uint32_t sbase = tcx::smem_u32(tsm);
  const uint32_t rawbase = sbase + RP_NSTAGE * RP_STAGE;
  constexpr uint64_t kLimit = 2000000000ull;
  if (tid == 0) {
    for (int i = 0; i < RP_NSTAGE; ++i) {
      tcx::mbar_init(&done[i], 1);
      tcx::mbar_init(&full[i], 2 * (RG_STG / 32) + 1);   // both CTAs' staging warps, CTA 0's expect
    }
    for (int i = 0; i < 2; ++i) {
      tcx::mbar_init(&accf[i], 1);
      tcx::mbar_init(&acce[i], 2 * (RG_EPI / 32));       // both CTAs' epilogue warps
    }
    for (int i = 0; i < RP_NRAW; ++i) {
      tcx::mbar_init(&rfull[i], 1);
      tcx::mbar_init(&rempty[i], RG_STG / 32);
    }
    *abort_p = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < N; i += RG_THREADS) {
    s_bias[i] = g.bias ? g.bias[i] : 0.0f;
    s_ev[i] = g.ea ? g.ev[i] : 0.0f;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tcx::smem_u32(tmem_holder)), "r"(2 * N));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tcx::fence_before();
  __syncthreads();
  rp_cluster_sync();            // both CTAs' barriers exist before any remote use
  tcx::fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nch = g.K / RP_KC;
  const int64_t ntiles = (g.rows + 2 * TG_M - 1) / (2 * TG_M);   // 256-row pair tiles
  const int64_t cid = rp_cluster(), ncl = rp_nclusters();
  // pair tile i = cid + i * ncl; chunk G of the pair is chunk G % nch of its
  // tile G / nch and uses stage G % 2 (parity (G / 2) % 2) and raw slot G % 4;
  // tile i uses accumulator i % 2 (parity (i / 2) % 2). Both CTAs lay out
  // shared memory alike, so the alignment test agrees between them.
  const bool aligned = ((sbase + RP_OUT) & 1023u) == 0;
  const int n_my = (cid < ntiles && aligned) ? (int)((ntiles - 1 - cid) / ncl + 1) : 0;
  if (tid == 0 && !aligned) atomicOr(flag, FLAG_BAD_INDEX);
  const int64_t total = (int64_t)n_my * nch;
  auto tile_row = [&](int64_t it) { return (cid + it * ncl) * (2 * TG_M) + rank * TG_M; };
  bool ok = true;
  constexpr int W_ISSUE = (RG_EPI + RG_STG) / 32, W_APROD = W_ISSUE + 1, W_BPROD = W_ISSUE + 2;
  if (warp == W_ISSUE) {
    // ------------------------------------------------------------- MMA issuer (CTA 0)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
                                 ((uint32_t)((2 * TG_M) >> 4) << 24);   // f32 <- tf32 x tf32, M 256
      int64_t G = 0, issued = -1;
      for (int it = 0; it < n_my && ok; ++it) {
        const int b = it & 1;
        if (it >= 2 && !rp_wait(&acce[b], (uint32_t)(((it >> 1) - 1) & 1), abort_p, flag, kLimit)) {
          ok = false;
          break;
        }
        const uint32_t acc = tmem + (uint32_t)(b * N);
        for (int c = 0; c < nch; ++c, ++G) {
          const int stage = (int)(G % RP_NSTAGE);
          if (!rp_wait(&full[stage], (uint32_t)((G / RP_NSTAGE) & 1), abort_p, flag, kLimit)) {
            ok = false;
            break;
          }
          tcx::fence_after();
          const uint32_t sa = sbase + stage * RP_STAGE;
          const uint64_t ah = tcx::sdesc(sa, TG_M * 16, 128), al = tcx::sdesc(sa + RP_A_HALF, TG_M * 16, 128);
          const uint64_t bh = tcx::sdesc(sa + 2 * RP_A_HALF, Nh * 16, 128);
          const uint64_t bl = tcx::sdesc(sa + 2 * RP_A_HALF + BH, Nh * 16, 128);
#pragma unroll
          for (int s = 0; s < RP_KC / 8; ++s) {
            const uint64_t da = (uint64_t)((s * 2 * TG_M * 16) >> 4), db = (uint64_t)((s * 2 * Nh * 16) >> 4);
            rp_mma(acc, ah + da, bh + db, idesc, (c | s) != 0);
            rp_mma(acc, ah + da, bl + db, idesc, 1);
            rp_mma(acc, al + da, bh + db, idesc, 1);
          }
          rp_commit(&done[stage]);
          if (c == nch - 1) rp_commit(&accf[b]);
          issued = G;
        }
      }
      // the MMAs already issued land before either CTA frees its memory, abort or not
      if (issued >= 0) {
        const uint64_t t0 = tcx::globaltimer();
        while (!rp_try(&done[issued % RP_NSTAGE], (uint32_t)((issued / RP_NSTAGE) & 1))) {
          if (tcx::globaltimer() - t0 > kLimit) {
            atomicOr(flag, FLAG_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= W_BPROD) {
    // ------------------------------------------------------------- weight copies
    // warp W_BPROD + q of each CTA copies that CTA's half of the weights of
    // chunks G = q, q + 2, ... into stage G % 2 once chunk G - 2's MMAs are done;
    // CTA 0 expects both halves' bytes on its full[] barrier
    if (lane == 0) {
      constexpr uint32_t half_bytes = 2 * BH;
      for (int64_t G = warp - W_BPROD; G < total; G += 2) {
        const int stage = (int)(G % RP_NSTAGE), c = (int)(G % nch);
        if (G >= RP_NSTAGE &&
            !rp_wait(&done[stage], (uint32_t)((G / RP_NSTAGE - 1) & 1), abort_p, flag, kLimit))
          break;
        if (rank == 0)
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                       ::"r"(tcx::smem_u32(&full[stage])), "r"(2 * half_bytes) : "memory");
        rp_load_pair(sbase + stage * RP_STAGE + 2 * RP_A_HALF, &bmap, 0, (2 * c + rank) * (2 * BH / 128),
                     &full[stage]);
      }
      // every copy lands before the final cluster barrier: the issuer waits
      // for each stage it consumes, and an aborted launch pauses before it
    }
    __syncwarp();
  } else if (warp == W_APROD) {
    // ------------------------------------------------------------- raw A producer
    if (lane == 0) {
      int64_t loaded = -1;
      for (int64_t G = 0; G < total && ok; ++G) {
        const int slot = (int)(G % RP_NRAW);
        if (G >= RP_NRAW &&
            !tcx::mbar_wait(&rempty[slot], (uint32_t)((G / RP_NRAW - 1) & 1), abort_p, flag, kLimit)) {
          ok = false;
          break;
        }
        const int64_t it = G / nch;
        const int c = (int)(G - it * nch);
        const int k = c * RP_KC;
        const int col = k < g.a_split ? g.a0 + k : g.a1 + k - g.a_split;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                     ::"r"(tcx::smem_u32(&rfull[slot])), "r"(RP_RAW) : "memory");
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
            ::"r"(rawbase + slot * RP_RAW), "l"(reinterpret_cast<uint64_t>(&amap)), "r"(col),
              "r"((int)tile_row(it)), "r"(tcx::smem_u32(&rfull[slot]))
            : "memory");
        loaded = G;
      }
      const uint64_t t0 = tcx::globaltimer();
      for (int64_t q = loaded; q >= 0 && q > loaded - RP_NRAW; --q)
        if (!tcx::mbar_drain(&rfull[q % RP_NRAW], (uint32_t)((q / RP_NRAW) & 1), flag, t0, kLimit)) break;
    }
    __syncwarp();
  } else if (warp >= RG_EPI / 32) {
    // ------------------------------------------------------------- staging warps
    // thread st owns row st % 128 of the chunk and its K groups kq = st / 128,
    // + 2, + 4, + 6 (four K columns each). The raw chunk arrives by a tensor copy
    // with the 128-byte swizzle (group kq of row r at 16 ((kq ^ (r % 8))) in the
    // row's 128 bytes), so a quarter-warp (eight consecutive rows, one group)
    // reads and writes without bank conflicts.
    const int st = tid - RG_EPI;
    const int arow = st & (TG_M - 1), kq0 = st >> 7;
    for (int64_t G = 0; G < total && ok; ++G) {
      const int slot = (int)(G % RP_NRAW), stage = (int)(G % RP_NSTAGE);
      bool w = tcx::mbar_wait(&rfull[slot], (uint32_t)((G / RP_NRAW) & 1), abort_p, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      const uint8_t* raw = tsm + RP_NSTAGE * RP_STAGE + slot * RP_RAW + arow * 128;
      float4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        v[j] = *reinterpret_cast<const float4*>(raw + (((kq0 + 2 * j) ^ (arow & 7)) * 16));
      w = G < RP_NSTAGE || rp_wait(&done[stage], (uint32_t)((G / RP_NSTAGE - 1) & 1), abort_p, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      const uint32_t sa = sbase + stage * RP_STAGE;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float hi[4], lo[4];
        tg_split(v[j].x, hi[0], lo[0]);
        tg_split(v[j].y, hi[1], lo[1]);
        tg_split(v[j].z, hi[2], lo[2]);
        tg_split(v[j].w, hi[3], lo[3]);
        const uint32_t o = tg_off(arow, 4 * (kq0 + 2 * j), TG_M);
        tcx::st_shared_v4(sa + o, __float_as_uint(hi[0]), __float_as_uint(hi[1]),
                          __float_as_uint(hi[2]), __float_as_uint(hi[3]));
        tcx::st_shared_v4(sa + RP_A_HALF + o, __float_as_uint(lo[0]), __float_as_uint(lo[1]),
                          __float_as_uint(lo[2]), __float_as_uint(lo[3]));
      }
      tcx::fence_async_smem();
      __syncwarp();
      // the raw slot is released only after the stores that consumed its loads
      if (lane == 0) {
        rp_arrive_cta0(&full[stage]);
        tcx::mbar_arrive(&rempty[slot]);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue warps
    const uint32_t obase = sbase + RP_OUT + warp * 2 * RG_OUTB;
    int nstore = 0;
    for (int it = 0; it < n_my && ok; ++it) {
      const int b = it & 1;
      const bool w = rp_wait(&accf[b], (uint32_t)((it >> 1) & 1), abort_p, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tcx::fence_after();
      const int64_t row0 = tile_row(it) + warp * 32;
      const int64_t row = row0 + lane;
      const bool live = row < g.rows;
      const float eav = (g.ea && live) ? g.ea[row * g.ldea] : 0.0f;
      const float* mrow = (g.mask && live) ? g.mask + row * g.ldm : nullptr;
      const float* rrow = (g.row_bias && live) ? g.row_bias + (row / g.rb_div) * g.n_out : nullptr;
      const float* srow = mrow ? mrow : rrow;
      float4 sd[8];
      auto load_side = [&](int cb, float4 (&m)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          m[j] = srow ? *reinterpret_cast<const float4*>(srow + cb + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
      };
      load_side(0, sd);
#pragma unroll 1
      for (int cb = 0; cb < N; cb += 32, ++nstore) {
        uint32_t u[32];
        tcx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * N + cb), u);
        float4 sd2[8];
        if (cb + 32 < N) load_side(cb + 32, sd2);
        if (lane == 0 && nstore >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
        const uint32_t ob = obase + (uint32_t)(nstore & 1) * RG_OUTB + (uint32_t)lane * 128;
        tcx::tmem_ld_wait(u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 bv = *reinterpret_cast<const float4*>(s_bias + cb + 4 * j);
          const float4 ev = *reinterpret_cast<const float4*>(s_ev + cb + 4 * j);
          float x[4] = {__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                        __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3])};
          const float bb[4] = {bv.x, bv.y, bv.z, bv.w}, ee[4] = {ev.x, ev.y, ev.z, ev.w};
          const float sv[4] = {sd[j].x, sd[j].y, sd[j].z, sd[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v = x[e];
            if (g.bias) v += bb[e];
            if (g.row_bias) v += sv[e];
            if (g.ea) v = fmaf(eav, ee[e], v);
            if (g.relu) v = fmaxf(v, 0.0f);
            if (g.mask) v = sv[e] > 0.0f ? v : 0.0f;
            x[e] = v;
          }
          tcx::st_shared_v4(ob + (uint32_t)((j ^ (lane & 7)) * 16), __float_as_uint(x[0]),
                            __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
        }
        tcx::fence_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < g.rows) {
          asm volatile(
              "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
              ::"l"(reinterpret_cast<uint64_t>(&omap)), "r"(cb), "r"((int)row0),
                "r"(obase + (uint32_t)(nstore & 1) * RG_OUTB)
              : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (cb + 32 < N) {
#pragma unroll
          for (int j = 0; j < 8; ++j) sd[j] = sd2[j];
        }
      }
      // this warp's rows of the accumulator are read out: tell CTA 0's issuer
      tcx::fence_before();
      __syncwarp();
      if (lane == 0) rp_arrive_cta0(&acce[b]);
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }
  tcx::fence_before();
  __syncthreads();
  if (tid == 0 && *abort_p) {   // an aborted launch: copies still in flight land first
    const uint64_t t1 = tcx::globaltimer();
    while (tcx::globaltimer() - t1 < 50000) {
    }
  }
  __syncthreads();
  rp_cluster_sync();            // the peer's MMAs, copies and arrivals into this CTA are over
  if (warp == 0) {
    tcx::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * N));
  }
}

// G[n][k] += sum_r A[r * lda + n] X(r, k) for n < N, k < K, rows in slices of
// `slice` (a multiple of 8), each slice's partial sums added atomically; the
// CTAs of the first column tile also add db[n] += sum_r A[r][n]. X(r, k) =
// X[r * ldx + x0 + k] for k < x_split, X[r * ldx + x1 + k - x_split] otherwise.
struct WGrad {
  const float* A; int64_t lda; int N;
  const float* X; int64_t ldx; int x0, x_split, x1; int K;
  int64_t rows, slice;
  float* G; int64_t ldg; float* db;
  int a_vec, x_vec;   // x_vec: X, ldx, x0, x1 and x_split all 16-byte / 4-float aligned
  unsigned* flag;     // the context's error word; set: the tensor-core kernel may run
};

template <bool XV>   // X rows 16-byte aligned and the split a multiple of 4
__global__ void __launch_bounds__(256, 2) wgrad_gemm_kernel(WGrad g) {
  __shared__ __align__(16) GemmSmem sm;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int nb = blockIdx.x * GT, kb = blockIdx.y * GT;
  const int64_t rs = (int64_t)blockIdx.z * g.slice;
  const int64_t re = rs + g.slice < g.rows ? rs + g.slice : g.rows;
  const int fr = tid >> 5, fc = (tid & 31) * 4;          // fetch role: row, 4 columns
  const int an = nb + fc, xk = kb + fc;
  // with XV, a thread's four X columns lie in one of the two ranges
  const bool x_lo = xk < g.x_split;
  const int xcol = x_lo ? g.x0 + xk : g.x1 + xk - g.x_split;
  // this thread's fetch row, advanced by 8 rows per fetch (two fetches per step)
  int64_t fr_row = rs + fr;
  const float* pa = g.A + fr_row * g.lda + an;
  const float* px = g.X + fr_row * g.ldx;
  const bool a_ok0 = an < g.N, a_ok1 = an + 1 < g.N, a_ok2 = an + 2 < g.N, a_ok3 = an + 3 < g.N;
  auto fetch = [&](float4& va, float4& vx) {
    va = make_float4(0.f, 0.f, 0.f, 0.f);
    vx = va;
    if (fr_row < re) {
      va = load4(pa, g.a_vec, a_ok0, a_ok1, a_ok2, a_ok3);
      if (XV) {
        vx = load4(px + xcol, true, xk < g.K, xk + 1 < g.K, xk + 2 < g.K, xk + 3 < g.K);
      } else {
        float t[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = xk + e;
          t[e] = k < g.K ? __ldg(px + (k < g.x_split ? g.x0 + k : g.x1 + k - g.x_split)) : 0.f;
        }
        vx = make_float4(t[0], t[1], t[2], t[3]);
      }
    }
    fr_row += 8;
    pa += 8 * g.lda;
    px += 8 * g.ldx;
  };
  auto put = [&](int buf, int rh, float4 va, float4 vx) {
    *reinterpret_cast<float4*>(&sm.a[buf][rh + fr][fc]) = va;
    *reinterpret_cast<float4*>(&sm.b[buf][rh + fr][fc]) = vx;
  };
  const bool bias_cta = g.db != nullptr && blockIdx.y == 0;
  float bsum = 0.0f;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  float4 va0, vx0, va1, vx1;
  fetch(va0, vx0);
  fetch(va1, vx1);
  put(0, 0, va0, vx0);
  put(0, 8, va1, vx1);
  __syncthreads();
  const int steps = (int)((re - rs + GK - 1) / GK);
  for (int s = 0; s < steps; ++s) {
    const int cur = s & 1;
    const bool more = s + 1 < steps;
    if (more) { fetch(va0, vx0); fetch(va1, vx1); }
    gemm_step(sm.a[cur], sm.b[cur], acc, ty, tx);
    if (bias_cta && tid < GT) {
#pragma unroll
      for (int k = 0; k < GK; ++k) bsum += sm.a[cur][k][tid];
    }
    if (more) { put(cur ^ 1, 0, va0, vx0); put(cur ^ 1, 8, va1, vx1); }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = nb + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
    if (n >= g.N) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = kb + (j < 4 ? 4 * tx + j : 64 + 4 * tx + j - 4);
      if (k < g.K) atomicAdd(g.G + (int64_t)n * g.ldg + k, acc[i][j]);
    }
  }
  if (bias_cta && tid < GT && nb + tid < g.N) atomicAdd(g.db + nb + tid, bsum);
}

// The same weight gradient on the tensor cores, for N = 128 or 256 and one
// column tile [k0, k0 + nt) of X (nt a power of two, 32..256; columns past K
// are zero): G[n][k0 + k] += sum_r A[r][n] X(r, k0 + k), and, in the tile
// with k0 = 0, db[n] += sum_r A[r][n]. The sum runs over the rows, so the rows
// are the MMA's K: the CTAs take equal contiguous runs of 16-row chunks, the
// worker warps split both operands per chunk (tf32 hi + fp32 remainder, as in
// the row GEMM) into K-major core matrices, thread t owning column t of A and
// of X, and the issuer warp accumulates hi*hi + hi*lo + lo*hi for each 128-row
// half of n in tensor memory (M 128, N nt). At the end the CTA's partial tile
// goes through shared memory and is added to G with coalesced atomics.
constexpr int WT_KC = 16;                               // rows per chunk
constexpr int WT_NSTAGE = 3;
constexpr int WT_PART = 256 * WT_KC * 4;                // A hi, A lo, X hi or X lo of a chunk: 16 KB
constexpr int WT_STAGE = 4 * WT_PART;
constexpr size_t WT_SMEM = (size_t)WT_NSTAGE * WT_STAGE + 64;
static_assert(128 * 257 * 4 <= WT_NSTAGE * WT_STAGE, "the epilogue tile fits in the stages");

__global__ void __launch_bounds__(TG_THREADS, 1) wgrad_tc_kernel(WGrad g, int k0, int nt,
                                                                 unsigned* flag) {
  extern __shared__ __align__(1024) uint8_t wsm[];
  uint64_t* done = reinterpret_cast<uint64_t*>(wsm + WT_NSTAGE * WT_STAGE);   // [3] MMAs of a stage
  uint64_t* afull = done + WT_NSTAGE;                                          // [3] stage staged
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(afull + WT_NSTAGE);
  __shared__ int abort_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = tcx::smem_u32(wsm);
  const int mh = g.N >> 7;                                   // 128-row halves of n
  const uint32_t ncols = (uint32_t)(mh * nt);                // a power of two, 32..512
  constexpr uint64_t kLimit = 2000000000ull;
  if (tid == 0) {
    for (int i = 0; i < WT_NSTAGE; ++i) {
      tcx::mbar_init(&done[i], 1);
      tcx::mbar_init(&afull[i], TG_WORKERS / 32);
    }
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tcx::smem_u32(tmem_holder)), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tcx::fence_before();
  __syncthreads();
  tcx::fence_after();
  const uint32_t tmem = *tmem_holder;
  const int64_t total = (g.rows + WT_KC - 1) / WT_KC;
  const int64_t cb = (int64_t)blockIdx.x * total / gridDim.x;
  const int nch = (int)((int64_t)(blockIdx.x + 1) * total / gridDim.x - cb);
  bool ok = true;
  if (warp == TG_WORKERS / 32) {
    // ------------------------------------------------------------- issuer warp
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(nt >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);   // f32 <- tf32 x tf32, M 128, N nt
      int issued = -1;
      for (int c = 0; c < nch; ++c) {
        const int s = c % WT_NSTAGE;
        if (!tcx::mbar_wait(&afull[s], (uint32_t)((c / WT_NSTAGE) & 1), &abort_s, flag, kLimit)) break;
        tcx::fence_after();
        const uint32_t sa = sbase + s * WT_STAGE;
        const uint64_t xh = tcx::sdesc(sa + 2 * WT_PART, nt * 16, 128);
        const uint64_t xl = tcx::sdesc(sa + 3 * WT_PART, nt * 16, 128);
        for (int h = 0; h < mh; ++h) {
          const uint64_t ah = tcx::sdesc(sa + h * (128 * WT_KC * 4), 128 * 16, 128);
          const uint64_t al = tcx::sdesc(sa + WT_PART + h * (128 * WT_KC * 4), 128 * 16, 128);
          const uint32_t d = tmem + (uint32_t)(h * nt);
#pragma unroll
          for (int ks = 0; ks < WT_KC / 8; ++ks) {
            const uint64_t da = (uint64_t)((ks * 2 * 128 * 16) >> 4);
            const uint64_t dx = (uint64_t)((ks * 2 * nt * 16) >> 4);
            tg_mma(d, ah + da, xh + dx, idesc, (c | ks) != 0);
            tg_mma(d, ah + da, xl + dx, idesc, 1);
            tg_mma(d, al + da, xh + dx, idesc, 1);
          }
        }
        tcx::mma_commit(&done[s]);
        issued = c;
      }
      // the MMAs already issued land before TMEM is freed, abort or not
      if (issued >= 0)
        tcx::mbar_drain(&done[issued % WT_NSTAGE], (uint32_t)((issued / WT_NSTAGE) & 1), flag,
                        tcx::globaltimer(), kLimit);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- workers
    const bool a_on = tid < g.N;
    const int kx = k0 + tid;
    const bool x_on = tid < nt && kx < g.K;
    const int64_t xcol = kx < g.x_split ? g.x0 + kx : g.x1 + kx - g.x_split;
    const int ah_ = tid >> 7, am = tid & 127;
    float dbs = 0.0f;
    auto fetch = [&](int c, float (&va)[WT_KC], float (&vx)[WT_KC]) {
      const int64_t r0 = (cb + c) * WT_KC;
#pragma unroll
      for (int i = 0; i < WT_KC; ++i) {
        const int64_t r = r0 + i;
        const bool live = c < nch && r < g.rows;
        va[i] = (live && a_on) ? __ldg(g.A + r * g.lda + tid) : 0.0f;
        vx[i] = (live && x_on) ? __ldg(g.X + r * g.ldx + xcol) : 0.0f;
      }
    };
    auto put = [&](int s, const float (&va)[WT_KC], const float (&vx)[WT_KC]) {
      const uint32_t sa = sbase + s * WT_STAGE;
      if (a_on) {
        const uint32_t base = sa + ah_ * (128 * WT_KC * 4);
#pragma unroll
        for (int q = 0; q < WT_KC / 4; ++q) {
          float hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tg_split(va[4 * q + j], hi[j], lo[j]);
            dbs += va[4 * q + j];
          }
          const uint32_t o = tg_off(am, 4 * q, 128);
          tcx::st_shared_v4(base + o, __float_as_uint(hi[0]), __float_as_uint(hi[1]),
                            __float_as_uint(hi[2]), __float_as_uint(hi[3]));
          tcx::st_shared_v4(base + WT_PART + o, __float_as_uint(lo[0]), __float_as_uint(lo[1]),
                            __float_as_uint(lo[2]), __float_as_uint(lo[3]));
        }
      }
      if (tid < nt) {
#pragma unroll
        for (int q = 0; q < WT_KC / 4; ++q) {
          float hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) tg_split(vx[4 * q + j], hi[j], lo[j]);
          const uint32_t o = tg_off(tid, 4 * q, nt);
          tcx::st_shared_v4(sa + 2 * WT_PART + o, __float_as_uint(hi[0]), __float_as_uint(hi[1]),
                            __float_as_uint(hi[2]), __float_as_uint(hi[3]));
          tcx::st_shared_v4(sa + 3 * WT_PART + o, __float_as_uint(lo[0]), __float_as_uint(lo[1]),
                            __float_as_uint(lo[2]), __float_as_uint(lo[3]));
        }
      }
    };
    // chunk c goes into stage c % 3 once chunk c - 3's MMAs are done; the rows
    // are fetched two chunks ahead into two alternating register sets
    auto stage_chunk = [&](int c, float (&va)[WT_KC], float (&vx)[WT_KC]) -> bool {
      const int s = c % WT_NSTAGE;
      const bool w = c < WT_NSTAGE ||
                     tcx::mbar_wait(&done[s], (uint32_t)((c / WT_NSTAGE - 1) & 1), &abort_s, flag, kLimit);
      if (!__all_sync(0xffffffffu, w)) return false;
      put(s, va, vx);
      tcx::fence_async_smem();
      __syncwarp();
      if (lane == 0) tcx::mbar_arrive(&afull[s]);
      fetch(c + 2, va, vx);
      return true;
    };
    float a0[WT_KC], x0[WT_KC], a1[WT_KC], x1[WT_KC];
    fetch(0, a0, x0);
    fetch(1, a1, x1);
    for (int c = 0; c < nch && ok; c += 2) {
      ok = stage_chunk(c, a0, x0);
      if (ok && c + 1 < nch) ok = stage_chunk(c + 1, a1, x1);
    }
    if (ok && nch > 0)
      ok = tcx::mbar_wait(&done[(nch - 1) % WT_NSTAGE], (uint32_t)(((nch - 1) / WT_NSTAGE) & 1),
                          &abort_s, flag, kLimit);
    ok = __all_sync(0xffffffffu, ok);
    tcx::fence_after();
    if (!__syncthreads_or_workers(!ok) && nch > 0) {
      // epilogue, one 128-row half of n at a time: TMEM -> tile [128][nt + 1]
      // (warp w reads lane quarter w % 4; warps w and w + 4 split the columns),
      // then thread t adds column t % nt of rows t / nt, + 256 / nt, ...
      float* tile = reinterpret_cast<float*>(wsm);
      const int ldt = nt + 1;
      const int q = warp & 3, nsplit = nt >= 64 ? 2 : 1, cw = nt / nsplit;
      for (int h = 0; h < mh; ++h) {
        if ((warp >> 2) < nsplit) {
          const int m = q * 32 + lane;
          for (int c0 = (warp >> 2) * cw; c0 < (warp >> 2) * cw + cw; c0 += 32) {
            uint32_t u[32];
            tcx::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * nt + c0), u);
            tcx::tmem_ld_wait(u);
#pragma unroll
            for (int j = 0; j < 32; ++j) tile[m * ldt + c0 + j] = __uint_as_float(u[j]);
          }
        }
        workers_sync();
        const int col = tid & (nt - 1), rstep = TG_WORKERS / nt;
        if (k0 + col < g.K) {
          float* gp = g.G + (int64_t)(h * 128) * g.ldg + k0 + col;
          for (int m = tid / nt; m < 128; m += rstep) atomicAdd(gp + (int64_t)m * g.ldg, tile[m * ldt + col]);
        }
        workers_sync();
      }
      if (k0 == 0 && g.db && a_on) atomicAdd(g.db + tid, dbs);
    }
  }
  tcx::fence_before();
  __syncthreads();
  if (warp == 0) {
    tcx::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
  }
}


// The weight gradient of a head with N <= 4 outputs (sigma: 1, rgb: 3): one
// thread per four input columns (the thread past the last one sums the bias),
// over a slice of rows, four rows in flight; the reads of X are 16-byte and
// coalesced across the threads. X rows and x0 are 4-float aligned, K % 4 == 0.
template <int NS>
__global__ void __launch_bounds__(128)
wgrad_head_kernel(const float* __restrict__ A, int64_t lda, const float* __restrict__ X,
                  int64_t ldx, int x0, int K, int64_t rows, int64_t slice, float* __restrict__ G,
                  int64_t ldg, float* __restrict__ db) {
  const int k = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (k > K) return;
  const bool bias = k == K;
  const int64_t rs = (int64_t)blockIdx.y * slice;
  const int64_t re = rs + slice < rows ? rs + slice : rows;
  float acc[NS][4];
#pragma unroll
  for (int n = 0; n < NS; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.0f;
  const float* px = X + x0 + k;
  int64_t r = rs;
  for (; r + 4 <= re; r += 4) {
    float4 x[4];
    float a[4][NS];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[u] = bias ? make_float4(1.f, 0.f, 0.f, 0.f)
                  : __ldg(reinterpret_cast<const float4*>(px + (r + u) * ldx));
#pragma unroll
      for (int n = 0; n < NS; ++n) a[u][n] = __ldg(A + (r + u) * lda + n);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int n = 0; n < NS; ++n) {
        acc[n][0] = fmaf(a[u][n], x[u].x, acc[n][0]);
        acc[n][1] = fmaf(a[u][n], x[u].y, acc[n][1]);
        acc[n][2] = fmaf(a[u][n], x[u].z, acc[n][2]);
        acc[n][3] = fmaf(a[u][n], x[u].w, acc[n][3]);
      }
  }
  for (; r < re; ++r) {
    const float4 x = bias ? make_float4(1.f, 0.f, 0.f, 0.f)
                          : __ldg(reinterpret_cast<const float4*>(px + r * ldx));
#pragma unroll
    for (int n = 0; n < NS; ++n) {
      const float a = __ldg(A + r * lda + n);
      acc[n][0] = fmaf(a, x.x, acc[n][0]);
      acc[n][1] = fmaf(a, x.y, acc[n][1]);
      acc[n][2] = fmaf(a, x.z, acc[n][2]);
      acc[n][3] = fmaf(a, x.w, acc[n][3]);
    }
  }
#pragma unroll
  for (int n = 0; n < NS; ++n) {
    if (bias) {
      atomicAdd(db + n, acc[n][0]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) atomicAdd(G + (int64_t)n * ldg + k + e, acc[n][e]);
    }
  }
}

// gamma(x) of every row into columns 0..63 of the activation store (the 64th
// is zero), x = o + t d with t from the sample source: the operations and
// rounding of the fused forward kernel's prologue.
__global__ void encode_store_kernel(const float* __restrict__ o, const float* __restrict__ d,
                                    int64_t R, SampleSpec ss, float* __restrict__ save,
                                    int64_t ldc, int64_t ray0) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= R * ss.S) return;
  float x[3];
  if (ss.mode == SAMPLES_GIVEN_X) {
    x[0] = ss.t[row * 3 + 0]; x[1] = ss.t[row * 3 + 1]; x[2] = ss.t[row * 3 + 2];
  } else {
    const int64_t ray = row / ss.S;
    const int s = (int)(row % ss.S);
    float t;
    if (ss.mode == SAMPLES_STRATIFIED) {
      const uint32_t m = ss.perturb ? draw_bits(ss.key, (uint64_t)(ray0 + ray), 0, (uint32_t)s) : 0u;
      t = stratified_t(ss.near, ss.step, s, m, ss.perturb != 0);
    } else {
      t = ss.t[row];
    }
#pragma unroll
    for (int c = 0; c < 3; ++c) x[c] = fadd(o[ray * 3 + c], fmul(t, d[ray * 3 + c]));
  }
  float v[64];
  v[0] = x[0]; v[1] = x[1]; v[2] = x[2]; v[63] = 0.0f;
#pragma unroll
  for (int c = 0; c < 3; ++c)
#pragma unroll
    for (int k = 0; k < 10; ++k) {
      float sn, cs;
      pe_sincos(x[c], k, &sn, &cs);
      v[3 + c * 10 + k] = sn;
      v[33 + c * 10 + k] = cs;
    }
  float* out = save + row * ldc;
#pragma unroll
  for (int q = 0; q < 16; ++q)
    *reinterpret_cast<float4*>(out + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2],
                                                          v[4 * q + 3]);
}

// raw[row] = (rgb, sigma): sigma = h_{D-1} . w_sigma + b_sigma, rgb_c = h_dir .
// W_rgb[c] + b_rgb[c] (no activation: the raw outputs). One warp per row.
__global__ void heads_fwd_kernel(const float* __restrict__ save, int64_t ldc, int hcol, int dcol,
                                 int W, const float* __restrict__ pk, PackedFp32 p, int64_t rows,
                                 float* __restrict__ raw) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* h = save + row * ldc + hcol;
  const float* hd = save + row * ldc + dcol;
  float sg = 0.f, c0 = 0.f, c1 = 0.f, c2 = 0.f;
  for (int k = 4 * lane; k < W; k += 128) {
    const float4 a = *reinterpret_cast<const float4*>(h + k);
    const float4 w = __ldg(reinterpret_cast<const float4*>(pk + p.sigma_w + k));
    sg = fmaf(a.x, w.x, sg); sg = fmaf(a.y, w.y, sg); sg = fmaf(a.z, w.z, sg); sg = fmaf(a.w, w.w, sg);
  }
  const int Wh = W / 2;
  for (int k = 4 * lane; k < Wh; k += 128) {
    const float4 a = *reinterpret_cast<const float4*>(hd + k);
    const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      c0 = fmaf(av[e], __ldg(pk + p.rgb_w + k + e), c0);
      c1 = fmaf(av[e], __ldg(pk + p.rgb_w + Wh + k + e), c1);
      c2 = fmaf(av[e], __ldg(pk + p.rgb_w + 2 * Wh + k + e), c2);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sg += __shfl_xor_sync(0xffffffffu, sg, off);
    c0 += __shfl_xor_sync(0xffffffffu, c0, off);
    c1 += __shfl_xor_sync(0xffffffffu, c1, off);
    c2 += __shfl_xor_sync(0xffffffffu, c2, off);
  }
  if (lane == 0)
    *reinterpret_cast<float4*>(raw + row * 4) =
        make_float4(c0 + __ldg(pk + p.rgb_b), c1 + __ldg(pk + p.rgb_b + 1),
                    c2 + __ldg(pk + p.rgb_b + 2), sg + __ldg(pk + p.sigma_b));
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

bool al16(const void* q) { return ((uintptr_t)q & 15u) == 0; }

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// fp32 matrix of `rows` rows of `ld` floats, boxes of TG_KC columns x TG_M rows
// (rows past the end read as zero).
EncodeTiledFn tiled_encoder() {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return nullptr;
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return encode;
}

cudaError_t encode_rows_map(CUtensorMap* m, const float* base, int64_t ld, int64_t rows) {
  EncodeTiledFn encode = tiled_encoder();
  if (!encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {TG_KC, TG_M};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// fp32 output matrix of `rows` rows of `ld` floats, `cols` of them written,
// boxes of 32 columns x 32 rows with the 128-byte swizzle (rows past the end
// are not written).
cudaError_t encode_out_map(CUtensorMap* m, float* base, int64_t ld, int cols, int64_t rows) {
  EncodeTiledFn encode = tiled_encoder();
  if (!encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The split weights as rows of 128 bytes; a box is one CTA's half of a chunk
// (N rows of 128 bytes: 32 KB for N = 256).
cudaError_t encode_bhalf_map(CUtensorMap* m, float* bsplit, int K, int N) {
  EncodeTiledFn encode = tiled_encoder();
  if (!encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {32, (cuuint64_t)K * N * 2 / 32};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {32, (cuuint32_t)(N * RP_KC / 32)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, bsplit, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The A rows for the pairs: boxes of RP_KC columns x TG_M rows, 128-byte swizzle.
cudaError_t encode_rows_map_sw(CUtensorMap* m, const float* base, int64_t ld, int64_t rows) {
  EncodeTiledFn encode = tiled_encoder();
  if (!encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {RP_KC, TG_M};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int N>
cudaError_t launch_row_gemm_pair(const RowGemm& g, const CUtensorMap& amap, const CUtensorMap& bmap,
                                 const CUtensorMap& omap, cudaStream_t st) {
  static int max_clusters = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(RG_THREADS);
  cfg.dynamicSmemBytes = RP_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_clusters <= 0) {
    cudaError_t e = cudaFuncSetAttribute(row_gemm_pair_kernel<N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RP_SMEM);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)sm_count() & ~1u);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, row_gemm_pair_kernel<N>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = sm_count() / 2;
    }
    max_clusters = n;
  }
  const int64_t pairs = (g.rows + 2 * TG_M - 1) / (2 * TG_M);
  cfg.gridDim = dim3((unsigned)(2 * std::min<int64_t>(pairs, max_clusters)));
  return cudaLaunchKernelEx(&cfg, row_gemm_pair_kernel<N>, g, amap, bmap, omap);
}

cudaError_t row_gemm(RowGemm g, cudaStream_t st) {
  if (g.rows == 0) return cudaSuccess;
  if (g.K % GK || g.a_split % GK || g.n_out % 4 || g.ldo % 4 || !al16(g.out))
    return cudaErrorInvalidValue;
  g.a_vec = al16(g.A) && g.lda % 4 == 0 && g.a0 % 4 == 0 && g.a1 % 4 == 0;
  g.b_vec = al16(g.B) && g.ldb % 4 == 0;
  // the network's layers (K a multiple of 32, 128 or 256 outputs) run on the
  // tensor cores; other shapes on the CUDA-core kernel
  // (the epilogue moves 16-byte pieces of the output, mask and row-bias rows)
  const bool side_vec = g.ldo % 4 == 0 && !(g.mask && g.row_bias) &&
                        (!g.mask || (al16(g.mask) && g.ldm % 4 == 0)) &&
                        (!g.row_bias || (al16(g.row_bias) && g.n_out % 4 == 0));
  // (the raw A chunks are 2-D tensor copies: 16-byte aligned rows and column
  // offsets on whole chunks)
  const bool a_tma = al16(g.A) && g.lda % 4 == 0 && g.a0 % TG_KC == 0 && g.a1 % TG_KC == 0 &&
                     g.a_split % TG_KC == 0 && g.rows < (int64_t)1 << 31;
  if (g.bsplit && side_vec && a_tma && g.K % TG_KC == 0 && (g.n_out == 128 || g.n_out == 256) &&
      (int64_t)g.K * g.n_out * 2 <= TRAIN_BSPLIT) {
    static bool attr_set[2] = {false, false};
    const int wide = g.n_out == 256;
    if (!attr_set[wide]) {
      cudaError_t e = wide ? cudaFuncSetAttribute(row_gemm_tc_kernel<256>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RG_SMEM)
                           : cudaFuncSetAttribute(row_gemm_tc_kernel<128>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RG_SMEM);
      if (e != cudaSuccess) return e;
      attr_set[wide] = true;
    }
    CUtensorMap amap, omap;
    cudaError_t e = encode_rows_map(&amap, g.A, g.lda, g.rows);
    if (e == cudaSuccess) e = encode_out_map(&omap, g.out, g.ldo, g.n_out, g.rows);
    if (e != cudaSuccess) return e;
    const int64_t nb = (int64_t)g.K * g.n_out;
    if (g.rows >= 2 * TG_M && g.K % RP_KC == 0 && g.a_split % RP_KC == 0 && g.a0 % RP_KC == 0 &&
        g.a1 % RP_KC == 0) {
      // CTA pairs: each SM reads half the weights per MMA (see row_gemm_pair_kernel)
      CUtensorMap bmap, amap2;
      if ((e = encode_bhalf_map(&bmap, g.bsplit, g.K, g.n_out)) != cudaSuccess) return e;
      if ((e = encode_rows_map_sw(&amap2, g.A, g.lda, g.rows)) != cudaSuccess) return e;
      split_b_pair_kernel<<<(unsigned)std::min<int64_t>(blocks_for(nb, 256), 1024), 256, 0, st>>>(
          g.B, g.ldb, g.K, g.n_out, g.bsplit);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      return wide ? launch_row_gemm_pair<256>(g, amap2, bmap, omap, st)
                  : launch_row_gemm_pair<128>(g, amap2, bmap, omap, st);
    }
    split_b_kernel<<<(unsigned)std::min<int64_t>(blocks_for(nb, 256), 1024), 256, 0, st>>>(
        g.B, g.ldb, g.K, g.n_out, g.bsplit);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM walks the row tiles
    const unsigned grid = (unsigned)std::min<int64_t>(blocks_for(g.rows, TG_M), sm_count());
    if (wide) row_gemm_tc_kernel<256><<<grid, RG_THREADS, RG_SMEM, st>>>(g, amap, omap);
    else row_gemm_tc_kernel<128><<<grid, RG_THREADS, RG_SMEM, st>>>(g, amap, omap);
    return cudaGetLastError();
  }
  row_gemm_kernel<<<dim3(blocks_for(g.rows, GT), blocks_for(g.n_out, GT)), 256, 0, st>>>(g);
  return cudaGetLastError();
}

// Row slices sized for about two waves of two CTAs per SM, at least 512 rows each.
int64_t slice_rows(int64_t rows, int tiles) {
  const int64_t want = std::max<int64_t>(1, (4 * (int64_t)sm_count()) / tiles);
  int64_t slice = (rows + want - 1) / want;
  slice = (slice + GK - 1) / GK * GK;
  return std::max<int64_t>(slice, 512);
}

cudaError_t wgrad(WGrad g, cudaStream_t st) {
  if (g.rows == 0) return cudaSuccess;
  // 128 or 256 outputs on the tensor cores, one launch per 256-column tile of X
  if (g.flag && (g.N == 128 || g.N == 256)) {
    static bool attr_set = false;
    if (!attr_set) {
      cudaError_t e = cudaFuncSetAttribute(wgrad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)WT_SMEM);
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    const unsigned grid = (unsigned)std::min<int64_t>((g.rows + WT_KC - 1) / WT_KC, sm_count());
    for (int k0 = 0; k0 < g.K; k0 += 256) {
      int nt = 32;
      while (nt < g.K - k0 && nt < 256) nt *= 2;
      wgrad_tc_kernel<<<grid, TG_THREADS, WT_SMEM, st>>>(g, k0, nt, g.flag);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  g.a_vec = al16(g.A) && g.lda % 4 == 0;
  g.x_vec = al16(g.X) && g.ldx % 4 == 0 && g.x0 % 4 == 0 && g.x1 % 4 == 0 && g.x_split % 4 == 0;
  const unsigned tn = blocks_for(g.N, GT), tk = blocks_for(g.K, GT);
  g.slice = slice_rows(g.rows, (int)(tn * tk));
  const dim3 grid(tn, tk, blocks_for(g.rows, g.slice));
  if (g.x_vec) wgrad_gemm_kernel<true><<<grid, 256, 0, st>>>(g);
  else wgrad_gemm_kernel<false><<<grid, 256, 0, st>>>(g);
  return cudaGetLastError();
}

template <int NS>
cudaError_t wgrad_head(const float* A, int64_t lda, const float* X, int64_t ldx, int x0, int K,
                       int64_t rows, float* G, int64_t ldg, float* db, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (K % 4 || x0 % 4 || ldx % 4 || !al16(X)) return cudaErrorInvalidValue;
  const unsigned bx = blocks_for(K / 4 + 1, 128);
  const int64_t slice = slice_rows(rows, (int)bx);
  wgrad_head_kernel<NS><<<dim3(bx, blocks_for(rows, slice)), 128, 0, st>>>(
      A, lda, X, ldx, x0, K, rows, slice, G, ldg, db);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_composite_bw(const float* raw, const SampleSpec& ss, const float* d, int64_t R,
                                const CompositeSpec& cs, const float* target, float inv3n,
                                float* d_raw, float* loss_terms, cudaStream_t st) {
  if (ss.S > CB_SMAX) return cudaErrorInvalidValue;
  composite_bw_kernel<<<blocks_for(R, CB_WARPS), CB_WARPS * 32, 0, st>>>(raw, ss, d, R, cs, target,
                                                                        inv3n, d_raw, loss_terms);
  return cudaGetLastError();
}

// The training path's forward of one network: the activation store is written
// layer by layer, each layer a row GEMM reading the previous layer's columns.
// The per-output summation order (fmaf over the inputs in order, then + bias,
// then ReLU) is that of the fused forward kernel.
cudaError_t mlp_forward_train_fp32(const PackedFp32& p, const float* pk, const float* dir_bias,
                                   const float* o, const float* d, int64_t R,
                                   const SampleSpec& ss, float* raw, float* save, float* bsplit,
                                   unsigned* flag, cudaStream_t st, int64_t ray0, bool compact) {
  const int D = p.D, W = p.W, Wh = W / 2;
  const int64_t rows = R * ss.S;
  if (rows == 0) return cudaSuccess;
  const int64_t ldc = compact ? compact_ldc(W) : 64 + (int64_t)(D + 1) * W + Wh;
  // compact: layer l writes slot l % 2 and reads slot (l - 1) % 2; the feature
  // layer writes slot D % 2, keeping h_{D-1} (slot (D - 1) % 2) for the sigma head
  auto hcol = [&](int l) { return compact ? 64 + (l & 1) * W : 64 + l * W; };
  const int feat_col = hcol(D), hdir_col = compact ? 64 + 2 * W : hcol(D + 1);
  encode_store_kernel<<<blocks_for(rows, 128), 128, 0, st>>>(o, d, R, ss, save, ldc, ray0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int l = 0; l < D && e == cudaSuccess; ++l) {
    RowGemm g{};
    g.A = save; g.lda = ldc;
    if (l == 0) { g.a0 = 0; g.a_split = 64; g.K = 64; }
    else { g.a0 = hcol(l - 1); g.a_split = W; g.a1 = 0; g.K = l == p.skip + 1 ? W + 64 : W; }
    g.B = pk + p.layer_w[l]; g.ldb = W; g.n_out = W; g.rows = rows;
    g.bias = pk + p.layer_b[l]; g.relu = 1;
    g.out = save + hcol(l); g.ldo = ldc;
    g.bsplit = bsplit; g.flag = flag;
    e = row_gemm(g, st);
  }
  if (e != cudaSuccess) return e;
  {  // feature layer (no activation)
    RowGemm g{};
    g.A = save; g.lda = ldc; g.a0 = hcol(D - 1); g.a_split = W; g.K = W;
    g.B = pk + p.feat_w; g.ldb = W; g.n_out = W; g.rows = rows; g.bias = pk + p.feat_b;
    g.out = save + feat_col; g.ldo = ldc;
    g.bsplit = bsplit; g.flag = flag;
    if ((e = row_gemm(g, st)) != cudaSuccess) return e;
  }
  {  // direction layer: per-ray bias (b_dir + W_dir[:, W:] gamma(d)), ReLU
    RowGemm g{};
    g.A = save; g.lda = ldc; g.a0 = feat_col; g.a_split = W; g.K = W;
    g.B = pk + p.dir_w; g.ldb = Wh; g.n_out = Wh; g.rows = rows;
    g.row_bias = dir_bias; g.rb_div = ss.S; g.relu = 1;
    g.out = save + hdir_col; g.ldo = ldc;
    g.bsplit = bsplit; g.flag = flag;
    if ((e = row_gemm(g, st)) != cudaSuccess) return e;
  }
  heads_fwd_kernel<<<blocks_for(rows * 32, 256), 256, 0, st>>>(save, ldc, hcol(D - 1), hdir_col, W,
                                                              pk, p, rows, raw);
  return cudaGetLastError();
}

// Backward of one network over rows = R * S, given d_raw [rows][4] and the
// forward's activation store. Adds into grad (the flat gradient blob, zeroed
// by the caller). w: the network's fp32 blob. tmp: 2 * rows * W + R * (W/2 + 27)
// floats of scratch.
cudaError_t mlp_backward_fp32(const PackedFp32& p, int L_dir, const float* w, const float* save,
                              int64_t R, int S, const float* d, const float* d_raw,
                              float* grad, float* tmp, float* bsplit, unsigned* flag,
                              cudaStream_t st) {
  const int D = p.D, W = p.W, Wh = W / 2, skip = p.skip;
  const int dir_ch = 3 + 6 * L_dir;
  const int64_t rows = R * S;
  if (rows == 0) return cudaSuccess;
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
  cudaError_t e;
#define NERF_TRY(x) if ((e = (x)) != cudaSuccess) return e
  auto wg = [&](const float* A, int64_t lda, int N, int x0, int split, int x1, int K, float* G,
                int64_t ldg, float* db) {
    WGrad g{};
    g.A = A; g.lda = lda; g.N = N; g.X = save; g.ldx = ldc; g.x0 = x0; g.x_split = split;
    g.x1 = x1; g.K = K; g.rows = rows; g.G = G; g.ldg = ldg; g.db = db; g.flag = flag;
    return wgrad(g, st);
  };
  auto in_grad = [&](const float* A, int64_t lda, int K, const float* B, int64_t ldb,
                     const float* ea, const float* ev, int mcol, float* out) {
    RowGemm g{};
    g.A = A; g.lda = lda; g.a_split = K; g.K = K; g.B = B; g.ldb = ldb; g.n_out = W;
    g.rows = rows; g.ea = ea; g.ldea = 4; g.ev = ev;
    if (mcol >= 0) { g.mask = save + mcol; g.ldm = ldc; }
    g.out = out; g.ldo = W;
    g.bsplit = bsplit; g.flag = flag;
    return row_gemm(g, st);
  };
  // rgb head: dz_dir = (d_rgb x Wr) masked by h_dir > 0; dWr, dbr
  head_bw_kernel<<<blocks_for(rows * Wh, 256), 256, 0, st>>>(d_raw, w + rgb_w, save, ldc, hdir_col,
                                                             rows, Wh, bufA);
  NERF_TRY(cudaGetLastError());
  NERF_TRY(wgrad_head<3>(d_raw, 4, save, ldc, hdir_col, Wh, rows, grad + rgb_w, Wh, grad + rgb_b,
                         st));
  // direction layer: input [feature | gamma(d)]; the gamma(d) part per ray
  NERF_TRY(wg(bufA, Wh, Wh, feat_col, W, 0, W, grad + dir_w, W + dir_ch, grad + dir_b));
  ray_sum_kernel<<<blocks_for(R * Wh, 256), 256, 0, st>>>(bufA, R, S, Wh, dz_ray);
  NERF_TRY(cudaGetLastError());
  dir_enc_kernel<<<blocks_for(R, 128), 128, 0, st>>>(d, R, L_dir, denc);
  NERF_TRY(cudaGetLastError());
  {
    WGrad g{};
    g.A = dz_ray; g.lda = Wh; g.N = Wh; g.X = denc; g.ldx = dir_ch; g.x0 = 0;
    g.x_split = dir_ch; g.x1 = 0; g.K = dir_ch; g.rows = R; g.G = grad + dir_w + W;
    g.ldg = W + dir_ch; g.db = nullptr;
    NERF_TRY(wgrad(g, st));
  }
  // d feature = dz_dir x Wd[:, :W] (no activation on the feature layer)
  NERF_TRY(in_grad(bufA, Wh, Wh, w + dir_w, W + dir_ch, nullptr, nullptr, -1, bufB));
  // feature and sigma heads, both reading h_{D-1}
  NERF_TRY(wg(bufB, W, W, hcol(D - 1), W, 0, W, grad + feat_w, W, grad + feat_b));
  NERF_TRY(wgrad_head<1>(d_raw + 3, 4, save, ldc, hcol(D - 1), W, rows, grad + sig_w, W,
                         grad + sig_b, st));
  // d h_{D-1} = d feature x Wf + d sigma x ws, masked by h_{D-1} > 0
  NERF_TRY(in_grad(bufB, W, W, w + feat_w, W, d_raw + 3, w + sig_w, hcol(D - 1), bufA));
  // the trunk, top down: bufA holds dz of layer l
  for (int l = D - 1; l >= 0; --l) {
    if (l == 0) {
      // gamma(x) is one column range; a split past K keeps the fetches vectorised
      NERF_TRY(wg(bufA, W, W, 0, 64, 0, 63, grad + wo[0], Kl[0], grad + bo[0]));
    } else if (l == skip + 1) {
      NERF_TRY(wg(bufA, W, W, hcol(l - 1), W, 0, W + 63, grad + wo[l], Kl[l], grad + bo[l]));
    } else {
      NERF_TRY(wg(bufA, W, W, hcol(l - 1), W, 0, W, grad + wo[l], Kl[l], grad + bo[l]));
    }
    if (l > 0) {
      NERF_TRY(in_grad(bufA, W, W, w + wo[l], Kl[l], nullptr, nullptr, hcol(l - 1), bufB));
      float* t = bufA; bufA = bufB; bufB = t;
    }
  }
#undef NERF_TRY
  return cudaSuccess;
}

cudaError_t launch_sum(const float* v, int64_t n, float* out, cudaStream_t st) {
  sum_kernel<<<1, 256, 0, st>>>(v, n, out);
  return cudaGetLastError();
}

}  // namespace nerfb
