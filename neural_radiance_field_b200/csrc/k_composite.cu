// Alpha compositing (NeRF page, Sections 1.3 and 2.5) and inverse-CDF
// resampling with the sorted merge (Section 2.6), one warp per ray.
#include "nerf_internal.cuh"

namespace nerfb {

namespace {

constexpr int WARPS = 8;

__device__ __forceinline__ float sample_t(const SampleSpec& ss, int64_t ray, int i) {
  if (ss.mode == SAMPLES_STRATIFIED) {
    uint32_t m = ss.perturb ? draw_bits(ss.key, (uint64_t)ray, 0, (uint32_t)i) : 0u;
    return stratified_t(ss.near, ss.step, i, m, ss.perturb != 0);
  }
  return ss.t[ray * ss.S + i];
}

__device__ __forceinline__ float act_sigma(float r, int mode) {
  if (mode == NERF_SIGMA_SOFTPLUS) return r > 30.0f ? r : log1pf(expf(r));
  return fmaxf(r, 0.0f);
}

__device__ __forceinline__ float sigmoidf_(float r) { return 1.0f / (1.0f + expf(-r)); }

// Composite one ray; lane owns samples lane*C .. lane*C+C-1. Returns the sums
// on every lane; writes per-sample weights to w_out (global or shared) if given.
template <int C>
__device__ void composite_ray(const float* __restrict__ raw, const SampleSpec& ss, int64_t ray,
                              float dnorm, const CompositeSpec& cs, float* w_out,
                              float res[5]) {
  const int lane = threadIdx.x & 31;
  const int S = ss.S;
  float tau[C], tv[C];
  float local = 0.0f;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    int i = lane * C + c;
    tau[c] = 0.0f;
    tv[c] = 0.0f;
    if (i < S) {
      float t = sample_t(ss, ray, i);
      float delta;
      if (i + 1 < S) {
        delta = (sample_t(ss, ray, i + 1) - t) * dnorm;
      } else {
        delta = cs.last_mode == NERF_LAST_1E10 ? 1e10f * dnorm
              : cs.last_mode == NERF_LAST_TO_FAR ? (cs.far - t) * dnorm
                                                 : cs.march_step * dnorm;
      }
      float sigma = act_sigma(raw[((int64_t)ray * S + i) * 4 + 3], cs.sigma_act);
      tau[c] = sigma * delta;
      tv[c] = t;
      local += tau[c];
    }
  }
  // exclusive scan of the lanes' sums (shifted inclusive scan: subtracting a
  // lane's own sum would cancel catastrophically next to the 1e10 interval)
  float incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  float run = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) run = 0.0f;
  float r = 0.f, g = 0.f, b = 0.f, dep = 0.f, acc = 0.f;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    int i = lane * C + c;
    if (i < S) {
      float w = expf(-run) * (-expm1f(-tau[c]));
      run += tau[c];
      const float4 q = *reinterpret_cast<const float4*>(raw + ((int64_t)ray * S + i) * 4);
      r += w * sigmoidf_(q.x);
      g += w * sigmoidf_(q.y);
      b += w * sigmoidf_(q.z);
      dep += w * tv[c];
      acc += w;
      if (w_out) w_out[i] = w;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    r += __shfl_xor_sync(0xffffffffu, r, off);
    g += __shfl_xor_sync(0xffffffffu, g, off);
    b += __shfl_xor_sync(0xffffffffu, b, off);
    dep += __shfl_xor_sync(0xffffffffu, dep, off);
    acc += __shfl_xor_sync(0xffffffffu, acc, off);
  }
  if (cs.white) { r += 1.0f - acc; g += 1.0f - acc; b += 1.0f - acc; }
  res[0] = r; res[1] = g; res[2] = b; res[3] = dep; res[4] = acc;
}

__device__ __forceinline__ float ray_norm(const float* d, int64_t ray) {
  float x = d[ray * 3], y = d[ray * 3 + 1], z = d[ray * 3 + 2];
  return sqrtf(x * x + y * y + z * z);
}

template <int C>
__global__ void composite_kernel(const float* __restrict__ raw, SampleSpec ss,
                                 const float* __restrict__ d, int64_t R, CompositeSpec cs,
                                 float* __restrict__ rgb, float* __restrict__ depth,
                                 float* __restrict__ accum, float* __restrict__ weights) {
  int64_t ray = (int64_t)blockIdx.x * WARPS + threadIdx.x / 32;
  if (ray >= R) return;
  float res[5];
  composite_ray<C>(raw, ss, ray, ray_norm(d, ray), cs, weights ? weights + ray * ss.S : nullptr,
                   res);
  if ((threadIdx.x & 31) == 0) {
    rgb[ray * 3 + 0] = res[0];
    rgb[ray * 3 + 1] = res[1];
    rgb[ray * 3 + 2] = res[2];
    depth[ray] = res[3];
    accum[ray] = res[4];
  }
}

// Per-warp scratch of the resampler.
struct ResampleSmem {
  float tc[64];
  float w[64];
  float bins[64];
  unsigned long long C[64];
  float tf[128];
};

// Inverse-CDF draws from the 62 interior coarse weights over the 63 midpoint
// bins, then the sorted union with the 64 coarse positions. tc, w already in sm.
__device__ void resample_ray(ResampleSmem& sm, int64_t ray, int Nf, uint64_t key, int perturb,
                             float* __restrict__ t_f, int32_t* __restrict__ below_out,
                             float* __restrict__ t_all) {
  const int lane = threadIdx.x & 31;
  // bins: fp32 midpoints
  for (int i = lane; i < 63; i += 32) sm.bins[i] = fmul(0.5f, fadd(sm.tc[i], sm.tc[i + 1]));
  // integer CDF over q_i = floor(fl(w_{i+1} + 1e-5) * 2^32), i = 0..61
  unsigned long long q0 = 0, q1 = 0;
  if (2 * lane < 62)
    q0 = (unsigned long long)((double)fadd(sm.w[1 + 2 * lane], 1e-5f) * 4294967296.0);
  if (2 * lane + 1 < 62)
    q1 = (unsigned long long)((double)fadd(sm.w[2 + 2 * lane], 1e-5f) * 4294967296.0);
  unsigned long long pair = q0 + q1, incl = pair;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    unsigned long long v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  unsigned long long excl = incl - pair;    // C_{2 lane}
  if (2 * lane < 63) sm.C[2 * lane] = excl;
  if (2 * lane + 1 < 63) sm.C[2 * lane + 1] = excl + q0;
  __syncwarp();
  const unsigned long long total = sm.C[62];
  for (int k = lane; k < Nf; k += 32) {
    uint32_t m = perturb ? draw_bits(key, (uint64_t)ray, 1, (uint32_t)k)
                         : (uint32_t)((((uint64_t)(2 * k + 1)) << 23) / (uint64_t)Nf);
    unsigned long long rhs = (unsigned long long)m * total;
    int lo = 0, hi = 63;  // idx = #{c : C_c * 2^24 <= rhs}
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if ((sm.C[mid] << 24) <= rhs) lo = mid + 1; else hi = mid;
    }
    int idx = lo;
    int below = idx - 1 < 0 ? 0 : idx - 1;
    int above = idx > 62 ? 62 : idx;
    unsigned long long cb = sm.C[below], ca = sm.C[above];
    float num = (float)(rhs - (cb << 24));
    float den = 16777216.0f * fmaxf((float)(ca - cb), 1e-5f * (float)total);
    float frac = num / den;
    float b0 = sm.bins[below], b1 = sm.bins[above];
    float t = b0 + frac * (b1 - b0);
    sm.tf[k] = t;
    if (t_f) t_f[ray * Nf + k] = t;
    if (below_out) below_out[ray * Nf + k] = below;
  }
  // pad the draws to 128 with +inf and sort them (bitonic network, 4 keys per lane)
  for (int k = Nf + lane; k < 128; k += 32) sm.tf[k] = __int_as_float(0x7f800000);
  __syncwarp();
  if (!t_all) return;
  for (int kb = 2; kb <= 128; kb <<= 1) {
    for (int j = kb >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = lane + 32 * q;
        const int p = i ^ j;
        if (p > i) {
          const float a = sm.tf[i], b = sm.tf[p];
          const bool up = (i & kb) == 0;
          if (up ? (a > b) : (a < b)) { sm.tf[i] = b; sm.tf[p] = a; }
        }
      }
      __syncwarp();
    }
  }
  // merge with the 64 sorted coarse positions (coarse first among equal values)
  const int S = 64 + Nf;
  for (int j = lane; j < Nf; j += 32) {
    const float v = sm.tf[j];
    int lo = 0, hi = 64;                       // #{c : tc[c] <= v}
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sm.tc[mid] <= v) lo = mid + 1; else hi = mid;
    }
    t_all[ray * S + j + lo] = v;
  }
  for (int c = lane; c < 64; c += 32) {
    const float v = sm.tc[c];
    int lo = 0, hi = Nf;                       // #{f : tf[f] < v}
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sm.tf[mid] < v) lo = mid + 1; else hi = mid;
    }
    t_all[ray * S + c + lo] = v;
  }
}

__global__ void coarse_resample_kernel(const float* __restrict__ raw_c, SampleSpec ss,
                                       const float* __restrict__ d, int64_t R, CompositeSpec cs,
                                       int Nf, uint64_t key, int perturb,
                                       float* __restrict__ t_all, ResampleTrace tr) {
  __shared__ ResampleSmem smem[WARPS];
  const int wid = threadIdx.x / 32, lane = threadIdx.x & 31;
  int64_t ray = (int64_t)blockIdx.x * WARPS + wid;
  if (ray >= R) return;
  ResampleSmem& sm = smem[wid];
  float res[5];
  composite_ray<2>(raw_c, ss, ray, ray_norm(d, ray), cs, sm.w, res);
  for (int i = lane; i < 64; i += 32) sm.tc[i] = sample_t(ss, ray, i);
  __syncwarp();
  if (tr.w)
    for (int i = lane; i < 64; i += 32) tr.w[ray * 64 + i] = sm.w[i];
  resample_ray(sm, ray, Nf, key, perturb, tr.t_f, tr.below, t_all);
}

__global__ void sample_pdf_kernel(const float* __restrict__ t_c, const float* __restrict__ w,
                                  int64_t R, int Nf, uint64_t key, int perturb,
                                  float* __restrict__ t_f, int32_t* __restrict__ below,
                                  float* __restrict__ t_all) {
  __shared__ ResampleSmem smem[WARPS];
  const int wid = threadIdx.x / 32, lane = threadIdx.x & 31;
  int64_t ray = (int64_t)blockIdx.x * WARPS + wid;
  if (ray >= R) return;
  ResampleSmem& sm = smem[wid];
  for (int i = lane; i < 64; i += 32) {
    sm.tc[i] = t_c[ray * 64 + i];
    sm.w[i] = w[ray * 64 + i];
  }
  __syncwarp();
  resample_ray(sm, ray, Nf, key, perturb, t_f, below, t_all);
}

}  // namespace

cudaError_t launch_composite(const float* raw, const SampleSpec& ss, const float* d, int64_t R,
                             const CompositeSpec& cs, float* rgb, float* depth, float* acc,
                             float* weights, cudaStream_t st) {
  unsigned blocks = (unsigned)((R + WARPS - 1) / WARPS);
  if (ss.S <= 64)
    composite_kernel<2><<<blocks, WARPS * 32, 0, st>>>(raw, ss, d, R, cs, rgb, depth, acc, weights);
  else if (ss.S <= 192)
    composite_kernel<6><<<blocks, WARPS * 32, 0, st>>>(raw, ss, d, R, cs, rgb, depth, acc, weights);
  else if (ss.S <= 512)
    composite_kernel<16><<<blocks, WARPS * 32, 0, st>>>(raw, ss, d, R, cs, rgb, depth, acc, weights);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_coarse_resample(const float* raw_c, const SampleSpec& coarse, const float* d,
                                   int64_t R, const CompositeSpec& cs, int Nf, uint64_t key,
                                   int perturb, float* t_all, cudaStream_t st,
                                   const ResampleTrace& tr) {
  if (coarse.S != 64 || Nf < 1 || Nf > 128) return cudaErrorInvalidValue;
  unsigned blocks = (unsigned)((R + WARPS - 1) / WARPS);
  coarse_resample_kernel<<<blocks, WARPS * 32, 0, st>>>(raw_c, coarse, d, R, cs, Nf, key, perturb,
                                                        t_all, tr);
  return cudaGetLastError();
}

cudaError_t launch_sample_pdf(const float* t_c, const float* w, int64_t R, int Nc, int Nf,
                              uint64_t key, int perturb, float* t_f, int32_t* below,
                              float* t_all, cudaStream_t st) {
  if (Nc != 64 || Nf < 1 || Nf > 128) return cudaErrorInvalidValue;
  unsigned blocks = (unsigned)((R + WARPS - 1) / WARPS);
  sample_pdf_kernel<<<blocks, WARPS * 32, 0, st>>>(t_c, w, R, Nf, key, perturb, t_f, below, t_all);
  return cudaGetLastError();
}

}  // namespace nerfb
