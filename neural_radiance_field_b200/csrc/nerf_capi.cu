// The C ABI: argument validation, the context's workspace and the order of the
// kernels of one render (NeRF page, Section 2.6 render_rays).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "nerf_internal.cuh"
#include "nerf_ctx.h"

using namespace nerfb;

namespace {

thread_local std::string g_create_error;

nerf_status fail(nerf_ctx* ctx, nerf_status st, const char* fmt, ...) __attribute__((format(printf, 3, 4)));
nerf_status fail(nerf_ctx* ctx, nerf_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (ctx) ctx->err = buf; else g_create_error = buf;
  return st;
}

nerf_status cuda_fail(nerf_ctx* ctx, cudaError_t e, const char* where) {
  return fail(ctx, NERF_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define NERF_CHECK_LAUNCH(ctx, expr)                                  \
  do {                                                                \
    cudaError_t e_ = (expr);                                          \
    if (e_ != cudaSuccess) return cuda_fail((ctx), e_, #expr);        \
  } while (0)

template <class T>
cudaError_t dalloc(T** p, size_t count) {
  *p = nullptr;
  if (count == 0) return cudaSuccess;
  return cudaMalloc((void**)p, count * sizeof(T));
}

int64_t mlp_param_count(int D, int W, int skip, int pos_ch, int dir_ch) {
  int64_t n = 0;
  for (int l = 0; l < D; ++l) {
    int k = l == 0 ? pos_ch : (l == skip + 1 ? W + pos_ch : W);
    n += (int64_t)W * k + W;
  }
  n += W + 1;                                   // sigma
  n += (int64_t)W * W + W;                      // feature
  n += (int64_t)(W / 2) * (W + dir_ch) + W / 2; // dir
  n += 3 * (W / 2) + 3;                         // rgb
  return n;
}

// Offsets of the direction layer's weight and bias in the ABI blob.
void dir_offsets(const nerf_config& c, int64_t* w_off, int64_t* b_off) {
  const int pos_ch = 3 * (1 + 2 * c.L_pos);
  int64_t n = 0;
  for (int l = 0; l < c.D; ++l) {
    int k = l == 0 ? pos_ch : (l == c.skip + 1 ? c.W + pos_ch : c.W);
    n += (int64_t)c.W * k + c.W;
  }
  n += c.W + 1;
  n += (int64_t)c.W * c.W + c.W;
  *w_off = n;
  *b_off = n + (int64_t)(c.W / 2) * (c.W + 3 * (1 + 2 * c.L_dir));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

void free_march(nerf_ctx* ctx) {
  MarchWs& w = ctx->mws;
  cudaFree(w.mask); cudaFree(w.count); cudaFree(w.off); cudaFree(w.scan_tmp);
  cudaFree(w.live); cudaFree(w.val); cudaFree(w.cell); cudaFree(w.order);
  cudaFree(w.cell_hist); cudaFree(w.cell_off); cudaFree(w.items); cudaFree(w.n_items);
  w = MarchWs{};
}

// Contexts of the march models: rays are processed in chunks of up to 2^19, each
// with room for every candidate of every ray, so no input can overflow it.
nerf_status create_march(const nerf_config& c, nerf_ctx** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(nullptr, NERF_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
  nerf_ctx* ctx = new nerf_ctx();
  ctx->cfg = c;
  ctx->device = dev;
  cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t chunk = c.max_rays < (int64_t(1) << 19) ? c.max_rays : (int64_t(1) << 19);
  ctx->chunk_rays = chunk;
  MarchWs& w = ctx->mws;
  w.cap = chunk * c.max_samples;
  bool ok = true;
  ok &= dalloc(&w.mask, (size_t)(chunk * 16)) == cudaSuccess;
  ok &= dalloc(&w.count, (size_t)chunk) == cudaSuccess;
  ok &= dalloc(&w.off, (size_t)(chunk + 1)) == cudaSuccess;
  ok &= dalloc(&w.scan_tmp, 2048) == cudaSuccess;
  ok &= dalloc(&w.live, (size_t)w.cap) == cudaSuccess;
  ok &= dalloc(&w.val, (size_t)(w.cap * 4)) == cudaSuccess;
  if (c.model == NERF_MODEL_KILONERF) {
    ok &= dalloc(&w.cell, (size_t)w.cap) == cudaSuccess;
    ok &= dalloc(&w.order, (size_t)w.cap) == cudaSuccess;
    ok &= dalloc(&w.cell_hist, 2 * 4096) == cudaSuccess;
    ok &= dalloc(&w.cell_off, 4097) == cudaSuccess;
    ok &= dalloc(&w.items, (size_t)(w.cap / 128 + 4096)) == cudaSuccess;
    ok &= dalloc(&w.n_items, 1) == cudaSuccess;
    if (ok) w.cell_fill = w.cell_hist + 4096;
  }
  ok &= dalloc(&ctx->stage, (size_t)(c.max_rays * 11)) == cudaSuccess;
  ok &= dalloc(&ctx->d_flag, 1) == cudaSuccess;
  if (ok) ok &= cudaMemset(ctx->d_flag, 0, sizeof(unsigned)) == cudaSuccess;
  if (ok) ok &= march_prepare(nullptr) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    nerf_destroy(ctx);
    return fail(nullptr, NERF_ERR_OOM, "march workspace allocation failed for max_rays=%lld, max_samples=%d",
                (long long)c.max_rays, c.max_samples);
  }
  *out = ctx;
  return NERF_OK;
}

}  // namespace

extern "C" {

const char* nerf_last_error(const nerf_ctx* ctx) {
  return ctx ? ctx->err.c_str() : g_create_error.c_str();
}

nerf_status nerf_create(const nerf_config* cfg, nerf_ctx** out) {
  if (!out) return fail(nullptr, NERF_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg) return fail(nullptr, NERF_ERR_INVALID_ARG, "cfg is NULL");
  const nerf_config c = *cfg;
  if (c.max_rays <= 0 || c.max_samples <= 0 || c.max_samples > 512)
    return fail(nullptr, NERF_ERR_INVALID_ARG, "max_rays must be > 0 and 0 < max_samples <= 512");
  if (c.last_delta_mode != NERF_LAST_1E10 && c.last_delta_mode != NERF_LAST_TO_FAR)
    return fail(nullptr, NERF_ERR_INVALID_ARG, "last_delta_mode must be 0 or 1");
  if (c.sigma_act != NERF_SIGMA_RELU && c.sigma_act != NERF_SIGMA_SOFTPLUS)
    return fail(nullptr, NERF_ERR_INVALID_ARG, "sigma_act must be RELU or SOFTPLUS");
  if (c.model == NERF_MODEL_MLP) {
    if (c.L_pos != 10 || c.L_dir != 4)
      return fail(nullptr, NERF_ERR_UNSUPPORTED, "L_pos must be 10 and L_dir 4");
    // compact shapes (NAS-NeRF page): any depth 1..8, width 64/128/256, the
    // skip concatenation after any layer but the last, or none
    const bool big = (c.W == 256 && c.D == 8 && c.skip == 4);
    const bool shape_ok = (c.W == 64 || c.W == 128 || c.W == 256) && c.D >= 1 && c.D <= 8 &&
                          (c.skip == -1 || (c.skip >= 0 && c.skip <= c.D - 2));
    if (!shape_ok)
      return fail(nullptr, NERF_ERR_UNSUPPORTED,
                  "network must have W in {64, 128, 256}, D in 1..8 and skip -1 or in 0..D-2");
    if (c.precision != NERF_FP32 && c.precision != NERF_BF16 && c.precision != NERF_TF32)
      return fail(nullptr, NERF_ERR_INVALID_ARG, "precision must be FP32, BF16 or TF32");
    if (c.precision == NERF_BF16 && !big)
      return fail(nullptr, NERF_ERR_UNSUPPORTED, "BF16 tensor-core path needs W=256, D=8");
    if (c.precision == NERF_TF32 && c.W == 64)
      return fail(nullptr, NERF_ERR_UNSUPPORTED, "TF32 tensor-core layers need W in {128, 256}");
  } else if (c.model == NERF_MODEL_KILONERF || c.model == NERF_MODEL_HASHGRID) {
    if (c.model == NERF_MODEL_HASHGRID && c.precision != NERF_FP32 && c.precision != NERF_BF16)
      return fail(nullptr, NERF_ERR_INVALID_ARG, "precision must be FP32 or BF16");
    return create_march(c, out);
  } else {
    return fail(nullptr, NERF_ERR_INVALID_ARG, "unknown model %d", c.model);
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(nullptr, NERF_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));

  nerf_ctx* ctx = new nerf_ctx();
  ctx->cfg = c;
  ctx->device = dev;
  const int pos_ch = 3 * (1 + 2 * c.L_pos), dir_ch = 3 * (1 + 2 * c.L_dir);
  ctx->plan = plan_fp32(c.D, c.W, c.skip, pos_ch, dir_ch);
  ctx->n_params = mlp_param_count(c.D, c.W, c.skip, pos_ch, dir_ch);
  const int64_t R = c.max_rays, S = c.max_samples;
  bool ok = true;
  ok &= dalloc(&ctx->packed, (size_t)ctx->plan.total) == cudaSuccess;
  ok &= dalloc(&ctx->dir_bias, (size_t)(R * (c.W / 2))) == cudaSuccess;
  ok &= dalloc(&ctx->raw, (size_t)(R * S * 4)) == cudaSuccess;
  ok &= dalloc(&ctx->t_all, (size_t)(R * S)) == cudaSuccess;
  ok &= dalloc(&ctx->stage, (size_t)(R * 11)) == cudaSuccess;
  ok &= dalloc(&ctx->d_flag, 1) == cudaSuccess;
  if (ok) ok &= cudaMemset(ctx->d_flag, 0, sizeof(unsigned)) == cudaSuccess;
  if (ok && c.precision == NERF_BF16) ok &= tc_alloc(ctx) == cudaSuccess;
  if (ok && c.precision == NERF_TF32) {
    // the layer outputs of a sub-batch of up to 2^20 samples
    ctx->fw_rows = std::min<int64_t>(R * S, (int64_t)1 << 20);
    ok &= dalloc(&ctx->fw_save, (size_t)(ctx->fw_rows * compact_ldc(c.W))) == cudaSuccess;
    ok &= dalloc(&ctx->tr_bsplit, (size_t)TRAIN_BSPLIT) == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    nerf_destroy(ctx);
    return fail(nullptr, NERF_ERR_OOM, "workspace allocation failed for max_rays=%lld, max_samples=%d",
                (long long)R, (int)S);
  }
  *out = ctx;
  return NERF_OK;
}

nerf_status nerf_destroy(nerf_ctx* ctx) {
  if (!ctx) return NERF_OK;
  cudaDeviceSynchronize();
  cudaFree(ctx->packed);
  cudaFree(ctx->dir_bias);
  cudaFree(ctx->raw);
  cudaFree(ctx->t_all);
  cudaFree(ctx->stage);
  cudaFree(ctx->d_flag);
  cudaFree(ctx->tr_save);
  cudaFree(ctx->tr_draw);
  cudaFree(ctx->tr_tmp);
  cudaFree(ctx->tr_bsplit);
  cudaFree(ctx->fw_save);
  cudaFree(ctx->tr_loss);
  free_march(ctx);
  if (ctx->ev) {
    for (int i = 0; i < 2 * kMaxTimed; ++i) cudaEventDestroy(ctx->ev[i]);
    delete[] ctx->ev;
    delete[] ctx->ev_kind;
  }
  tc_free(ctx);
  delete ctx;
  return NERF_OK;
}

nerf_status nerf_sync_status(nerf_ctx* ctx, void* stream) {
  if (!ctx) return fail(nullptr, NERF_ERR_INVALID_ARG, "ctx is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaStreamSynchronize");
  unsigned flag = 0;
  e = cudaMemcpy(&flag, ctx->d_flag, sizeof flag, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "reading the device flag");
  if (flag) {
    cudaMemset(ctx->d_flag, 0, sizeof(unsigned));
    if (flag & FLAG_TIMEOUT) return fail(ctx, NERF_ERR_TIMEOUT, "a bounded device wait gave up (flag 0x%x)", flag);
    return fail(ctx, NERF_ERR_DEVICE_FLAG, "a kernel reported an out-of-range input (flag 0x%x)", flag);
  }
  return NERF_OK;
}

nerf_status nerf_raygen(int H, int W, float focal, const float* c2w_host, float* rays_o,
                        float* rays_d, void* stream) {
  if (H <= 0 || W <= 0 || !(focal > 0.0f) || !c2w_host || !rays_o || !rays_d)
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_raygen: bad size, focal or NULL pointer");
  NERF_CHECK_LAUNCH(nullptr, launch_raygen(H, W, focal, c2w_host, rays_o, rays_d, (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_raygen_batch(int H, int W, float focal, int n_cams, const float* c2w_host,
                              float* rays_o, float* rays_d, void* stream) {
  if (H <= 0 || W <= 0 || n_cams <= 0 || !(focal > 0.0f) || !c2w_host || !rays_o || !rays_d)
    return fail(nullptr, NERF_ERR_INVALID_ARG,
                "nerf_raygen_batch: bad size, camera count, focal or NULL pointer");
  if ((int64_t)H * W * n_cams > ((int64_t)1 << 40))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_raygen_batch: too many rays");
  NERF_CHECK_LAUNCH(nullptr, launch_raygen_batch(H, W, focal, n_cams, c2w_host, rays_o, rays_d,
                                                 (cudaStream_t)stream));
  return NERF_OK;
}

}  // extern "C"

// --------------------------------------------------------------------------
// render
// --------------------------------------------------------------------------

namespace {

// Events around the launches of one kernel class while timing is enabled.
struct TimedScope {
  KernelTimer tm;
  cudaStream_t st;
  int slot;
  TimedScope(nerf_ctx* c, int kind, cudaStream_t s) : tm(c->timer()), st(s) {
    slot = tm.begin(kind, st);
  }
  ~TimedScope() { tm.end(slot, st); }
};

// Runs one network (coarse or fine) over R rays with S samples each; `save`
// (fp32 path only) receives the activations the training path's backward reads.
nerf_status run_network(nerf_ctx* ctx, const void* blob, const float* o, const float* d,
                        int64_t R, const SampleSpec& ss, float* raw, cudaStream_t st,
                        float* save = nullptr) {
  const nerf_config& c = ctx->cfg;
  int64_t w_off, b_off;
  dir_offsets(c, &w_off, &b_off);
  {
    TimedScope ts(ctx, TK_DIR_BIAS, st);
    NERF_CHECK_LAUNCH(ctx, launch_dir_bias(d, R, blob, c.precision, c.W, c.L_dir, w_off, b_off,
                                           ctx->dir_bias, st));
  }
  if (c.precision == NERF_BF16 && ctx->tc_enabled) {
    NERF_CHECK_LAUNCH(ctx, tc_pack(ctx, blob, st));
    TimedScope ts(ctx, TK_NETWORK, st);
    NERF_CHECK_LAUNCH(ctx, tc_run(ctx, o, d, R, ss, raw, st));
    return NERF_OK;
  }
  const int dir_ch = 3 * (1 + 2 * c.L_dir);
  NERF_CHECK_LAUNCH(ctx, launch_pack_fp32(blob, c.precision, ctx->plan, dir_ch, ctx->packed, st));
  TimedScope ts(ctx, TK_NETWORK, st);
  if (save) {
    NERF_CHECK_LAUNCH(ctx, mlp_forward_train_fp32(ctx->plan, ctx->packed, ctx->dir_bias, o, d, R,
                                                  ss, raw, save, ctx->tr_bsplit, ctx->d_flag, st));
  } else if (c.precision == NERF_TF32) {
    // layer by layer on the tensor cores, in sub-batches of whole rays that fit
    // the activation store
    const int64_t per = std::max<int64_t>(1, ctx->fw_rows / ss.S);
    for (int64_t r0 = 0; r0 < R; r0 += per) {
      const int64_t n = std::min(per, R - r0);
      SampleSpec sub = ss;
      if (ss.mode == SAMPLES_GIVEN_T) sub.t = ss.t + r0 * ss.S;
      if (ss.mode == SAMPLES_GIVEN_X) sub.t = ss.t + r0 * ss.S * 3;
      NERF_CHECK_LAUNCH(ctx, mlp_forward_train_fp32(ctx->plan, ctx->packed,
                                                    ctx->dir_bias + r0 * (c.W / 2), o + r0 * 3,
                                                    d + r0 * 3, n, sub, raw + r0 * ss.S * 4,
                                                    ctx->fw_save, ctx->tr_bsplit, ctx->d_flag, st,
                                                    r0, true));
    }
  } else {
    NERF_CHECK_LAUNCH(ctx, launch_mlp_fp32(ctx->plan, ctx->packed, ctx->dir_bias, o, d, R, ss, raw,
                                           st));
  }
  return NERF_OK;
}

nerf_status check_render_args(nerf_ctx* ctx, const float* o, const float* d, int64_t n_rays,
                              float near, float far, int n_coarse, int n_fine,
                              const nerf_params* p, const float* rgb, const float* depth,
                              const float* acc) {
  if (!ctx) return fail(nullptr, NERF_ERR_INVALID_ARG, "ctx is NULL");
  const nerf_config& c = ctx->cfg;
  if (!o || !d || !p || !rgb || !depth || !acc)
    return fail(ctx, NERF_ERR_INVALID_ARG, "NULL ray, params or output pointer");
  if (n_rays <= 0 || n_rays > c.max_rays)
    return fail(ctx, NERF_ERR_INVALID_ARG, "n_rays=%lld outside (0, max_rays=%lld]",
                (long long)n_rays, (long long)c.max_rays);
  if (!(near < far)) return fail(ctx, NERF_ERR_INVALID_ARG, "near must be < far");
  if (n_coarse <= 0 || n_fine < 0 || n_coarse + n_fine > c.max_samples)
    return fail(ctx, NERF_ERR_INVALID_ARG, "n_coarse + n_fine must be in (0, max_samples=%d]",
                c.max_samples);
  if (c.model == NERF_MODEL_MLP) {
    if (!p->coarse_w) return fail(ctx, NERF_ERR_INVALID_ARG, "coarse_w is NULL");
    if (n_fine > 0) {
      if (!p->fine_w) return fail(ctx, NERF_ERR_INVALID_ARG, "fine_w is NULL with n_fine > 0");
      if (n_coarse != 64 || n_fine > 128)
        return fail(ctx, NERF_ERR_UNSUPPORTED, "the fine pass needs n_coarse = 64, n_fine <= 128");
    }
    if (c.precision == NERF_BF16 && (!aligned16(p->coarse_w) || (n_fine > 0 && !aligned16(p->fine_w))))
      return fail(ctx, NERF_ERR_INVALID_ARG, "bf16 weight blobs must be 16-byte aligned");
  } else {
    if (n_fine != 0) return fail(ctx, NERF_ERR_INVALID_ARG, "march models take n_fine = 0");
    if (n_coarse > 512) return fail(ctx, NERF_ERR_INVALID_ARG, "march candidates must be <= 512");
    if (!p->occupancy) return fail(ctx, NERF_ERR_INVALID_ARG, "occupancy grid is NULL");
    if (!(p->march_step > 0.0f)) return fail(ctx, NERF_ERR_INVALID_ARG, "march_step must be > 0");
    if (!(p->ert_T >= 0.0f && p->ert_T < 1.0f))
      return fail(ctx, NERF_ERR_INVALID_ARG, "ert_T must be in [0, 1)");
    if (c.model == NERF_MODEL_KILONERF && !p->cell_w)
      return fail(ctx, NERF_ERR_INVALID_ARG, "cell_w is NULL");
    if (c.model == NERF_MODEL_HASHGRID && (!p->hash_table || !p->hash_mlp || !aligned16(p->hash_mlp)))
      return fail(ctx, NERF_ERR_INVALID_ARG, "hash_table / hash_mlp NULL or misaligned");
  }
  return NERF_OK;
}

nerf_status render_march(nerf_ctx* ctx, const float* o, const float* d, int64_t R, float near,
                         int K, const nerf_params* p, float* rgb, float* depth, float* acc,
                         cudaStream_t st) {
  MarchArgs a{};
  a.model = ctx->cfg.model;
  a.o = o;
  a.d = d;
  a.near = near;
  a.step = p->march_step;
  a.ert_T = p->ert_T;
  a.K = K;
  a.occ = p->occupancy;
  a.cell_w = p->cell_w;
  a.hash_table = p->hash_table;
  a.hash_mlp = p->hash_mlp;
  a.sh = sh_constants();
  a.rgb = rgb;
  a.depth = depth;
  a.acc = acc;
  a.flag = ctx->d_flag;
  a.num_sms = ctx->num_sms;
  a.hash_tc = ctx->cfg.model == NERF_MODEL_HASHGRID && ctx->cfg.precision == NERF_BF16;
  a.ws = ctx->mws;
  for (int64_t r0 = 0; r0 < R; r0 += ctx->chunk_rays) {
    a.r0 = r0;
    a.R = R - r0 < ctx->chunk_rays ? R - r0 : ctx->chunk_rays;
    a.timer = ctx->timer();
    NERF_CHECK_LAUNCH(ctx, march_render_chunk(a, st));
  }
  return NERF_OK;
}

// The NeRF model's render (Section 2.6 render_rays): coarse network, coarse
// compositing fused with resampling and the sorted merge, fine network, fine
// compositing. `tr` (may be NULL) receives copies of the intermediates.
nerf_status render_mlp(nerf_ctx* ctx, const float* rays_o, const float* rays_d, int64_t R,
                       float near, float far, int n_coarse, int n_fine, const nerf_params* params,
                       float* out_rgb, float* out_depth, float* out_acc, const nerf_trace* tr,
                       cudaStream_t st) {
  const nerf_config& c = ctx->cfg;
  const uint64_t key = sm64_mix(params->seed);
  SampleSpec coarse{};
  coarse.mode = SAMPLES_STRATIFIED;
  coarse.S = n_coarse;
  coarse.near = near;
  coarse.step = (far - near) / (float)n_coarse;
  coarse.key = key;
  coarse.perturb = params->perturb;
  CompositeSpec cs{c.last_delta_mode, far, 0.0f, c.sigma_act, c.white_bkgd};

  nerf_status s = run_network(ctx, params->coarse_w, rays_o, rays_d, R, coarse, ctx->raw, st);
  if (s != NERF_OK) return s;
  if (tr && tr->raw_coarse)
    NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(tr->raw_coarse, ctx->raw, (size_t)R * n_coarse * 16,
                                           cudaMemcpyDeviceToDevice, st));
  if (n_fine == 0) {
    TimedScope ts(ctx, TK_COMPOSITE, st);
    NERF_CHECK_LAUNCH(ctx, launch_composite(ctx->raw, coarse, rays_d, R, cs, out_rgb, out_depth,
                                            out_acc, tr ? tr->w_coarse : nullptr, st));
    return NERF_OK;
  }
  ResampleTrace rt{};
  if (tr) {
    rt.w = tr->w_coarse;
    rt.t_f = tr->t_fine;
    rt.below = tr->below;
  }
  {
    TimedScope ts(ctx, TK_RESAMPLE, st);
    NERF_CHECK_LAUNCH(ctx, launch_coarse_resample(ctx->raw, coarse, rays_d, R, cs, n_fine, key,
                                                  params->perturb, ctx->t_all, st, rt));
  }
  SampleSpec fine{};
  fine.mode = SAMPLES_GIVEN_T;
  fine.S = n_coarse + n_fine;
  fine.t = ctx->t_all;
  if (tr && tr->t_all)
    NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(tr->t_all, ctx->t_all, (size_t)R * fine.S * 4,
                                           cudaMemcpyDeviceToDevice, st));
  s = run_network(ctx, params->fine_w, rays_o, rays_d, R, fine, ctx->raw, st);
  if (s != NERF_OK) return s;
  if (tr && tr->raw_fine)
    NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(tr->raw_fine, ctx->raw, (size_t)R * fine.S * 16,
                                           cudaMemcpyDeviceToDevice, st));
  TimedScope ts(ctx, TK_COMPOSITE, st);
  NERF_CHECK_LAUNCH(ctx, launch_composite(ctx->raw, fine, rays_d, R, cs, out_rgb, out_depth,
                                          out_acc, nullptr, st));
  return NERF_OK;
}

}  // namespace

extern "C" {

nerf_status nerf_render(nerf_ctx* ctx, const float* rays_o, const float* rays_d, int64_t n_rays,
                        float near, float far, int n_coarse, int n_fine, const nerf_params* params,
                        float* out_rgb, float* out_depth, float* out_acc, void* stream) {
  nerf_status s = check_render_args(ctx, rays_o, rays_d, n_rays, near, far, n_coarse, n_fine,
                                    params, out_rgb, out_depth, out_acc);
  if (s != NERF_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (ctx->cfg.model != NERF_MODEL_MLP)
    return render_march(ctx, rays_o, rays_d, n_rays, near, n_coarse, params, out_rgb, out_depth,
                        out_acc, st);
  return render_mlp(ctx, rays_o, rays_d, n_rays, near, far, n_coarse, n_fine, params, out_rgb,
                    out_depth, out_acc, nullptr, st);
}

nerf_status nerf_render_trace(nerf_ctx* ctx, const float* rays_o, const float* rays_d,
                              int64_t n_rays, float near, float far, int n_coarse, int n_fine,
                              const nerf_params* params, float* out_rgb, float* out_depth,
                              float* out_acc, const nerf_trace* trace, void* stream) {
  nerf_status s = check_render_args(ctx, rays_o, rays_d, n_rays, near, far, n_coarse, n_fine,
                                    params, out_rgb, out_depth, out_acc);
  if (s != NERF_OK) return s;
  if (!trace) return fail(ctx, NERF_ERR_INVALID_ARG, "trace is NULL");
  if (ctx->cfg.model != NERF_MODEL_MLP)
    return fail(ctx, NERF_ERR_UNSUPPORTED, "nerf_render_trace needs a NERF_MODEL_MLP context");
  return render_mlp(ctx, rays_o, rays_d, n_rays, near, far, n_coarse, n_fine, params, out_rgb,
                    out_depth, out_acc, trace, (cudaStream_t)stream);
}

nerf_status nerf_loss_grad(nerf_ctx* ctx, const float* rays_o, const float* rays_d,
                           int64_t n_rays, float near, float far, int n_coarse, int n_fine,
                           const nerf_params* params, const float* target_rgb, float* out_loss,
                           float* grad_coarse, float* grad_fine, void* stream) {
  if (!ctx) return fail(nullptr, NERF_ERR_INVALID_ARG, "ctx is NULL");
  const nerf_config& c = ctx->cfg;
  if (c.model != NERF_MODEL_MLP || (c.precision != NERF_FP32 && c.precision != NERF_TF32))
    return fail(ctx, NERF_ERR_UNSUPPORTED, "nerf_loss_grad needs an fp32 NERF_MODEL_MLP context");
  if (!rays_o || !rays_d || !params || !target_rgb || !out_loss || !grad_coarse ||
      (n_fine > 0 && !grad_fine))
    return fail(ctx, NERF_ERR_INVALID_ARG, "NULL ray, params, target, loss or gradient pointer");
  if (n_rays <= 0 || n_rays > c.max_rays)
    return fail(ctx, NERF_ERR_INVALID_ARG, "n_rays=%lld outside (0, max_rays=%lld]",
                (long long)n_rays, (long long)c.max_rays);
  if (!(near < far)) return fail(ctx, NERF_ERR_INVALID_ARG, "near must be < far");
  const int s_max = c.max_samples < 256 ? c.max_samples : 256;
  if (n_coarse < 2 || n_fine < 0 || n_coarse + n_fine > s_max)
    return fail(ctx, NERF_ERR_INVALID_ARG,
                "n_coarse >= 2 and n_coarse + n_fine <= min(max_samples, 256) on the training path");
  if (!params->coarse_w || (n_fine > 0 && !params->fine_w))
    return fail(ctx, NERF_ERR_INVALID_ARG, "weight blob is NULL");
  if (n_fine > 0 && (n_coarse != 64 || n_fine > 128))
    return fail(ctx, NERF_ERR_UNSUPPORTED, "the fine pass needs n_coarse = 64, n_fine <= 128");
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t R = n_rays, W = c.W;
  const int64_t ldc = 64 + (int64_t)(c.D + 1) * W + W / 2;
  const int dir_ch = 3 * (1 + 2 * c.L_dir);
  if (!ctx->tr_save) {
    const int64_t rows = c.max_rays * (int64_t)s_max;
    bool ok = dalloc(&ctx->tr_save, (size_t)(rows * ldc)) == cudaSuccess;
    ok &= dalloc(&ctx->tr_draw, (size_t)(rows * 4)) == cudaSuccess;
    ok &= dalloc(&ctx->tr_tmp, (size_t)(2 * rows * W + c.max_rays * (W / 2 + dir_ch))) == cudaSuccess;
    ok &= dalloc(&ctx->tr_loss, (size_t)(2 * c.max_rays)) == cudaSuccess;
    if (ok && !ctx->tr_bsplit) ok &= dalloc(&ctx->tr_bsplit, (size_t)TRAIN_BSPLIT) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      cudaFree(ctx->tr_save); cudaFree(ctx->tr_draw); cudaFree(ctx->tr_tmp); cudaFree(ctx->tr_loss);
      ctx->tr_save = ctx->tr_draw = ctx->tr_tmp = ctx->tr_loss = nullptr;
      return fail(ctx, NERF_ERR_OOM, "training workspace allocation failed");
    }
  }
  const size_t gbytes = (size_t)ctx->n_params * sizeof(float);
  NERF_CHECK_LAUNCH(ctx, cudaMemsetAsync(grad_coarse, 0, gbytes, st));
  if (n_fine > 0) NERF_CHECK_LAUNCH(ctx, cudaMemsetAsync(grad_fine, 0, gbytes, st));
  const uint64_t key = sm64_mix(params->seed);
  SampleSpec coarse{};
  coarse.mode = SAMPLES_STRATIFIED;
  coarse.S = n_coarse;
  coarse.near = near;
  coarse.step = (far - near) / (float)n_coarse;
  coarse.key = key;
  coarse.perturb = params->perturb;
  CompositeSpec cs{c.last_delta_mode, far, 0.0f, c.sigma_act, c.white_bkgd};
  const float inv3n = 1.0f / (3.0f * (float)R);
  // coarse pass: forward with the activation store, the fine positions from
  // its (detached) weights, then its backward
  nerf_status s = run_network(ctx, params->coarse_w, rays_o, rays_d, R, coarse, ctx->raw, st,
                              ctx->tr_save);
  if (s != NERF_OK) return s;
  if (n_fine > 0)
    NERF_CHECK_LAUNCH(ctx, launch_coarse_resample(ctx->raw, coarse, rays_d, R, cs, n_fine, key,
                                                  params->perturb, ctx->t_all, st));
  NERF_CHECK_LAUNCH(ctx, launch_composite_bw(ctx->raw, coarse, rays_d, R, cs, target_rgb, inv3n,
                                             ctx->tr_draw, ctx->tr_loss, st));
  NERF_CHECK_LAUNCH(ctx, mlp_backward_fp32(ctx->plan, c.L_dir, (const float*)params->coarse_w,
                                           ctx->tr_save, R, n_coarse, rays_d, ctx->tr_draw,
                                           grad_coarse, ctx->tr_tmp, ctx->tr_bsplit, ctx->d_flag,
                                           st));
  if (n_fine > 0) {
    SampleSpec fine{};
    fine.mode = SAMPLES_GIVEN_T;
    fine.S = n_coarse + n_fine;
    fine.t = ctx->t_all;
    s = run_network(ctx, params->fine_w, rays_o, rays_d, R, fine, ctx->raw, st, ctx->tr_save);
    if (s != NERF_OK) return s;
    NERF_CHECK_LAUNCH(ctx, launch_composite_bw(ctx->raw, fine, rays_d, R, cs, target_rgb, inv3n,
                                               ctx->tr_draw, ctx->tr_loss + R, st));
    NERF_CHECK_LAUNCH(ctx, mlp_backward_fp32(ctx->plan, c.L_dir, (const float*)params->fine_w,
                                             ctx->tr_save, R, fine.S, rays_d, ctx->tr_draw,
                                             grad_fine, ctx->tr_tmp, ctx->tr_bsplit, ctx->d_flag,
                                             st));
  }
  NERF_CHECK_LAUNCH(ctx, launch_sum(ctx->tr_loss, n_fine > 0 ? 2 * R : R, out_loss, st));
  return NERF_OK;
}

nerf_status nerf_render_host(nerf_ctx* ctx, const float* rays_o_host, const float* rays_d_host,
                             int64_t n_rays, float near, float far, int n_coarse, int n_fine,
                             const nerf_params* params, float* out_rgb_host, float* out_depth_host,
                             float* out_acc_host, void* stream) {
  nerf_status s = check_render_args(ctx, rays_o_host, rays_d_host, n_rays, near, far, n_coarse,
                                    n_fine, params, out_rgb_host, out_depth_host, out_acc_host);
  if (s != NERF_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t R = n_rays;
  float* o = ctx->stage;
  float* d = o + R * 3;
  float* rgb = d + R * 3;
  float* dep = rgb + R * 3;
  float* acc = dep + R;
  NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(o, rays_o_host, R * 12, cudaMemcpyHostToDevice, st));
  NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(d, rays_d_host, R * 12, cudaMemcpyHostToDevice, st));
  s = nerf_render(ctx, o, d, R, near, far, n_coarse, n_fine, params, rgb, dep, acc, stream);
  if (s != NERF_OK) return s;
  NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(out_rgb_host, rgb, R * 12, cudaMemcpyDeviceToHost, st));
  NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(out_depth_host, dep, R * 4, cudaMemcpyDeviceToHost, st));
  NERF_CHECK_LAUNCH(ctx, cudaMemcpyAsync(out_acc_host, acc, R * 4, cudaMemcpyDeviceToHost, st));
  NERF_CHECK_LAUNCH(ctx, cudaStreamSynchronize(st));
  return NERF_OK;
}

nerf_status nerf_timing_enable(nerf_ctx* ctx, int enable) {
  if (!ctx) return fail(nullptr, NERF_ERR_INVALID_ARG, "ctx is NULL");
  if (enable && !ctx->ev) {
    ctx->ev = new cudaEvent_t[2 * kMaxTimed]();
    ctx->ev_kind = new int[kMaxTimed]();
    for (int i = 0; i < 2 * kMaxTimed; ++i) {
      cudaError_t e = cudaEventCreate(&ctx->ev[i]);
      if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaEventCreate");
    }
  }
  ctx->timing = enable != 0;
  ctx->n_timed = 0;
  return NERF_OK;
}

nerf_status nerf_timing_read_kinds(nerf_ctx* ctx, double* ms, int64_t* launches) {
  if (!ctx || !ms || !launches) return fail(ctx, NERF_ERR_INVALID_ARG, "NULL argument");
  for (int k = 0; k < NERF_TIMED_KINDS; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  for (int i = 0; i < ctx->n_timed; ++i) {
    cudaError_t e = cudaEventSynchronize(ctx->ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaEventSynchronize");
    float t = 0.0f;
    e = cudaEventElapsedTime(&t, ctx->ev[2 * i], ctx->ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaEventElapsedTime");
    ms[ctx->ev_kind[i]] += t;
    launches[ctx->ev_kind[i]] += 1;
  }
  ctx->n_timed = 0;
  return NERF_OK;
}

nerf_status nerf_timing_read(nerf_ctx* ctx, double* ms, int64_t* launches) {
  if (!ctx || !ms || !launches) return fail(ctx, NERF_ERR_INVALID_ARG, "NULL argument");
  double all_ms[NERF_TIMED_KINDS];
  int64_t all_n[NERF_TIMED_KINDS];
  nerf_status s = nerf_timing_read_kinds(ctx, all_ms, all_n);
  if (s != NERF_OK) return s;
  *ms = all_ms[NERF_TIMED_NETWORK];
  *launches = all_n[NERF_TIMED_NETWORK];
  return NERF_OK;
}

// ----------------------------------------------------------------- unit entry points

nerf_status nerf_test_stratified(const float* rays_o, const float* rays_d, int64_t n_rays,
                                 float near, float far, int n, uint64_t seed, int perturb,
                                 float* out_t, float* out_x, void* stream) {
  if (!rays_o || !rays_d || !out_t || n_rays <= 0 || n <= 0 || n > 65536 || !(near < far))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_stratified: bad argument");
  NERF_CHECK_LAUNCH(nullptr, launch_stratified(rays_o, rays_d, n_rays, near, far, n, sm64_mix(seed),
                                               perturb, out_t, out_x, (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_test_pe(const float* x, int64_t n, int L, float* out, void* stream) {
  if (!x || !out || n <= 0 || L < 1 || L > 16)
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_pe: bad argument");
  NERF_CHECK_LAUNCH(nullptr, launch_pe(x, n, L, out, (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_test_mlp(nerf_ctx* ctx, const void* weights, const float* x, const float* d,
                          int64_t n, float* out_raw, void* stream) {
  if (!ctx) return fail(nullptr, NERF_ERR_INVALID_ARG, "ctx is NULL");
  if (ctx->cfg.model != NERF_MODEL_MLP)
    return fail(ctx, NERF_ERR_INVALID_ARG, "nerf_test_mlp needs an MLP context");
  if (!weights || !x || !d || !out_raw || n <= 0 || n > ctx->cfg.max_rays)
    return fail(ctx, NERF_ERR_INVALID_ARG, "nerf_test_mlp: bad argument");
  if (ctx->cfg.precision == NERF_BF16 && !aligned16(weights))
    return fail(ctx, NERF_ERR_INVALID_ARG, "bf16 weight blobs must be 16-byte aligned");
  SampleSpec ss{};
  ss.mode = SAMPLES_GIVEN_X;
  ss.S = 1;
  ss.t = x;
  return run_network(ctx, weights, x, d, n, ss, out_raw, (cudaStream_t)stream);
}

nerf_status nerf_test_composite(const float* raw, const float* t, const float* rays_d,
                                int64_t n_rays, int S, float far, int last_delta_mode,
                                float march_step, int sigma_act, int white_bkgd, float* out_rgb,
                                float* out_depth, float* out_acc, float* out_weights,
                                void* stream) {
  if (!raw || !t || !rays_d || !out_rgb || !out_depth || !out_acc || n_rays <= 0 || S <= 0 ||
      S > 512 || last_delta_mode < 0 || last_delta_mode > 2 || !aligned16(raw))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_composite: bad argument");
  SampleSpec ss{};
  ss.mode = SAMPLES_GIVEN_T;
  ss.S = S;
  ss.t = t;
  CompositeSpec cs{last_delta_mode, far, march_step, sigma_act, white_bkgd};
  NERF_CHECK_LAUNCH(nullptr, launch_composite(raw, ss, rays_d, n_rays, cs, out_rgb, out_depth,
                                              out_acc, out_weights, (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_test_sample_pdf(const float* t_coarse, const float* weights, int64_t n_rays,
                                 int Nc, int Nf, uint64_t seed, int perturb, float* out_t_fine,
                                 int32_t* out_below, float* out_t_all, void* stream) {
  if (!t_coarse || !weights || n_rays <= 0 || Nc != 64 || Nf < 1 || Nf > 128 ||
      (!out_t_fine && !out_t_all))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_sample_pdf: bad argument (Nc must be 64, 1 <= Nf <= 128)");
  NERF_CHECK_LAUNCH(nullptr, launch_sample_pdf(t_coarse, weights, n_rays, Nc, Nf, sm64_mix(seed),
                                               perturb, out_t_fine, out_below, out_t_all,
                                               (cudaStream_t)stream));
  return NERF_OK;
}

}  // extern "C"

// ----------------------------------------------------------------- march unit entry points

extern "C" {

nerf_status nerf_test_march(const float* rays_o, const float* rays_d, int64_t n_rays, float near,
                            float step, int K, const uint32_t* occupancy, int32_t* out_count,
                            uint8_t* out_live, void* stream) {
  if (!rays_o || !rays_d || !occupancy || !out_count || n_rays <= 0 || K < 1 || K > 512 ||
      !(step > 0.0f))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_march: bad argument");
  NERF_CHECK_LAUNCH(nullptr, launch_march_mask(rays_o, rays_d, n_rays, near, step, K, occupancy,
                                               nullptr, out_count, out_live, (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_test_route_cells(const float* x, int64_t n, int32_t* out_cell,
                                  int32_t* out_cell_count, int32_t* out_cell_offset,
                                  int32_t* out_order, void* stream) {
  if (!x || !out_cell || !out_cell_count || !out_cell_offset || n <= 0 || n > (int64_t(1) << 30))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_route_cells: bad argument");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t* scratch = nullptr;   // cell fill counters [4096] + scan partials [2048]
  NERF_CHECK_LAUNCH(nullptr, cudaMallocAsync((void**)&scratch, (4096 + 2048) * sizeof(int32_t), st));
  unsigned* flag = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&flag, sizeof(unsigned), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(flag, 0, sizeof(unsigned), st);
  if (e == cudaSuccess)
    e = launch_route_points(x, n, out_cell, out_cell_count, out_cell_offset, out_order, scratch,
                            scratch + 4096, flag, st);
  cudaFreeAsync(scratch, st);
  if (flag) cudaFreeAsync(flag, st);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "nerf_test_route_cells");
  return NERF_OK;
}

nerf_status nerf_test_hash_encode(const float* x, int64_t n, const uint16_t* hash_table,
                                  float* out_feat, int32_t* out_rows, void* stream) {
  if (!x || !hash_table || !out_feat || n <= 0)
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_hash_encode: bad argument");
  NERF_CHECK_LAUNCH(nullptr, march_prepare(nullptr));
  NERF_CHECK_LAUNCH(nullptr, launch_hash_encode(x, n, hash_table, out_feat, out_rows,
                                                (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_hash_encode_backward(const float* x, int64_t n, const float* d_feat,
                                      float* grad_table, int deterministic, void* stream) {
  if (!x || !d_feat || !grad_table || n <= 0 || n > (int64_t(1) << 40))
    return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_hash_encode_backward: bad argument");
  NERF_CHECK_LAUNCH(nullptr, march_prepare(nullptr));
  NERF_CHECK_LAUNCH(nullptr, launch_hash_encode_backward(x, n, d_feat, grad_table, deterministic,
                                                         (cudaStream_t)stream));
  return NERF_OK;
}

nerf_status nerf_test_sh(const float* d, int64_t n, float* out, void* stream) {
  if (!d || !out || n <= 0) return fail(nullptr, NERF_ERR_INVALID_ARG, "nerf_test_sh: bad argument");
  NERF_CHECK_LAUNCH(nullptr, launch_sh(d, n, out, (cudaStream_t)stream));
  return NERF_OK;
}

}  // extern "C"

namespace nerfb {
// Records a context-free error message for nerf_last_error(NULL).
void set_global_error(const char* msg) { g_create_error = msg; }
}  // namespace nerfb

extern "C" nerf_status nerf_test_bounded_wait(uint32_t timeout_us, uint32_t* out_flag,
                                              uint32_t* out_waited_us, void* stream) {
  if (!out_flag || timeout_us < 1 || timeout_us > 2000000) {
    nerfb::set_global_error("nerf_test_bounded_wait: bad argument");
    return NERF_ERR_INVALID_ARG;
  }
  cudaError_t e = nerfb::launch_bounded_wait_probe(timeout_us, out_flag, out_waited_us,
                                                   (cudaStream_t)stream);
  return e == cudaSuccess ? NERF_OK : NERF_ERR_CUDA;
}
