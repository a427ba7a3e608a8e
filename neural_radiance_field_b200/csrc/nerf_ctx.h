// The context behind the opaque nerf_ctx handle.
#pragma once

#include <string>

#include "nerf_internal.cuh"
#include "nerf_march.cuh"

struct nerf_ctx {
  nerf_config cfg{};
  int device = -1;
  std::string err;
  int64_t n_params = 0;
  nerfb::PackedFp32 plan{};

  // workspace (device), sized at create for max_rays x max_samples
  float* packed = nullptr;     // fp32 packed weights of the network being run
  float* dir_bias = nullptr;   // [max_rays][W/2]
  float* raw = nullptr;        // [max_rays * max_samples][4]
  float* t_all = nullptr;      // [max_rays][max_samples]
  float* stage = nullptr;      // host-path staging: o, d, rgb [R][3]; depth, acc [R]
  unsigned* d_flag = nullptr;  // device error flag
  // training path (nerf_loss_grad), allocated on its first call
  float* tr_save = nullptr;    // [max_rays * S][64 + (D+1) W + W/2] activation store
  float* tr_draw = nullptr;    // [max_rays * S][4] d raw
  float* tr_tmp = nullptr;     // backward scratch
  float* tr_loss = nullptr;    // [2 max_rays] per-ray loss terms
  float* tr_bsplit = nullptr;  // split weights of one tensor-core row GEMM (TRAIN_BSPLIT floats)
  float* fw_save = nullptr;    // precision TF32: [fw_rows][64 + 2 W + W/2] layer outputs of a sub-batch
  int64_t fw_rows = 0;

  // kernel timing (nerf_timing_enable / nerf_timing_read / nerf_timing_read_kinds)
  bool timing = false;
  int n_timed = 0;
  cudaEvent_t* ev = nullptr;   // 2 * kMaxTimed events, created on first enable
  int* ev_kind = nullptr;      // kernel class of each event pair
  nerfb::KernelTimer timer();

  // march models (KILONERF, HASHGRID): ray chunks and their live-entry workspace
  int64_t chunk_rays = 0;
  nerfb::MarchWs mws{};

  // tensor-core (bf16) path
  bool tc_enabled = false;
  void* tc_weights = nullptr;  // packed bf16 operand images + fp32 epilogue vectors
  int num_sms = 0;
};

namespace nerfb {
constexpr int kMaxTimed = 4096;
}  // namespace nerfb

inline nerfb::KernelTimer nerf_ctx::timer() {
  nerfb::KernelTimer t;
  if (timing && ev) {
    t.ev = ev;
    t.kind = ev_kind;
    t.n = &n_timed;
    t.cap = nerfb::kMaxTimed;
  }
  return t;
}

namespace nerfb {
cudaError_t tc_alloc(nerf_ctx* ctx);
void tc_free(nerf_ctx* ctx);
cudaError_t tc_pack(nerf_ctx* ctx, const void* blob, cudaStream_t st);
cudaError_t launch_bounded_wait_probe(uint32_t timeout_us, uint32_t* flag, uint32_t* waited_us,
                                      cudaStream_t st);
cudaError_t tc_run(nerf_ctx* ctx, const float* o, const float* d, int64_t R,
                   const SampleSpec& ss, float* raw, cudaStream_t st);
}  // namespace nerfb
