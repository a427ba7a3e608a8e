/*
 * nerf.h - C ABI of the B200 forward NeRF renderer (libnerf.so, sm_100a).
 *
 * The library renders batches of rays with the method of "Spatial Intelligence -
 * Part 1: NeRF" (halannhile.github.io): stratified samples on [near, far],
 * positional encoding gamma(x), gamma(d), the scene MLP F_theta(x, d) -> (c, sigma),
 * alpha compositing with T_i = exp(-sum_{j<i} sigma_j delta_j), then inverse-CDF
 * resampling and a fine pass (Sections 1.3, 1.4 and 2.2-2.6 of that page). Two
 * alternative scene functions march a 128^3 occupancy grid instead: a 16^3 grid
 * of tiny MLPs (the KiloNeRF page, abstract) and a 3D multiresolution hash grid
 * with a small MLP (the Instant-NGP notebook, "A shared toolkit" and Experiment 1).
 *
 * Conventions for every entry point:
 *  - Pointers named *_host are host memory; every other buffer pointer is device
 *    memory on the current CUDA device, owned by the caller, and must stay valid
 *    until the work enqueued on `stream` has completed.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls only
 *    enqueue work; they never synchronise, except nerf_render_host and
 *    nerf_sync_status, which say so.
 *  - Arrays are dense, row-major, fp32 unless stated; [R][3] means R rows of 3.
 *  - Argument errors are reported synchronously (NERF_ERR_INVALID_ARG) before any
 *    work is enqueued. Launch errors come back as NERF_ERR_CUDA. Errors that the
 *    kernels detect set a device flag that nerf_sync_status reports.
 *  - A context is not thread-safe; use one context per host thread.
 *  - There is no CPU implementation behind this ABI: without a usable CUDA
 *    device every call that needs one returns NERF_ERR_CUDA.
 */
#ifndef NERF_B200_H
#define NERF_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NERF_API __attribute__((visibility("default")))
#else
#define NERF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct nerf_ctx nerf_ctx;

typedef enum {
  NERF_OK = 0,
  NERF_ERR_INVALID_ARG = 1,   /* bad pointer, size or mode; nothing was enqueued */
  NERF_ERR_CUDA = 2,          /* CUDA runtime or launch error */
  NERF_ERR_UNSUPPORTED = 3,   /* valid request that this library does not implement */
  NERF_ERR_OOM = 4,           /* workspace allocation failed at create time */
  NERF_ERR_TIMEOUT = 5,       /* a bounded device wait gave up */
  NERF_ERR_DEVICE_FLAG = 6    /* a kernel reported an out-of-range input */
} nerf_status;

enum { NERF_MODEL_MLP = 0, NERF_MODEL_KILONERF = 1, NERF_MODEL_HASHGRID = 2 };
enum { NERF_SIGMA_RELU = 0, NERF_SIGMA_SOFTPLUS = 1 };
enum { NERF_FP32 = 0, NERF_BF16 = 1, NERF_TF32 = 2 };
/* Length of the last interval of a ray: 1e10 as in the NeRF page's volume_render
 * (Section 2.5), or up to `far` (the closed form of T(t) on [t_n, t_f]). */
enum { NERF_LAST_1E10 = 0, NERF_LAST_TO_FAR = 1 };

/* Fixed at create time. For NERF_MODEL_MLP the network is the NeRF page's
 * F_theta (Section 2.4): D layers of width W with ReLU, gamma(x) concatenated
 * after layer `skip` (skip < 0: none), sigma head Linear(W,1), feature layer
 * Linear(W,W), direction layer Linear(W + 3(1+2 L_dir), W/2) + ReLU, rgb head
 * Linear(W/2, 3). Supported with precision FP32: W in {64, 128, 256}, D in
 * 1..8, skip = -1 or 0 <= skip <= D-2 (the compact, scene-specialised shapes
 * of the NAS-NeRF page; the CUDA-core kernel is compiled per width), with
 * L_pos = 10, L_dir = 4. precision BF16 selects the tensor-core path, built
 * for the page's (W=256, D=8, skip=4) network only (NERF_ERR_UNSUPPORTED
 * otherwise); sigma_act and white_bkgd are applied in compositing.
 * precision TF32 takes the fp32 blobs and evaluates the same network layer by
 * layer on the tensor cores: every operand v is split into hi = v rounded to
 * tf32 and lo = v - hi, each product accumulates hi*hi + hi*lo + lo*hi in
 * fp32 (the dropped lo*lo term is below 2^-22 of it), so results agree with
 * FP32 to fp32 rounding level; W in {128, 256}, any D and skip as for FP32
 * (NERF_ERR_UNSUPPORTED for W = 64). The context then holds an activation
 * store of up to 2^20 samples (64 + 2.5 W floats each) for the layer outputs.
 * KILONERF ignores D..precision; HASHGRID ignores D..sigma_act and takes
 * precision FP32 (the whole scene function in fp32 on the CUDA cores) or BF16
 * (the encoding and the sigma / rgb heads in fp32, the four hidden layers on the
 * tensor cores with bf16 weights and activations and fp32 accumulation;
 * NERF_ERR_INVALID_ARG for any other value). max_rays and max_samples size
 * the context's workspace (max_samples >= n_coarse + n_fine of any render). */
typedef struct {
  int model;
  int D, W, skip, L_pos, L_dir;
  int sigma_act;
  int precision;
  int last_delta_mode;
  int white_bkgd;
  int64_t max_rays;
  int max_samples;
} nerf_config;

/* Per-render inputs (device pointers unless stated).
 *  coarse_w, fine_w  NERF_MODEL_MLP: flat parameter blobs, fp32 (precision FP32)
 *                    or bf16 (precision BF16). Layer order: pts0..pts{D-1},
 *                    sigma, feature, dir, rgb; each layer is its weight matrix
 *                    [N_out][K_in] row-major followed by its bias [N_out].
 *                    fine_w may be NULL when n_fine == 0.
 *  occupancy         march models: 128^3 occupancy bits over [-1.5, 1.5)^3,
 *                    uint32[65536]; voxel (ix,iy,iz) is bit (i & 31) of word
 *                    i >> 5, i = (ix*128 + iy)*128 + iz.
 *  cell_w            KILONERF: fp32 [4096][3317] per-cell parameters, cell id
 *                    (cx*16+cy)*16+cz; per cell: W1[32][63] b1[32] W2[32][32]
 *                    b2[32] w_sigma[32] b_sigma[1] Wc[3][59] bc[3].
 *  hash_table        HASHGRID: fp16 [6101902][2], all 16 levels concatenated.
 *  hash_mlp          HASHGRID: fp32 blob d0[64][32] b, d1[64][64] b, sigma[1][64] b,
 *                    c0[64][80] b, c1[64][64] b, rgb[3][64] b.
 *  march_step        march models: t_k = near + k * march_step, k < n_coarse.
 *  ert_T             march models: stop a ray before the first occupied sample
 *                    with transmittance below ert_T (0 disables).
 *  seed, perturb     jitter of the stratified samples and the inverse-CDF draws
 *                    (counter-based SplitMix64); perturb = 0 uses u = 0.5 for the
 *                    jitter and evenly spaced draws (k + 0.5) / n_fine.
 */
typedef struct {
  const void* coarse_w;
  const void* fine_w;
  const uint32_t* occupancy;
  const float* cell_w;
  const uint16_t* hash_table;
  const float* hash_mlp;
  float march_step;
  float ert_T;
  uint64_t seed;
  int perturb;
} nerf_params;

/* Create a context: validates `cfg`, allocates the workspace on the current
 * device (NERF_ERR_OOM on failure). *out is NULL on error. */
NERF_API nerf_status nerf_create(const nerf_config* cfg, nerf_ctx** out);

/* Free the workspace (synchronises the device first). NULL is a no-op. */
NERF_API nerf_status nerf_destroy(nerf_ctx* ctx);

/* Message of the last error on this context (or of the last failed create when
 * ctx is NULL). Owned by the library; valid until the next call. */
NERF_API const char* nerf_last_error(const nerf_ctx* ctx);

/* Waits for `stream`, then reports launch errors and the device error flag
 * (clearing it): NERF_OK, NERF_ERR_CUDA, NERF_ERR_TIMEOUT or
 * NERF_ERR_DEVICE_FLAG. */
NERF_API nerf_status nerf_sync_status(nerf_ctx* ctx, void* stream);

/* Pinhole rays for an H x W image (NeRF page, Section 2.2, get_rays):
 * camera-space direction ((i - W/2)/focal, -(j - H/2)/focal, -1) rotated by the
 * upper 3x3 of c2w (not normalised), origin = c2w translation. Pixel (j, i)
 * is row j*W + i. c2w_host: 12 floats, row-major [3][4], read during the call.
 * rays_o, rays_d: [H*W][3]. Evaluated in IEEE fp32 without contraction. */
NERF_API nerf_status nerf_raygen(int H, int W, float focal, const float* c2w_host,
                        float* rays_o, float* rays_d, void* stream);

/* The rays of n_cams cameras in one buffer, for a multi-view sweep (NeRF page,
 * Section 3: a novel-view video of 24 frames circling the scene, every frame a
 * new camera pose through the same network). Camera c's pixel (i, j) becomes
 * ray c*H*W + j*W + i, and each value is bit-identical to what nerf_raygen
 * writes for that camera alone. c2w_host: [n_cams][3][4] row-major, host
 * memory, read before the call returns. rays_o, rays_d: device
 * [n_cams*H*W][3] fp32, caller-owned. Enqueued on `stream` (one launch per 32
 * cameras); does not synchronise. A whole sweep then goes through one
 * nerf_render call whose max_rays covers n_cams*H*W.
 * Errors: NERF_ERR_INVALID_ARG (H, W, n_cams <= 0, focal <= 0, NULL pointer,
 * more than 2^40 rays), NERF_ERR_CUDA on a launch failure. */
NERF_API nerf_status nerf_raygen_batch(int H, int W, float focal, int n_cams,
                                       const float* c2w_host, float* rays_o, float* rays_d,
                                       void* stream);

/* Render n_rays rays (NeRF page, Section 2.6 render_rays):
 *  NERF_MODEL_MLP: n_coarse stratified samples on [near, far] through the coarse
 *    network; if n_fine > 0, n_fine inverse-CDF draws from the coarse weights of
 *    the interior samples, the sorted union of n_coarse + n_fine positions
 *    through the fine network; the output is the last pass. n_coarse must be 64
 *    when n_fine > 0; n_coarse + n_fine <= max_samples.
 *  march models: n_coarse fixed-step candidates (march_step), only occupied ones
 *    evaluated; n_fine must be 0.
 * Outputs: out_rgb [n_rays][3], out_depth [n_rays] (sum of w_i t_i, in t units),
 * out_acc [n_rays] (sum of w_i). rays_o, rays_d: [n_rays][3]. 0 < n_rays <=
 * max_rays, near < far. */
NERF_API nerf_status nerf_render(nerf_ctx* ctx, const float* rays_o, const float* rays_d,
                        int64_t n_rays, float near, float far, int n_coarse, int n_fine,
                        const nerf_params* params, float* out_rgb, float* out_depth,
                        float* out_acc, void* stream);

/* Intermediates of one NERF_MODEL_MLP render, for checking every stage of the
 * path on its own inputs. All pointers are device memory owned by the caller;
 * any may be NULL (not written). R = n_rays, Nc = n_coarse, Nf = n_fine.
 *  raw_coarse [R][Nc][4]      the coarse network's raw (r, g, b, sigma)
 *  w_coarse   [R][Nc]         the coarse compositing weights w_i = T_i alpha_i
 *                             (with n_fine > 0, those the fine positions were
 *                             drawn from)
 *  t_fine     [R][Nf]         the inverse-CDF draws, in draw order
 *  below      [R][Nf] int32   the bin of each draw (searchsorted - 1, clamped)
 *  t_all      [R][Nc+Nf]      the sorted union of coarse and fine positions
 *  raw_fine   [R][Nc+Nf][4]   the fine network's raw outputs at t_all
 * The fine-pass fields are ignored when n_fine == 0. */
typedef struct {
  float* raw_coarse;
  float* w_coarse;
  float* t_fine;
  int32_t* below;
  float* t_all;
  float* raw_fine;
} nerf_trace;

/* nerf_render (NeRF page, Section 2.6 render_rays) of a NERF_MODEL_MLP context
 * that also copies the render's own intermediates into `trace` (coarse network
 * output and weights, Section 2.5; the sample_pdf draws and bins, Section 2.6;
 * the sorted union and the fine network output). The kernels, launch shapes
 * and outputs are those of nerf_render; only device-to-device copies of the
 * workspace and the resampler's optional stores are added. Same argument
 * rules and errors as nerf_render; NERF_ERR_UNSUPPORTED for the march models;
 * NERF_ERR_INVALID_ARG if trace is NULL. Enqueued on `stream`. */
NERF_API nerf_status nerf_render_trace(nerf_ctx* ctx, const float* rays_o, const float* rays_d,
                                       int64_t n_rays, float near, float far, int n_coarse,
                                       int n_fine, const nerf_params* params, float* out_rgb,
                                       float* out_depth, float* out_acc, const nerf_trace* trace,
                                       void* stream);

/* Loss and parameter gradients of one training step (NeRF page, "7. Training
 * loop"): the rays are rendered as nerf_render does (coarse pass; with n_fine >
 * 0 the fine pass on the sorted union of positions drawn from the coarse
 * weights, which are detached: "6. Hierarchical sampling"), and
 *   loss = mse(rgb_coarse, target) + mse(rgb_fine, target)
 * (each mse the mean over n_rays x 3 values; without a fine pass only the
 * coarse term). Writes *out_loss and the gradients of the loss with respect to
 * every parameter of the coarse and fine networks.
 * ctx: NERF_MODEL_MLP with precision FP32 or TF32 (NERF_ERR_UNSUPPORTED otherwise).
 * target_rgb: device [n_rays][3] fp32. out_loss: device, one float.
 * grad_coarse, grad_fine: device fp32 buffers of the network's parameter count,
 * laid out like the weight blobs (per Linear: W row-major [N][K], then b);
 * overwritten. grad_fine may be NULL when n_fine == 0. n_coarse >= 2 and
 * n_coarse + n_fine <= min(max_samples, 256); the fine pass needs n_coarse = 64.
 * The first call allocates the training workspace on the current device, about
 * max_rays x min(max_samples, 256) x (64 + (D+1) W + 2.5 W + 4) floats
 * (NERF_ERR_OOM if that fails). The gradients are summed with fp32 atomics, so
 * their last bits vary between runs. Enqueued on `stream`; does not synchronise. */
NERF_API nerf_status nerf_loss_grad(nerf_ctx* ctx, const float* rays_o, const float* rays_d,
                                    int64_t n_rays, float near, float far, int n_coarse,
                                    int n_fine, const nerf_params* params,
                                    const float* target_rgb, float* out_loss, float* grad_coarse,
                                    float* grad_fine, void* stream);

/* nerf_render (NeRF page, Section 2.6 render_rays) with HOST ray and output
 * buffers (pinned memory recommended): copies the rays into the context's
 * staging buffers, renders, copies the results back and synchronises `stream`
 * before returning. Same argument rules and errors as nerf_render; the host
 * buffers stay the caller's. */
NERF_API nerf_status nerf_render_host(nerf_ctx* ctx, const float* rays_o_host, const float* rays_d_host,
                             int64_t n_rays, float near, float far, int n_coarse, int n_fine,
                             const nerf_params* params, float* out_rgb_host,
                             float* out_depth_host, float* out_acc_host, void* stream);

/* Device timing of the library's kernels, for benchmarks. While enabled, the
 * launches of every kernel class below that nerf_render / nerf_test_mlp issue
 * are bracketed by CUDA events recorded on the caller's stream (at most 4096
 * event pairs between reads; further launches are not timed). The classes:
 *   NETWORK          the scene-network kernel (NeRF MLP; march models: the
 *                    hash-grid or KiloNeRF scene function)
 *   COMPOSITE        compositing of the last NeRF pass (Section 2.5)
 *   RESAMPLE         coarse compositing + inverse-CDF draws + sorted merge
 *                    (Section 2.6)
 *   DIR_BIAS         the per-ray direction-encoding bias of the direction layer
 *   MARCH_MASK       the occupancy test of every march candidate
 *   MARCH_COMPACT    the scan and compaction of the live candidates
 *   ROUTER           KiloNeRF cell routing (histogram, scan, scatter, work items)
 *   MARCH_COMPOSITE  march compositing with early termination
 * nerf_timing_read waits for the recorded events and returns the summed time
 * (milliseconds) and launch count of the NETWORK class; nerf_timing_read_kinds
 * returns every class (arrays of NERF_TIMED_KINDS, indexed by the enum). Both
 * start a new count. */
enum {
  NERF_TIMED_NETWORK = 0,
  NERF_TIMED_COMPOSITE = 1,
  NERF_TIMED_RESAMPLE = 2,
  NERF_TIMED_DIR_BIAS = 3,
  NERF_TIMED_MARCH_MASK = 4,
  NERF_TIMED_MARCH_COMPACT = 5,
  NERF_TIMED_ROUTER = 6,
  NERF_TIMED_MARCH_COMPOSITE = 7,
  NERF_TIMED_KINDS = 8
};
NERF_API nerf_status nerf_timing_enable(nerf_ctx* ctx, int enable);
NERF_API nerf_status nerf_timing_read(nerf_ctx* ctx, double* ms, int64_t* launches);
NERF_API nerf_status nerf_timing_read_kinds(nerf_ctx* ctx, double* ms, int64_t* launches);

/* ---------------------------------------------------------------------------
 * Unit entry points: one step of the path each, same conventions as above.
 * ------------------------------------------------------------------------- */

/* Stratified samples (NeRF page, Section 1.4.2): t_i = near + (i + u_i) * (far -
 * near)/n in fp32 (step = (far-near)/n, s = i + u, t = near + s*step, each op
 * rounded) and points x = o + t d (fp32, no contraction). out_t [R][n],
 * out_x [R][n][3] (may be NULL). */
NERF_API nerf_status nerf_test_stratified(const float* rays_o, const float* rays_d, int64_t n_rays,
                                 float near, float far, int n, uint64_t seed, int perturb,
                                 float* out_t, float* out_x, void* stream);

/* Positional encoding (NeRF page, Section 1.4.1): [x, sin(2^k pi x_c),
 * cos(2^k pi x_c)], sin and cos blocks coordinate-major. x [P][3], out [P][3+6L]. */
NERF_API nerf_status nerf_test_pe(const float* x, int64_t n, int L, float* out, void* stream);

/* The context's scene network F_theta (NeRF page, Section 2.4) on arbitrary
 * points x [P][3] seen from directions d [P][3] (normalised inside): raw output
 * [P][4] = (r, g, b, sigma) before activations. NERF_MODEL_MLP contexts only;
 * P <= max_rays (NERF_ERR_INVALID_ARG otherwise). */
NERF_API nerf_status nerf_test_mlp(nerf_ctx* ctx, const void* weights, const float* x, const float* d,
                          int64_t n, float* out_raw, void* stream);

/* Compositing (NeRF page, Sections 1.3 and 2.5) of raw network outputs
 * raw [R][S][4] at positions t [R][S] along rays with directions d [R][3]:
 * delta_i = (t_{i+1} - t_i) ||d||, last interval per last_delta_mode (march_step
 * * ||d|| when last_delta_mode == 2), sigma = act(raw), c = sigmoid(raw).
 * Outputs rgb [R][3], depth [R], acc [R], weights [R][S] (may be NULL). */
NERF_API nerf_status nerf_test_composite(const float* raw, const float* t, const float* rays_d,
                                int64_t n_rays, int S, float far, int last_delta_mode,
                                float march_step, int sigma_act, int white_bkgd,
                                float* out_rgb, float* out_depth, float* out_acc,
                                float* out_weights, void* stream);

/* Inverse-CDF resampling and merge (NeRF page, Section 2.6 sample_pdf and the
 * sorted union): bins are the fp32 midpoints of t_c [R][Nc], the pdf is
 * weights[R][1..Nc-2] + 1e-5, draws u = m 2^-24 (seed, stream 1) or (k+0.5)/Nf.
 * The CDF is exact: q_i = floor(fl32(w_i + 1e-5) 2^32), bin = #{k : C_k 2^24 <=
 * m C_total}. out_t_fine [R][Nf] (draw order), out_below [R][Nf] int32 (bin
 * index, may be NULL), out_t_all [R][Nc+Nf] ascending. Nc = 64, Nf <= 128. */
NERF_API nerf_status nerf_test_sample_pdf(const float* t_coarse, const float* weights, int64_t n_rays,
                                 int Nc, int Nf, uint64_t seed, int perturb, float* out_t_fine,
                                 int32_t* out_below, float* out_t_all, void* stream);

/* Occupancy march: empty-space skipping over the 128^3 grid of nerf_params (the
 * Instant-NGP notebook, "Connection to the broader theory"; the NeRF page,
 * Section 1.4, on uniform sampling spending most of its work on empty space):
 * candidates t_k = near + k * step (fp32, k < K <= 512), points x = o + t_k d
 * (fp32, no contraction); a point is live when it lies in [-1.5, 1.5)^3 and its
 * voxel (the exact floor of (x + 1.5) * 128 / 3 per axis) is occupied.
 * out_count [R] int32: live candidates per ray; out_live [R][K] uint8 (may be
 * NULL): 1 where candidate k is live. */
NERF_API nerf_status nerf_test_march(const float* rays_o, const float* rays_d, int64_t n_rays,
                                     float near, float step, int K, const uint32_t* occupancy,
                                     int32_t* out_count, uint8_t* out_live, void* stream);

/* KiloNeRF routing of points x [P][3] (inside [-1.5, 1.5)^3): out_cell [P]
 * int32 = (cx*16 + cy)*16 + cz with c = voxel >> 3; out_cell_count [4096] and
 * out_cell_offset [4097] int32 (exclusive scan); out_order [P] int32 (may be
 * NULL): point indices grouped by cell (cell-major; order inside a cell
 * unspecified). */
NERF_API nerf_status nerf_test_route_cells(const float* x, int64_t n, int32_t* out_cell,
                                           int32_t* out_cell_count, int32_t* out_cell_offset,
                                           int32_t* out_order, void* stream);

/* Hash-grid encoding (Instant-NGP notebook, HashGrid2D.encode, extended to 3D):
 * 16 levels N_l = round(16 b^l), b = (2048/16)^(1/15); T = 2^19 entries per level,
 * 2 fp16 features per entry (table: nerf_params.hash_table layout); direct
 * index (ix*(N+1)+iy)*(N+1)+iz while (N+1)^3 <= T, else (ix XOR iy*2654435761
 * XOR iz*805459861) mod T; trilinear weights of c = fl(fl((x + 1.5)/3) * N).
 * x [P][3]; out_feat [P][32] (level-major); out_rows [P][16][8] int32 (may be
 * NULL): global table row of every corner (dx, dy, dz loop order). */
NERF_API nerf_status nerf_test_hash_encode(const float* x, int64_t n, const uint16_t* hash_table,
                                           float* out_feat, int32_t* out_rows, void* stream);

/* Backward of the hash-grid encoding above, the scatter-add that trains the
 * grid (Instant-NGP notebook, Experiment 1, in 3D): for every point and level,
 * d_feat[point][2 l + f] * (corner weight) is added to grad_table[row][f] for
 * each of the level's 8 corner rows (the same rows and trilinear weights as
 * nerf_test_hash_encode). x [n][3] and d_feat [n][32] fp32 device;
 * grad_table: device fp32 [6,101,902][2], ACCUMULATED into (zero it first).
 * deterministic = 0: fp32 atomics, whose summation order (hence the last bits)
 * varies from run to run. deterministic = 1: every term is rounded to a
 * multiple of 2^-E, E = 62 - ceil(log2(n * max|d_feat|)), and summed as int64
 * (associative, so bit-identical across runs; no sum can overflow since a
 * point's 8 weights per level add to 1), then converted and added; this mode
 * allocates 97.6 MB of stream-ordered scratch (cudaMallocAsync) per call.
 * Enqueued on `stream`; does not synchronise. Errors: NERF_ERR_INVALID_ARG
 * (NULL pointer, n <= 0), NERF_ERR_CUDA. */
NERF_API nerf_status nerf_hash_encode_backward(const float* x, int64_t n, const float* d_feat,
                                               float* grad_table, int deterministic,
                                               void* stream);

/* Real spherical harmonics of bands 0..3 (16 values, index l*l + l + m, no
 * Condon-Shortley phase) of the unit vectors d/|d|: the hash-grid MLP's view
 * encoding. The pages do not describe it; degree-4 real SH with the textbook
 * normalisation is this library's reading of the hash workload's colour input.
 * d [P][3], out [P][16]. */
NERF_API nerf_status nerf_test_sh(const float* d, int64_t n, float* out, void* stream);

/* Failure detection of the device waits. Every wait of the library's kernels on
 * a barrier (weight arrival, MMA completion, epilogue hand-off) gives up after a
 * bound (2 s), sets NERF_ERR_TIMEOUT's flag bit and lets the kernel return, so
 * the context stays usable and nerf_sync_status reports the timeout. This entry
 * point runs that same bounded wait, with timeout_us (1..2,000,000), on a
 * barrier that nothing ever completes: out_flag (device uint32, caller-zeroed)
 * receives the flag bit (2), out_waited_us (device uint32, may be NULL) the
 * time waited in microseconds. */
NERF_API nerf_status nerf_test_bounded_wait(uint32_t timeout_us, uint32_t* out_flag,
                                            uint32_t* out_waited_us, void* stream);

/* ---------------------------------------------------------------------------
 * Entry point that allocates no device memory. The pages have no counterpart;
 * it exists for callers that cannot call cudaMalloc, such as a host framework
 * that owns all device memory through its own allocator, or a render loop held
 * to a fixed memory budget.
 *
 * Occupancy-march compaction (the live-candidate test of nerf_test_march) that
 * writes, for n_rays <= 1,048,576 rays: out_offsets [n_rays + 1] int32, the
 * exclusive prefix sum of the per-ray live counts (out_offsets[n_rays] = total
 * live), and out_live [n_rays * K] uint32 (caller-sized for the worst case),
 * whose first out_offsets[n_rays] entries are (ray << 9) | k in ray-major, then
 * k-ascending order. out_live is also used as temporary storage during the call.
 * Its only scratch is a static 4 KB device array compiled into the library (one
 * int32 per 1024 rays); every device that loads the library holds it until the
 * process exits. The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress); make that first call before any stream
 * capture. All calls share the array and it keeps the last call's contents:
 * calls whose work overlaps on the GPU (different streams) race on it.
 * n_rays above the limit returns NERF_ERR_INVALID_ARG with a message in
 * nerf_last_error(NULL). */
NERF_API nerf_status nerf_march_compact_noalloc(const float* rays_o, const float* rays_d,
                                                int64_t n_rays, float near, float step, int K,
                                                const uint32_t* occupancy, int32_t* out_offsets,
                                                uint32_t* out_live, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NERF_B200_H */
