// bf16 tensor-core evaluation of the NeRF scene MLP (NeRF page, Section 2.4) on
// sm_100a: tcgen05.mma with fp32 accumulators in tensor memory, weights streamed
// by the bulk-copy engine, activations kept on chip for the whole network.
//
// Persistent kernel, one CTA per SM, 18 warps:
//   warp 0       issues the MMAs (one elected thread) and owns the TMEM allocation
//   warp 1       streams the packed weights into a 4-slot shared-memory ring
//   warps 2-9    epilogue of tile A: warp w drains TMEM lane quarter (w % 4) of
//                column half ((w - 2) / 4) % 2, i.e. thread = (row, half)
//   warps 10-17  epilogue of tile B, same split
// A CTA works on pairs of 128-row tiles. Every weight chunk that lands in the
// ring feeds both tiles before its slot is refilled, so each weight byte read
// from L2 serves 256 rows. Per layer the accumulators of both tiles (2 x 256
// fp32 columns = all 512 TMEM columns) are drained by the epilogue warps, which
// add the bias, apply ReLU, round to bf16 and write the next layer's A operand
// back into shared memory. Two warps per lane quarter keep twice as many TMEM
// loads in flight as one would; the drain is latency-bound, not bandwidth-bound.
//
// Shared memory (231,680 B): act[2] = per tile 128 rows x 320 bf16 holding
// [h (256) | gamma(x) (63) | 0], so the skip layer reads columns 0..319 and the
// first layer columns 256..319; ring[4] = weight chunks of K = 32 columns;
// 2 KB of per-layer epilogue vectors; barriers.
// Operands use the no-swizzle K-major core-matrix layout: element (r, k) of a
// block of R rows sits at (k/8)*R*16 + (r/8)*128 + (r%8)*16 + (k%8)*2 bytes.
#include "nerf_ctx.h"

namespace nerfb {

namespace {

constexpr int TM = 128;
constexpr int ACT_K = 320;
constexpr int ACT_BYTES = TM * ACT_K * 2;           // 81920
constexpr int CHUNK_K = 32;
constexpr int NSTAGE = 4;
constexpr int RING_BYTES = 256 * CHUNK_K * 2;       // 16384 per slot
constexpr int NLAYER = 10;                          // pts0..pts7, feature, dir
constexpr int EPI_THREADS = 512;                    // 16 epilogue warps
constexpr int TILE_THREADS = 256;                   // epilogue threads per tile
constexpr int NTHREADS = 64 + EPI_THREADS;
constexpr int VEC_BYTES = 2 * 256 * 4;              // staged epilogue vectors
constexpr size_t SMEM_BYTES = 2 * ACT_BYTES + NSTAGE * RING_BYTES + VEC_BYTES + 256;


// Packed weight stream (bf16 chunks in consumption order) and fp32 vectors.
struct TcLayout {
  int64_t chunk_off[80];     // byte offset of every chunk in the stream
  int chunk_bytes[80];
  int n_chunks;
  int64_t stream_bytes;
  int64_t vec_off;           // byte offset of the fp32 vectors
  // fp32 vector block (element offsets inside it)
  int bias[NLAYER];          // 256 (128 for dir) each
  int w_sigma, b_sigma, w_rgb, b_rgb;
  int vec_count;
};

TcLayout make_layout() {
  TcLayout L{};
  const int kch[NLAYER] = {2, 8, 8, 8, 8, 10, 8, 8, 8, 8};
  const int nout[NLAYER] = {256, 256, 256, 256, 256, 256, 256, 256, 256, 128};
  int64_t off = 0;
  int q = 0;
  for (int l = 0; l < NLAYER; ++l)
    for (int c = 0; c < kch[l]; ++c) {
      L.chunk_off[q] = off;
      L.chunk_bytes[q] = nout[l] * CHUNK_K * 2;
      off += L.chunk_bytes[q];
      ++q;
    }
  L.n_chunks = q;
  L.stream_bytes = off;
  L.vec_off = (off + 255) & ~int64_t(255);
  int v = 0;
  for (int l = 0; l < NLAYER; ++l) { L.bias[l] = v; v += 256; }
  L.w_sigma = v; v += 256;
  L.b_sigma = v; v += 4;
  L.w_rgb = v; v += 3 * 128;
  L.b_rgb = v; v += 4;
  L.vec_count = v;
  return L;
}

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

struct Ctl {
  volatile int* abort;
  unsigned* flag;
  uint64_t limit_ns;   // wait bound (2 s in the kernels)
};
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Bounded wait: gives up after ctl.limit_ns, raises the timeout flag and the CTA abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const Ctl& ctl) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (*ctl.abort) return false;
    if (globaltimer() - t0 > ctl.limit_ns) {
      atomicOr(ctl.flag, FLAG_TIMEOUT);
      *ctl.abort = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor, no swizzle, K-major core matrices.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;                    // descriptor version for sm_100
  return d;                                  // base offset 0, swizzle none
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// Two fp32 -> packed bf16x2 with ReLU (lo = first element in memory order).
__device__ __forceinline__ uint32_t pack_relu(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.relu.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint32_t pack_plain(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d) : "memory");
}

// Byte offset of 8 consecutive K elements (k0 % 8 == 0) of row r in a 128-row block.
__device__ __forceinline__ uint32_t act_off(int r, int k0) {
  return (uint32_t)((k0 >> 3) * (TM * 16) + (r >> 3) * 128 + (r & 7) * 16);
}

struct Params {
  const uint8_t* stream;     // packed bf16 chunks
  const float* vec;          // fp32 vectors
  TcLayout lay;
  const float* dir_bias;     // [R][128]
  const float* o;
  const float* d;
  int64_t R;
  SampleSpec ss;
  float* raw;                // [R*S][4]
  unsigned* flag;
  int64_t n_pairs;
};

// Issue a 32-column TMEM load; the registers are valid after tmem_wait32.
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Wait for outstanding TMEM loads; the registers are threaded through the asm
// so that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait32(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Named barriers: 1 = all 512 epilogue threads, 2 + g = the 256 threads of tile g.
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier over all epilogue threads that returns whether any passed true.
__device__ __forceinline__ bool epilogue_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 512, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// One 32-column block of a hidden layer: bias, activation, bf16, store to the
// next layer's A operand; on the last trunk layer also accumulates sigma. Works
// 8 columns at a time so that only the loaded block stays live.
template <bool RELU, bool SIGMA>
__device__ __forceinline__ void epi_block(const uint32_t* u, const float* sb_bias,
                                          const float* sb_ws, int cb, uint32_t act_base, int r,
                                          float& sigma) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 b0 = *reinterpret_cast<const float4*>(sb_bias + cb + 8 * j);
    const float4 b1 = *reinterpret_cast<const float4*>(sb_bias + cb + 8 * j + 4);
    float v[8];
    v[0] = __uint_as_float(u[8 * j + 0]) + b0.x;
    v[1] = __uint_as_float(u[8 * j + 1]) + b0.y;
    v[2] = __uint_as_float(u[8 * j + 2]) + b0.z;
    v[3] = __uint_as_float(u[8 * j + 3]) + b0.w;
    v[4] = __uint_as_float(u[8 * j + 4]) + b1.x;
    v[5] = __uint_as_float(u[8 * j + 5]) + b1.y;
    v[6] = __uint_as_float(u[8 * j + 6]) + b1.z;
    v[7] = __uint_as_float(u[8 * j + 7]) + b1.w;
    if (SIGMA) {
      const float4 w0 = *reinterpret_cast<const float4*>(sb_ws + cb + 8 * j);
      const float4 w1 = *reinterpret_cast<const float4*>(sb_ws + cb + 8 * j + 4);
      sigma = fmaf(fmaxf(v[0], 0.f), w0.x, sigma);
      sigma = fmaf(fmaxf(v[1], 0.f), w0.y, sigma);
      sigma = fmaf(fmaxf(v[2], 0.f), w0.z, sigma);
      sigma = fmaf(fmaxf(v[3], 0.f), w0.w, sigma);
      sigma = fmaf(fmaxf(v[4], 0.f), w1.x, sigma);
      sigma = fmaf(fmaxf(v[5], 0.f), w1.y, sigma);
      sigma = fmaf(fmaxf(v[6], 0.f), w1.z, sigma);
      sigma = fmaf(fmaxf(v[7], 0.f), w1.w, sigma);
    }
    uint32_t w0, w1, w2, w3;
    if (RELU) {
      w0 = pack_relu(v[0], v[1]); w1 = pack_relu(v[2], v[3]);
      w2 = pack_relu(v[4], v[5]); w3 = pack_relu(v[6], v[7]);
    } else {
      w0 = pack_plain(v[0], v[1]); w1 = pack_plain(v[2], v[3]);
      w2 = pack_plain(v[4], v[5]); w3 = pack_plain(v[6], v[7]);
    }
    st_shared_v4(act_base + act_off(r, cb + 8 * j), w0, w1, w2, w3);
  }
}

// 128 columns [c0, c0 + 128) of a 256-wide hidden layer, two TMEM loads in flight.
template <bool RELU, bool SIGMA>
__device__ __forceinline__ void epi_half(uint32_t t_row, int c0, const float* sb_bias,
                                         const float* sb_ws, uint32_t act_base, int r,
                                         float& sigma) {
  uint32_t ua[32], ub[32];
  tmem_ld32_issue(t_row + c0, ua);
  tmem_ld32_issue(t_row + c0 + 32, ub);
  tmem_wait32(ua);
  tmem_wait32(ub);
  epi_block<RELU, SIGMA>(ua, sb_bias, sb_ws, c0, act_base, r, sigma);
  tmem_ld32_issue(t_row + c0 + 64, ua);
  epi_block<RELU, SIGMA>(ub, sb_bias, sb_ws, c0 + 32, act_base, r, sigma);
  tmem_ld32_issue(t_row + c0 + 96, ub);
  tmem_wait32(ua);
  tmem_wait32(ub);
  epi_block<RELU, SIGMA>(ua, sb_bias, sb_ws, c0 + 64, act_base, r, sigma);
  epi_block<RELU, SIGMA>(ub, sb_bias, sb_ws, c0 + 96, act_base, r, sigma);
}

// Positional-encoding value J (0..63) of a point: [x, sin block, cos block, 0],
// sin and cos blocks coordinate-major (c * 10 + k): sin/cos(pi 2^k x_c).
template <int J>
__device__ __forceinline__ float pe_value(float x0, float x1, float x2) {
  if (J < 3) return J == 0 ? x0 : (J == 1 ? x1 : x2);
  if (J == 63) return 0.0f;
  constexpr int jj = J < 33 ? J - 3 : J - 33;
  constexpr int c = jj / 10, k = jj % 10;
  const float xc = c == 0 ? x0 : (c == 1 ? x1 : x2);
  return J < 33 ? sinpif(ldexpf(xc, k)) : cospif(ldexpf(xc, k));
}

// Columns [32 H, 32 H + 32) of gamma(x), packed to bf16 and stored as the
// A operand's K-groups 32 + 4H .. 35 + 4H.
template <int H, int G = 0>
__device__ __forceinline__ void store_pe(float x0, float x1, float x2, uint32_t act_base, int r) {
  if constexpr (G < 4) {
    constexpr int k0 = H * 32 + 8 * G;
    st_shared_v4(act_base + act_off(r, 256 + k0),
                 pack_plain(pe_value<k0 + 0>(x0, x1, x2), pe_value<k0 + 1>(x0, x1, x2)),
                 pack_plain(pe_value<k0 + 2>(x0, x1, x2), pe_value<k0 + 3>(x0, x1, x2)),
                 pack_plain(pe_value<k0 + 4>(x0, x1, x2), pe_value<k0 + 5>(x0, x1, x2)),
                 pack_plain(pe_value<k0 + 6>(x0, x1, x2), pe_value<k0 + 7>(x0, x1, x2)));
    store_pe<H, G + 1>(x0, x1, x2, act_base, r);
  }
}

// The MMAs of one layer for both tiles of the pair, issued by one thread. The
// tensor pipe finishes an M = 128, N = 256, K = 16 MMA in 128 cycles, and a
// single thread's dependent integer work easily takes longer than that, so
// everything that can be is a compile-time constant (shape, instruction
// descriptor, descriptor strides) and the operand descriptors advance by adds.
//   N: output width; KG0: first K-group of the A operand; NCH: K chunks
template <int N, int KG0, int NCH>
__device__ __forceinline__ bool mma_layer(uint32_t& q, uint32_t (&ph_act)[2], uint64_t* full,
                                          uint64_t* empty, uint64_t* mma_done,
                                          uint64_t* act_ready, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t tmem, const Ctl& ctl) {
  if (!mbar_wait(&act_ready[0], ph_act[0], ctl) || !mbar_wait(&act_ready[1], ph_act[1], ctl))
    return false;
  ph_act[0] ^= 1;
  ph_act[1] ^= 1;
  tc_fence_after();
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                             ((uint32_t)(TM >> 4) << 24);
  // descriptor address steps (bytes >> 4)
  constexpr uint64_t A_KSTEP = (2 * TM * 16) >> 4;        // K = 16: two K-groups
  constexpr uint64_t A_CHUNK = (4 * TM * 16) >> 4;        // K = 32
  constexpr uint64_t A_TILE = ACT_BYTES >> 4;
  constexpr uint64_t B_KSTEP = (2 * N * 16) >> 4;
  constexpr uint64_t B_SLOT = RING_BYTES >> 4;
  // B descriptors of ring slot 0 carry this layer's K-group stride (N * 16 B)
  const uint64_t b0 = (b_desc & ~(0x3FFFull << 16)) | ((uint64_t)((N * 16) >> 4) << 16);
  const uint64_t a0 = a_desc + (uint64_t)((KG0 * TM * 16) >> 4);
#pragma unroll 2
  for (int c = 0; c < NCH; ++c, ++q) {
    const uint32_t slot = q & (NSTAGE - 1);
    if (!mbar_wait(&full[slot], (q / NSTAGE) & 1, ctl)) return false;
    tc_fence_after();
    const uint64_t b = b0 + slot * B_SLOT;
    const uint64_t a = a0 + (uint64_t)c * A_CHUNK;
    const uint32_t acc = c != 0;
    mma_bf16(tmem, a, b, idesc, acc);
    mma_bf16(tmem, a + A_KSTEP, b + B_KSTEP, idesc, 1);
    mma_bf16(tmem + 256, a + A_TILE, b, idesc, acc);
    mma_bf16(tmem + 256, a + A_TILE + A_KSTEP, b + B_KSTEP, idesc, 1);
    mma_commit(&empty[slot]);
  }
  mma_commit(&mma_done[0]);
  mma_commit(&mma_done[1]);
  return true;
}

__global__ void __launch_bounds__(NTHREADS, 1) mlp_tc_kernel(Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* act = smem;                                   // 2 x ACT_BYTES
  uint8_t* ring = smem + 2 * ACT_BYTES;                  // NSTAGE x RING_BYTES
  float* svec = reinterpret_cast<float*>(ring + NSTAGE * RING_BYTES);   // 2 x 256 fp32
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + NSTAGE * RING_BYTES + VEC_BYTES);
  uint64_t* full = bars;                 // [NSTAGE]
  uint64_t* empty = bars + NSTAGE;       // [NSTAGE]
  uint64_t* mma_done = bars + 2 * NSTAGE;     // [2]
  uint64_t* act_ready = bars + 2 * NSTAGE + 2;  // [2]
  uint64_t* final_bar = bars + 2 * NSTAGE + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NSTAGE + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  Ctl ctl{abort_flag, P.flag, kWaitLimitNs};

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&mma_done[g], 1);
      mbar_init(&act_ready[g], TILE_THREADS);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_holder)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int64_t rows = P.R * P.ss.S;

  if (warp == 0) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t q = 0, ph_act[2] = {0, 0};
      bool ok = true;
      const uint64_t a_desc = sdesc(smem_u32(act), TM * 16, 128);
      const uint64_t b_desc = sdesc(smem_u32(ring), 0, 128);
      for (int64_t pr = blockIdx.x; pr < P.n_pairs && ok; pr += gridDim.x) {
        // layer shapes: pts0 (K = 63 -> 64, from the gamma columns), pts1..4,
        // pts5 (skip: K = 256 + 64), pts6, pts7, feature, direction (N = 128)
        ok = mma_layer<256, 32, 2>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 10>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<256, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl) &&
             mma_layer<128, 0, 8>(q, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl);
      }
      // drain: everything issued so far completes before the CTA frees TMEM
      mma_commit(final_bar);
      uint64_t t0 = globaltimer();
      while (!mbar_try(final_bar, 0) && globaltimer() - t0 < kWaitLimitNs) {}
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- weight loader
    if (lane == 0) {
      uint32_t q = 0;
      for (int64_t pr = blockIdx.x; pr < P.n_pairs; pr += gridDim.x) {
        bool ok = true;
        for (int j = 0; j < P.lay.n_chunks; ++j, ++q) {
          const int slot = q % NSTAGE;
          if (!mbar_wait(&empty[slot], ((q / NSTAGE) & 1) ^ 1, ctl)) { ok = false; break; }
          const uint32_t bytes = (uint32_t)P.lay.chunk_bytes[j];
          mbar_arrive_tx(&full[slot], bytes);
          bulk_g2s(ring + slot * RING_BYTES, P.stream + P.lay.chunk_off[j], bytes, &full[slot]);
        }
        if (!ok) break;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int et = threadIdx.x - 64;              // 0..511
    const int g = et >> 8;                        // tile within the pair
    const int h = (et >> 7) & 1;                  // column half
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;            // row in the tile = TMEM lane
    uint8_t* my_act = act + g * ACT_BYTES;
    const uint32_t act_base = smem_u32(my_act);
    const uint32_t t_row = tmem + (uint32_t)(g * 256) + ((uint32_t)(quarter * 32) << 16);
    float* sb0 = svec;          // layer bias / rgb weights rows 0, 1
    float* sb1 = svec + 256;    // sigma weights / rgb row 2, rgb and sigma biases
    // partial (sigma, r, g, b) of the second column half, handed to the first
    // half through the tile's (then idle) activation buffer
    float4* xchg = reinterpret_cast<float4*>(my_act);
    uint32_t ph_md = 0;
    const float* vec = P.vec;
    for (int64_t pr = blockIdx.x; pr < P.n_pairs; pr += gridDim.x) {
      const int64_t row = (pr * 2 + g) * TM + r;
      const bool valid = row < rows;
      int64_t ray = 0;
      float x[3] = {0.f, 0.f, 0.f};
      if (valid) {
        ray = row / P.ss.S;
        const int s = (int)(row % P.ss.S);
        if (P.ss.mode == SAMPLES_GIVEN_X) {
          x[0] = P.ss.t[row * 3]; x[1] = P.ss.t[row * 3 + 1]; x[2] = P.ss.t[row * 3 + 2];
        } else {
          float t;
          if (P.ss.mode == SAMPLES_STRATIFIED) {
            uint32_t m = P.ss.perturb ? draw_bits(P.ss.key, (uint64_t)ray, 0, (uint32_t)s) : 0u;
            t = stratified_t(P.ss.near, P.ss.step, s, m, P.ss.perturb != 0);
          } else {
            t = P.ss.t[row];
          }
#pragma unroll
          for (int c = 0; c < 3; ++c) x[c] = fadd(P.o[ray * 3 + c], fmul(t, P.d[ray * 3 + c]));
        }
      }
      // gamma(x) -> columns 256..319; this half writes 32 of the 64 columns
      if (h == 0) store_pe<0>(x[0], x[1], x[2], act_base, r);
      else store_pe<1>(x[0], x[1], x[2], act_base, r);
      fence_async_smem();
      mbar_arrive(&act_ready[g]);

      float sigma = 0.0f;
      for (int l = 0; l < NLAYER; ++l) {
        // this layer's epilogue vectors: loaded now, staged after the MMA wait
        float pre;
        if (l < 9) {
          pre = et < 256 ? __ldg(vec + P.lay.bias[l] + et)
                         : (l == 7 ? __ldg(vec + P.lay.w_sigma + et - 256) : 0.0f);
        } else {
          const int q2 = et - 256;
          pre = et < 256 ? __ldg(vec + P.lay.w_rgb + et)
              : q2 < 128 ? __ldg(vec + P.lay.w_rgb + 256 + q2)
              : q2 < 131 ? __ldg(vec + P.lay.b_rgb + q2 - 128)
              : q2 == 131 ? __ldg(vec + P.lay.b_sigma) : 0.0f;
        }
        const bool waited = mbar_wait(&mma_done[g], ph_md, ctl);
        ph_md ^= 1;
        tc_fence_after();
        // every epilogue thread is done with the previous vectors; all agree on
        // giving up together, so no thread is left behind at a barrier
        if (epilogue_sync_or(!waited || *abort_flag)) break;
        svec[et] = pre;
        named_sync(1, EPI_THREADS);
        if (l < 9) {
          const int c0 = h * 128;
          if (l == 8) epi_half<false, false>(t_row, c0, sb0, sb1, act_base, r, sigma);
          else if (l == 7) epi_half<true, true>(t_row, c0, sb0, sb1, act_base, r, sigma);
          else epi_half<true, false>(t_row, c0, sb0, sb1, act_base, r, sigma);
          tc_fence_before();
          fence_async_smem();
          mbar_arrive(&act_ready[g]);
        } else {
          // direction layer (N = 128): + per-ray bias, ReLU, the rgb head in fp32
          // on this half's 64 columns; the halves are summed through shared memory
          const float* rb = P.dir_bias + ray * 128;
          float rgb0 = 0.f, rgb1 = 0.f, rgb2 = 0.f;
#pragma unroll 1
          for (int cb = h * 64; cb < h * 64 + 64; cb += 32) {
            uint32_t u[32];
            tmem_ld32_issue(t_row + cb, u);
            float4 bb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) bb[i] = __ldg(reinterpret_cast<const float4*>(rb + cb) + i);
            tmem_wait32(u);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int c = cb + 4 * i;
              const float h0 = fmaxf(__uint_as_float(u[4 * i]) + bb[i].x, 0.f);
              const float h1 = fmaxf(__uint_as_float(u[4 * i + 1]) + bb[i].y, 0.f);
              const float h2 = fmaxf(__uint_as_float(u[4 * i + 2]) + bb[i].z, 0.f);
              const float h3 = fmaxf(__uint_as_float(u[4 * i + 3]) + bb[i].w, 0.f);
              const float4 a4 = *reinterpret_cast<const float4*>(sb0 + c);
              const float4 c4 = *reinterpret_cast<const float4*>(sb0 + 128 + c);
              const float4 d4 = *reinterpret_cast<const float4*>(sb1 + c);
              rgb0 = fmaf(h0, a4.x, fmaf(h1, a4.y, fmaf(h2, a4.z, fmaf(h3, a4.w, rgb0))));
              rgb1 = fmaf(h0, c4.x, fmaf(h1, c4.y, fmaf(h2, c4.z, fmaf(h3, c4.w, rgb1))));
              rgb2 = fmaf(h0, d4.x, fmaf(h1, d4.y, fmaf(h2, d4.z, fmaf(h3, d4.w, rgb2))));
            }
          }
          tc_fence_before();
          if (h == 1) xchg[r] = make_float4(sigma, rgb0, rgb1, rgb2);
          named_sync(2 + g, TILE_THREADS);
          if (h == 0 && valid) {
            const float4 o2 = xchg[r];
            *reinterpret_cast<float4*>(P.raw + row * 4) =
                make_float4(rgb0 + o2.y + sb1[128], rgb1 + o2.z + sb1[129],
                            rgb2 + o2.w + sb1[130], sigma + o2.x + sb1[131]);
          }
          named_sync(2 + g, TILE_THREADS);
        }
      }
      if (epilogue_sync_or(*abort_flag)) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// A wait that nothing completes, bounded by limit_ns: exercises the timeout
// path of the kernels' waits (flag bit FLAG_TIMEOUT, no hang, context intact).
__global__ void bounded_wait_probe_kernel(unsigned* flag, uint64_t limit_ns,
                                          unsigned* waited_us) {
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Ctl ctl{&abort_s, flag, limit_ns};
    const uint64_t t0 = globaltimer();
    mbar_wait(&bar, 0, ctl);
    if (waited_us) *waited_us = (unsigned)((globaltimer() - t0) / 1000);
  }
}

// ------------------------------------------------------------------ weight packing

struct PackLayer {
  int64_t src_w;      // element offset of W [N][K_src] in the blob
  int64_t src_b;
  int N, K_src, n_chunks;
  int chunk0;         // index of the layer's first chunk
};
struct PackPlan {
  PackLayer L[NLAYER];
  int64_t sigma_w, sigma_b, rgb_w, rgb_b;
};

__global__ void tc_pack_kernel(const __nv_bfloat16* __restrict__ blob, PackPlan plan,
                               TcLayout lay, uint8_t* __restrict__ out) {
  const int layer = blockIdx.y;
  const PackLayer& pl = plan.L[layer];
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out);
  const int64_t total = (int64_t)pl.n_chunks * CHUNK_K * pl.N;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(q / (CHUNK_K * pl.N));
    const int rem = (int)(q % (CHUNK_K * pl.N));
    const int n = rem / CHUNK_K, kl = rem % CHUNK_K;
    const int k = c * CHUNK_K + kl;
    __nv_bfloat16 v = k < pl.K_src ? blob[pl.src_w + (int64_t)n * pl.K_src + k]
                                   : __float2bfloat16(0.0f);
    const int64_t byte = lay.chunk_off[pl.chunk0 + c] + (kl >> 3) * (pl.N * 16) + (n >> 3) * 128 +
                         (n & 7) * 16 + (kl & 7) * 2;
    dst[byte / 2] = v;
  }
  // fp32 vectors (done by the y = 0 slice)
  if (layer == 0) {
    float* vec = reinterpret_cast<float*>(out + lay.vec_off);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < lay.vec_count;
         i += gridDim.x * blockDim.x) {
      float v = 0.0f;
      for (int l = 0; l < NLAYER; ++l)
        if (i >= lay.bias[l] && i < lay.bias[l] + plan.L[l].N)
          v = __bfloat162float(blob[plan.L[l].src_b + (i - lay.bias[l])]);
      if (i >= lay.w_sigma && i < lay.w_sigma + 256) v = __bfloat162float(blob[plan.sigma_w + i - lay.w_sigma]);
      if (i == lay.b_sigma) v = __bfloat162float(blob[plan.sigma_b]);
      if (i >= lay.w_rgb && i < lay.w_rgb + 384) v = __bfloat162float(blob[plan.rgb_w + i - lay.w_rgb]);
      if (i >= lay.b_rgb && i < lay.b_rgb + 3) v = __bfloat162float(blob[plan.rgb_b + i - lay.b_rgb]);
      vec[i] = v;
    }
  }
}

struct TcState {
  TcLayout lay;
  PackPlan plan;
  uint8_t* buf = nullptr;
};

}  // namespace

cudaError_t tc_alloc(nerf_ctx* ctx) {
  TcState* s = new TcState();
  s->lay = make_layout();
  // blob offsets of the 8x256 network (layer order of the ABI)
  const int W = 256, pos_ch = 63, dir_ch = 27;
  int64_t off = 0;
  int chunk = 0;
  for (int l = 0; l < 8; ++l) {
    const int K = l == 0 ? pos_ch : (l == 5 ? W + pos_ch : W);
    s->plan.L[l] = {off, off + (int64_t)W * K, W, K, l == 0 ? 2 : (l == 5 ? 10 : 8), chunk};
    chunk += s->plan.L[l].n_chunks;
    off += (int64_t)W * K + W;
  }
  s->plan.sigma_w = off; off += W;
  s->plan.sigma_b = off; off += 1;
  s->plan.L[8] = {off, off + (int64_t)W * W, W, W, 8, chunk};
  chunk += 8;
  off += (int64_t)W * W + W;
  // direction layer: W_dir [128][W + dir_ch]; only its first W columns are packed,
  // read with row stride W + dir_ch
  s->plan.L[9] = {off, off + (int64_t)(W / 2) * (W + dir_ch), W / 2, W + dir_ch, 8, chunk};
  off += (int64_t)(W / 2) * (W + dir_ch) + W / 2;
  s->plan.rgb_w = off; off += 3 * (W / 2);
  s->plan.rgb_b = off;
  cudaError_t e = cudaMalloc(&s->buf, s->lay.vec_off + s->lay.vec_count * sizeof(float));
  if (e != cudaSuccess) { delete s; return e; }
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaFuncSetAttribute(mlp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES);
  if (e != cudaSuccess) { cudaFree(s->buf); delete s; return e; }
  ctx->tc_weights = s;
  ctx->tc_enabled = true;
  return cudaSuccess;
}

void tc_free(nerf_ctx* ctx) {
  TcState* s = static_cast<TcState*>(ctx->tc_weights);
  if (!s) return;
  cudaFree(s->buf);
  delete s;
  ctx->tc_weights = nullptr;
  ctx->tc_enabled = false;
}

cudaError_t launch_bounded_wait_probe(uint32_t timeout_us, uint32_t* flag, uint32_t* waited_us,
                                      cudaStream_t st) {
  bounded_wait_probe_kernel<<<1, 32, 0, st>>>(flag, (uint64_t)timeout_us * 1000ull, waited_us);
  return cudaGetLastError();
}

cudaError_t tc_pack(nerf_ctx* ctx, const void* blob, cudaStream_t st) {
  TcState* s = static_cast<TcState*>(ctx->tc_weights);
  // The dir layer's K columns 0..255 are read with the blob's row stride
  // (W + dir_ch); the pack kernel indexes rows with K_src, so pass the stride
  // and clip the packed K range to the first W columns.
  PackPlan plan = s->plan;
  dim3 grid(128, NLAYER);
  tc_pack_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(blob), plan, s->lay,
                                       s->buf);
  return cudaGetLastError();
}

cudaError_t tc_run(nerf_ctx* ctx, const float* o, const float* d, int64_t R, const SampleSpec& ss,
                   float* raw, cudaStream_t st) {
  TcState* s = static_cast<TcState*>(ctx->tc_weights);
  Params P;
  P.stream = s->buf;
  P.vec = reinterpret_cast<const float*>(s->buf + s->lay.vec_off);
  P.lay = s->lay;
  P.dir_bias = ctx->dir_bias;
  P.o = o;
  P.d = d;
  P.R = R;
  P.ss = ss;
  P.raw = raw;
  P.flag = ctx->d_flag;
  const int64_t rows = R * ss.S;
  P.n_pairs = (rows + 2 * TM - 1) / (2 * TM);
  const int64_t grid = P.n_pairs < ctx->num_sms ? P.n_pairs : ctx->num_sms;
  mlp_tc_kernel<<<(unsigned)grid, NTHREADS, SMEM_BYTES, st>>>(P);
  return cudaGetLastError();
}

}  // namespace nerfb
