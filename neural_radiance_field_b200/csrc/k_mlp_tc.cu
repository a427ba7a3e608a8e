// bf16 tensor-core evaluation of the NeRF scene MLP (NeRF page, Section 2.4) on
// sm_100a: tcgen05.mma with fp32 accumulators in tensor memory, weights streamed
// by TMA, activations kept on chip for the whole network.
//
// Clusters of two CTAs on two SMs run 2-SM MMAs (cta_group::2, M = 256): each
// CTA holds 128 rows of a 256-row tile and half of every weight chunk, and
// receives its 128 rows x N of the accumulator in its own tensor memory. A
// cluster works on pairs of such tiles, A and B, whose layers alternate on the
// tensor cores (A0 B0 A1 B1 ...), so that one tile's epilogue runs while the
// other tile's layer is computed. Each weight chunk that lands in the ring
// serves both tiles (tile A's pass waits for it, tile B's pass frees its slot),
// so each weight byte read from L2 serves 512 rows. Per CTA, 18 warps:
//   warp 0       CTA 0: issues the MMAs of the pair; both CTAs: TMEM allocation
//   warp 1       streams this CTA's half of each weight chunk into an 8-slot ring
//                (one 256-input layer)
//   warps 2-9    epilogue of tile A: warp w drains TMEM lane quarter (w % 4) of
//                column half ((w - 2) / 4) % 2, i.e. thread = (row, half)
//   warps 10-17  epilogue of tile B, same split
// The epilogue adds the bias, applies ReLU, rounds to bf16 and writes the next
// layer's A operand into shared memory; the last layers add the sigma and rgb
// heads in fp32.
//
// Shared memory per CTA (231,680 B): act[2] = per tile 128 rows x 320 bf16 holding
// [h (256) | gamma(x) (63) | 0], so the skip layer reads columns 0..319 and the
// first layer columns 256..319; ring[8] = half weight chunks (N/2 rows x 32 K);
// 2 KB of per-tile epilogue vectors (bf16); barriers.
// Operands use the no-swizzle K-major core-matrix layout: element (r, k) of a
// block of R rows sits at (k/8)*R*16 + (r/8)*128 + (r%8)*16 + (k%8)*2 bytes.
#include <cuda.h>

#include "nerf_ctx.h"
#include "tc_ptx.cuh"

namespace nerfb {

namespace {

constexpr int TM = 128;
constexpr int ACT_K = 320;
constexpr int ACT_BYTES = TM * ACT_K * 2;           // 81920
constexpr int CHUNK_K = 32;
constexpr int NSTAGE = 8;                           // ring slots (chunks)
constexpr int RING_BYTES = 128 * CHUNK_K * 2;       // 8192: one CTA's half of a chunk
constexpr int UNIT_CHUNKS = 4;                      // chunks per load and per barrier
constexpr int NGROUP = NSTAGE / UNIT_CHUNKS;        // slot groups, one unit each
constexpr int GROUP_BYTES = UNIT_CHUNKS * RING_BYTES;
constexpr int NLAYER = 10;                          // pts0..pts7, feature, dir
constexpr int EPI_THREADS = 512;                    // 16 epilogue warps
constexpr int TILE_THREADS = 256;                   // epilogue threads per tile
constexpr int NTHREADS = 64 + EPI_THREADS;
constexpr int VEC_BYTES = 2 * 512 * 2;              // per-tile staged epilogue vectors (bf16)
constexpr size_t SMEM_BYTES = 2 * ACT_BYTES + NSTAGE * RING_BYTES + VEC_BYTES + 256;

// Packed weight stream and fp32 vectors. The stream is two half-streams, one
// per CTA of the pair: half-stream c holds, in consumption order, every chunk's
// rows [c N/2, (c + 1) N/2), so that a CTA's halves of consecutive chunks are
// contiguous. The chunks of a layer travel in units of four (the last unit of
// a layer may hold two): one bulk-tensor load per CTA and unit; in the MMA
// warp, one barrier wait (first tile) or slot release (second tile) per unit
// around the unit's eight MMAs, which are issued back to back in straight-line
// code. (Measured on the 8 x 256 network: units of two 0.5 % slower; a loop
// with runtime slot arithmetic between the MMAs 5 % slower.)
struct TcLayout {
  int64_t half_off[80];      // byte offset of a chunk's half within a half-stream
  int half_bytes[80];        // bytes of one CTA's half of the chunk
  int n_chunks;
  int n_units;               // load units of one pass over the network
  int unit_chunk0[40];       // first chunk of each unit
  int unit_bytes[40];        // bytes of one CTA's half of each unit (a full or a half group)
  int64_t half_stream_bytes;
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
  int u = 0;
  for (int l = 0; l < NLAYER; ++l)
    for (int c = 0; c < kch[l]; ++c) {
      if (c % UNIT_CHUNKS == 0) {          // units of four within the layer, the rest last
        L.unit_chunk0[u] = q;
        L.unit_bytes[u] = 0;
        ++u;
      }
      L.half_off[q] = off;
      L.half_bytes[q] = (nout[l] / 2) * CHUNK_K * 2;
      L.unit_bytes[u - 1] += L.half_bytes[q];
      off += L.half_bytes[q];
      ++q;
    }
  L.n_chunks = q;
  L.n_units = u;
  L.half_stream_bytes = off;
  L.stream_bytes = 2 * off;
  L.vec_off = (L.stream_bytes + 255) & ~int64_t(255);   // the vectors follow both half-streams
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

// the single-CTA wrappers shared with the other tensor-core kernels
using tcx::globaltimer;
using tcx::mbar_arrive;
using tcx::mbar_init;
using tcx::mbar_try;
using tcx::sdesc;
using tcx::smem_u32;
using tcx::st_shared_v4;
__device__ __forceinline__ void tc_fence_before() { tcx::fence_before(); }
__device__ __forceinline__ void tc_fence_after() { tcx::fence_after(); }
__device__ __forceinline__ void fence_async_smem() { tcx::fence_async_smem(); }

__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes) : "memory");
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

// Two fp32 -> packed bf16x2 with ReLU (lo = first element in memory order).
__device__ __forceinline__ uint32_t pack_relu(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.relu.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint32_t pack_plain(float lo, float hi) { return tcx::pack_bf16(lo, hi); }

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

// 32-column TMEM loads of this warp's lane quarter (valid after tmem_wait32).
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t* r) { tcx::tmem_ld32(taddr, r); }
__device__ __forceinline__ void tmem_wait32(uint32_t* r) { tcx::tmem_ld_wait(r); }

// Named barrier 1 + g over the 256 epilogue threads of tile g.
__device__ __forceinline__ void tile_sync(int g) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

// The same barrier, returning whether any of the tile's threads passed true.
__device__ __forceinline__ bool tile_sync_or(int g, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "bar.red.or.pred q, %1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(1 + g), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Eight bf16 values (16 bytes of shared memory) widened exactly to fp32.
__device__ __forceinline__ void load_bf16x8(const uint16_t* p, float* f) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  f[0] = __uint_as_float(w.x << 16); f[1] = __uint_as_float(w.x & 0xFFFF0000u);
  f[2] = __uint_as_float(w.y << 16); f[3] = __uint_as_float(w.y & 0xFFFF0000u);
  f[4] = __uint_as_float(w.z << 16); f[5] = __uint_as_float(w.z & 0xFFFF0000u);
  f[6] = __uint_as_float(w.w << 16); f[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

// One 32-column block of a hidden layer: bias, activation, bf16, store to the
// next layer's A operand; on the last trunk layer also accumulates sigma. Works
// 8 columns at a time so that only the loaded block stays live.
template <bool RELU, bool SIGMA>
__device__ __forceinline__ void epi_block(const uint32_t* u, const uint16_t* sb_bias,
                                          const uint16_t* sb_ws, int cb, uint32_t act_base, int r,
                                          float& sigma) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float b[8];
    load_bf16x8(sb_bias + cb + 8 * j, b);
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2)
      asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
          "mov.b64 ra, {%2, %3};\n\t"
          "mov.b64 rb, {%4, %5};\n\t"
          "add.rn.f32x2 rd, ra, rb;\n\t"
          "mov.b64 {%0, %1}, rd;\n\t}"
          : "=f"(v[i]), "=f"(v[i + 1])
          : "f"(__uint_as_float(u[8 * j + i])), "f"(__uint_as_float(u[8 * j + i + 1])),
            "f"(b[i]), "f"(b[i + 1]));
    if (SIGMA) {
      float w[8];
      load_bf16x8(sb_ws + cb + 8 * j, w);
#pragma unroll
      for (int i = 0; i < 8; ++i) sigma = fmaf(fmaxf(v[i], 0.f), w[i], sigma);
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
__device__ __forceinline__ void epi_half(uint32_t t_row, int c0, const uint16_t* sb_bias,
                                         const uint16_t* sb_ws, uint32_t act_base, int r,
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

// ---- 2-SM additions (cluster of 2 CTAs, tcgen05 cta_group::2) ----

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// try_wait with cluster-scope acquire: the barrier may be completed by the peer CTA.
__device__ __forceinline__ bool mbar_try_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, const Ctl& ctl) {
  if (mbar_try_cl(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_cl(bar, parity)) {
    if (*ctl.abort) return false;
    if (globaltimer() - t0 > ctl.limit_ns) {
      atomicOr(ctl.flag, FLAG_TIMEOUT);
      *ctl.abort = 1;
      return false;
    }
  }
  return true;
}

// Arrive on the barrier at the same offset in CTA 0 of the cluster, releasing
// at cluster scope this CTA's shared-memory writes (including those the calling
// thread has acquired from other threads): a release fence restricted to
// shared::cta operations, then a relaxed remote arrive. A full cluster-scope
// release on the arrive itself costs about 1,100 cycles more (measured).
__device__ __forceinline__ void mbar_arrive_leader(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, 0;\n\t"
      "fence.release.sync_restrict::shared::cta.cluster;\n\t"
      "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}"
      ::"r"(smem_u32(bar))
      : "memory");
}

// 2-D tensor load into this CTA's shared memory whose completion is counted on
// CTA 0's barrier (the barrier address with the peer bit cleared).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* tmap, int x, int y,
                                                 uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tmap)),
        "r"(smem_u32(bar) & 0xFEFFFFFFu), "r"(x), "r"(y)
      : "memory");
}


// The MMA warp runs its loop converged (all 32 lanes: warp-uniform operands and
// control), and lane 0 alone issues each tcgen05 instruction, predicated inside
// the asm. The converged issue loop is 8 % faster than one lane running it
// alone (measured on the 8 x 256 network).
__device__ __forceinline__ void mma_bf16_pair(uint32_t tmem_d, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\t"
      "mov.u32 ln, %%laneid;\n\t"
      "setp.eq.u32 e, ln, 0;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}

// Arrive (once each) on the barrier at this offset in both CTAs of the pair
// when every MMA previously issued by lane 0 of the calling warp has completed
// (lane 0 issues the commit).
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 ln;\n\t"
      "mov.u32 ln, %%laneid;\n\t"
      "setp.eq.u32 e, ln, 0;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;\n\t}"
      ::"r"(smem_u32(bar)), "h"((uint16_t)3)
      : "memory");
}

// The MMAs of tile g over one unit of a layer, chunks [C0, C0 + NC), held by
// slot group grp of the ring, issued back to back by CTA 0's MMA warp: a 2-SM
// MMA (M = 256, N = 256, K = 16) takes 128 cycles on the tensor pipe, and the
// unit's 2 NC MMAs run without a barrier operation or loop overhead between
// them (shapes, offsets and the accumulate flags are compile-time constants).
//   N: output width; KG0: first K-group of the A operand
template <int N, int KG0, int C0, int NC>
__device__ __forceinline__ void mma_unit(int g, uint32_t grp, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t tmem) {
  constexpr int Nh = N / 2;                 // rows of B held by each CTA
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                             (16u << 24);   // M = 256
  constexpr uint64_t A_KSTEP = (2 * TM * 16) >> 4;
  constexpr uint64_t A_CHUNK = (4 * TM * 16) >> 4;
  constexpr uint64_t A_TILE = ACT_BYTES >> 4;
  constexpr uint64_t B_KSTEP = (2 * Nh * 16) >> 4;
  constexpr uint64_t B_CHUNK = (Nh * CHUNK_K * 2) >> 4;   // one chunk's half, packed in the unit
  constexpr uint64_t B_GROUP = GROUP_BYTES >> 4;
  const uint64_t b0 = ((b_desc & ~(0x3FFFull << 16)) | ((uint64_t)((Nh * 16) >> 4) << 16)) +
                      (uint64_t)grp * B_GROUP;
  const uint64_t a0 = a_desc + (uint64_t)g * A_TILE + (uint64_t)((KG0 * TM * 16) >> 4) +
                      (uint64_t)C0 * A_CHUNK;
  const uint32_t td = tmem + (uint32_t)g * 256;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    mma_bf16_pair(td, a0 + c * A_CHUNK, b0 + c * B_CHUNK, idesc, C0 + c != 0);
    mma_bf16_pair(td, a0 + c * A_CHUNK + A_KSTEP, b0 + c * B_CHUNK + B_KSTEP, idesc, 1);
  }
}

// The epilogue's hand-off to the MMA warp: every lane has made its stores
// visible to the async proxy; after the warp converges, one lane arrives on the
// MMA warp's barrier in CTA 0 (remotely from CTA 1, with the restricted
// release fence of mbar_arrive_leader). 256 per-thread arrivals on one barrier
// would serialize; 8 per CTA do not.
__device__ __forceinline__ void warp_arrive_act(uint64_t* bar, uint32_t cta, int lane) {
  __syncwarp();
  if (lane == 0) {
    if (cta == 0) mbar_arrive(bar);
    else mbar_arrive_leader(bar);
  }
}

__device__ __forceinline__ bool wait_act(int g, uint32_t (&ph_act)[2], uint64_t* act_ready,
                                         const Ctl& ctl) {
  if (!mbar_wait_cl(&act_ready[g], ph_act[g], ctl)) return false;
  ph_act[g] ^= 1;
  tc_fence_after();
  return true;
}

// Units [K, KEND) of one layer for tile g, in straight-line code: tile A's
// pass (FIRST) waits for each unit to land before its MMAs, tile B's pass
// releases each unit's slots after its MMAs. Unit U + K of the kernel sits in
// slot group (U + K) % NGROUP, whose barriers complete once per unit.
template <int N, int KG0, int NCH, int K, int KEND, bool FIRST>
__device__ __forceinline__ bool mma_units(int g, uint32_t U, uint64_t* full, uint64_t* empty,
                                          uint64_t a_desc, uint64_t b_desc, uint32_t tmem,
                                          const Ctl& ctl) {
  if constexpr (K < KEND) {
    constexpr int C0 = K * UNIT_CHUNKS;
    constexpr int NC = NCH - C0 < UNIT_CHUNKS ? NCH - C0 : UNIT_CHUNKS;
    const uint32_t u = U + K, grp = u % NGROUP;
    if (FIRST) {
      if (!mbar_wait_cl(&full[grp], (u / NGROUP) & 1, ctl)) return false;
      tc_fence_after();
    }
    mma_unit<N, KG0, C0, NC>(g, grp, a_desc, b_desc, tmem);
    if (!FIRST) mma_commit_pair(&empty[grp]);
    return mma_units<N, KG0, NCH, K + 1, KEND, FIRST>(g, U, full, empty, a_desc, b_desc, tmem, ctl);
  } else {
    return true;
  }
}

// One layer of both tiles, tile A first: while one tile's accumulator is
// drained by its epilogue, the other tile's layer runs. Every unit serves both
// tiles. The ring holds one 8-chunk layer; the 10-chunk skip layer runs as
// A[0..7] B[0..7] A[8, 9] B[8, 9], its last unit reusing the slots that tile B
// has released. U counts the units of the kernel.
template <int N, int KG0, int NCH>
__device__ __forceinline__ bool mma_layer_pingpong(uint32_t& U, uint32_t (&ph_act)[2],
                                                   uint64_t* full, uint64_t* empty,
                                                   uint64_t* mma_done, uint64_t* act_ready,
                                                   uint64_t a_desc, uint64_t b_desc,
                                                   uint32_t tmem, const Ctl& ctl) {
  constexpr int NU = (NCH + UNIT_CHUNKS - 1) / UNIT_CHUNKS;
  constexpr int NA = NU < NGROUP ? NU : NGROUP;          // units of the first round
  static_assert(NU <= NA + NGROUP && NCH - NA * UNIT_CHUNKS <= NSTAGE, "unit schedule");
  if (!wait_act(0, ph_act, act_ready, ctl) ||
      !mma_units<N, KG0, NCH, 0, NA, true>(0, U, full, empty, a_desc, b_desc, tmem, ctl))
    return false;
  if (NU == NA) mma_commit_pair(&mma_done[0]);
  if (!wait_act(1, ph_act, act_ready, ctl)) return false;
  mma_units<N, KG0, NCH, 0, NA, false>(1, U, full, empty, a_desc, b_desc, tmem, ctl);
  if (NU > NA) {
    if (!mma_units<N, KG0, NCH, NA, NU, true>(0, U, full, empty, a_desc, b_desc, tmem, ctl))
      return false;
    mma_commit_pair(&mma_done[0]);
    mma_units<N, KG0, NCH, NA, NU, false>(1, U, full, empty, a_desc, b_desc, tmem, ctl);
  }
  mma_commit_pair(&mma_done[1]);
  U += NU;
  return true;
}

__global__ void __launch_bounds__(NTHREADS, 1) mlp_tc_kernel(Params P, const __grid_constant__ CUtensorMap tmap_unit,
              const __grid_constant__ CUtensorMap tmap_half) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* act = smem;                                   // 2 x ACT_BYTES
  uint8_t* ring = smem + 2 * ACT_BYTES;                  // NSTAGE x RING_BYTES
  uint16_t* svec = reinterpret_cast<uint16_t*>(ring + NSTAGE * RING_BYTES);  // 2 tiles x 512 bf16
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + NSTAGE * RING_BYTES + VEC_BYTES);
  uint64_t* full = bars;                 // [NGROUP] (used in CTA 0)
  uint64_t* empty = bars + NGROUP;       // [NGROUP]
  uint64_t* mma_done = bars + 2 * NGROUP;     // [2]
  uint64_t* act_ready = bars + 2 * NGROUP + 2;  // [2] (used in CTA 0)
  uint64_t* final_bar = bars + 2 * NGROUP + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * NGROUP + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = (int)cluster_ctarank();      // 0 issues the MMAs of the pair
  const int64_t cid = cluster_id_x(), ncl = nclusters_x();
  Ctl ctl{abort_flag, P.flag, kWaitLimitNs};

  if (threadIdx.x == 0) {
    for (int s = 0; s < NGROUP; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&mma_done[g], 1);
      mbar_init(&act_ready[g], 2 * TILE_THREADS / 32);   // one arrival per epilogue warp
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_holder)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();            // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int64_t rows = P.R * P.ss.S;

  if (warp == 0) {
    // ---------------------------------------------------------- MMA issuer (CTA 0)
    if (cta == 0) {
      uint32_t U = 0, ph_act[2] = {0, 0};
      bool ok = true;
      const uint64_t a_desc = sdesc(smem_u32(act), TM * 16, 128);
      const uint64_t b_desc = sdesc(smem_u32(ring), 0, 128);
#define NERF_PP_LAYER(N, KG0, NCH) \
  mma_layer_pingpong<N, KG0, NCH>(U, ph_act, full, empty, mma_done, act_ready, a_desc, b_desc, tmem, ctl)
      for (int64_t pr = cid; pr < P.n_pairs && ok; pr += ncl) {
        // layer shapes: pts0 (K = 63 -> 64, from the gamma columns), pts1..4,
        // pts5 (skip: K = 256 + 64), pts6, pts7, feature, direction (N = 128).
        // One copy of the code per shape: the MMA warp's code stays small enough
        // for the instruction cache (ten inlined copies measured 16 % slower).
#pragma unroll 1
        for (int l = 0; l < NLAYER && ok; ++l) {
          if (l == 0) ok = NERF_PP_LAYER(256, 32, 2);
          else if (l == 5) ok = NERF_PP_LAYER(256, 0, 10);
          else if (l == 9) ok = NERF_PP_LAYER(128, 0, 8);
          else ok = NERF_PP_LAYER(256, 0, 8);
        }
      }
#undef NERF_PP_LAYER
      // drain: everything issued so far completes before the pair frees TMEM.
      // The wait does not stop on an abort (the MMAs already issued must land
      // first); if it runs out, the timeout is reported like any other wait's.
      mma_commit_pair(final_bar);
      const uint64_t t0 = globaltimer();
      bool drained = mbar_try_cl(final_bar, 0);
      while (!drained && globaltimer() - t0 < ctl.limit_ns) drained = mbar_try_cl(final_bar, 0);
      if (!drained) {
        atomicOr(ctl.flag, FLAG_TIMEOUT);
        *ctl.abort = 1;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- weight loader (both CTAs)
    // Each CTA loads its halves (rows [cta * N/2, (cta + 1) * N/2) of the layer)
    // of a unit's chunks with one request into the unit's slot group; the bytes
    // of both CTAs are counted on CTA 0's barrier of the group. The warp runs
    // the loop converged; lane 0 issues the requests.
    {
      uint32_t U = 0;
      for (int64_t pr = cid; pr < P.n_pairs; pr += ncl) {
        bool ok = true;
        for (int u = 0; u < P.lay.n_units; ++u, ++U) {
          const uint32_t grp = U % NGROUP;
          // the group's previous unit has served both tiles
          if (!mbar_wait_cl(&empty[grp], ((U / NGROUP) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          const uint32_t bytes = (uint32_t)P.lay.unit_bytes[u];
          const int64_t off = (int64_t)cta * P.lay.half_stream_bytes + P.lay.half_off[P.lay.unit_chunk0[u]];
          if (lane == 0) {
            if (cta == 0) mbar_arrive_tx(&full[grp], 2 * bytes);
            tma_load_2d_pair(ring + grp * GROUP_BYTES,
                             bytes == GROUP_BYTES ? (const void*)&tmap_unit : (const void*)&tmap_half,
                             0, (int)(off / 128), &full[grp]);
          }
          __syncwarp();
        }
        if (!ok) break;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue (both CTAs)
    const int et = threadIdx.x - 64;              // 0..511
    const int g = et >> 8;                        // tile within the pair
    const int h = (et >> 7) & 1;                  // column half
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;            // row in this CTA's half tile = TMEM lane
    uint8_t* my_act = act + g * ACT_BYTES;
    const uint32_t act_base = smem_u32(my_act);
    const uint32_t t_row = tmem + (uint32_t)(g * 256) + ((uint32_t)(quarter * 32) << 16);
    const int tt = et & 255;                      // thread within the tile
    uint16_t* sb0 = svec + g * 512;   // layer bias / rgb weights rows 0, 1 (bf16)
    uint16_t* sb1 = sb0 + 256;        // sigma weights / rgb row 2, rgb and sigma biases
    // partial (sigma, r, g, b) of the second column half, handed to the first
    // half through the tile's (then idle) activation buffer
    float4* xchg = reinterpret_cast<float4*>(my_act);
    uint32_t ph_md = 0;
    const float* vec = P.vec;
    for (int64_t pr = cid; pr < P.n_pairs; pr += ncl) {
      const int64_t row = (pr * 2 + g) * (2 * TM) + cta * TM + r;
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
      warp_arrive_act(&act_ready[g], cta, lane);

      float sigma = 0.0f;
      // A layer's epilogue vectors (all bf16 weights of the blob, so the bf16
      // staging is exact) are staged while the tile waits for that layer's
      // MMAs, so that nothing but the accumulator stands between the MMAs'
      // completion and the epilogue.
      auto stage_vectors = [&](int l) {
        float pre0, pre1 = 0.0f;
        if (l < 9) {
          pre0 = __ldg(vec + P.lay.bias[l] + tt);
          if (l == 7) pre1 = __ldg(vec + P.lay.w_sigma + tt);
        } else {
          pre0 = __ldg(vec + P.lay.w_rgb + tt);
          pre1 = tt < 128 ? __ldg(vec + P.lay.w_rgb + 256 + tt)
               : tt < 131 ? __ldg(vec + P.lay.b_rgb + tt - 128)
               : tt == 131 ? __ldg(vec + P.lay.b_sigma) : 0.0f;
        }
        sb0[tt] = __bfloat16_as_ushort(__float2bfloat16_rn(pre0));
        sb1[tt] = __bfloat16_as_ushort(__float2bfloat16_rn(pre1));
      };
      // the tile's threads are done with the previous pair's vectors; all
      // agree on giving up together, so no thread is left behind at a barrier
      if (tile_sync_or(g, *abort_flag)) break;
      stage_vectors(0);
      tile_sync(g);
      bool stop = false;
      for (int l = 0; l < NLAYER; ++l) {
        const bool waited = mbar_wait_cl(&mma_done[g], ph_md, ctl);
        ph_md ^= 1;
        tc_fence_after();
        if (l < 9) {
          const int c0 = h * 128;
          if (l == 8) epi_half<false, false>(t_row, c0, sb0, sb1, act_base, r, sigma);
          else if (l == 7) epi_half<true, true>(t_row, c0, sb0, sb1, act_base, r, sigma);
          else epi_half<true, false>(t_row, c0, sb0, sb1, act_base, r, sigma);
          tc_fence_before();
          fence_async_smem();
          warp_arrive_act(&act_ready[g], cta, lane);
          if (tile_sync_or(g, !waited || *abort_flag)) { stop = true; break; }
          stage_vectors(l + 1);
          tile_sync(g);
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
              const uint2 a2 = *reinterpret_cast<const uint2*>(sb0 + c);
              const uint2 c2 = *reinterpret_cast<const uint2*>(sb0 + 128 + c);
              const uint2 d2 = *reinterpret_cast<const uint2*>(sb1 + c);
              rgb0 = fmaf(h0, __uint_as_float(a2.x << 16), fmaf(h1, __uint_as_float(a2.x & 0xFFFF0000u),
                     fmaf(h2, __uint_as_float(a2.y << 16), fmaf(h3, __uint_as_float(a2.y & 0xFFFF0000u), rgb0))));
              rgb1 = fmaf(h0, __uint_as_float(c2.x << 16), fmaf(h1, __uint_as_float(c2.x & 0xFFFF0000u),
                     fmaf(h2, __uint_as_float(c2.y << 16), fmaf(h3, __uint_as_float(c2.y & 0xFFFF0000u), rgb1))));
              rgb2 = fmaf(h0, __uint_as_float(d2.x << 16), fmaf(h1, __uint_as_float(d2.x & 0xFFFF0000u),
                     fmaf(h2, __uint_as_float(d2.y << 16), fmaf(h3, __uint_as_float(d2.y & 0xFFFF0000u), rgb2))));
            }
          }
          tc_fence_before();
          if (h == 1) xchg[r] = make_float4(sigma, rgb0, rgb1, rgb2);
          tile_sync(g);
          if (h == 0 && valid) {
            const float4 o2 = xchg[r];
            auto bf = [&](int i) { return __uint_as_float((uint32_t)sb1[i] << 16); };
            *reinterpret_cast<float4*>(P.raw + row * 4) =
                make_float4(rgb0 + o2.y + bf(128), rgb1 + o2.z + bf(129),
                            rgb2 + o2.w + bf(130), sigma + o2.x + bf(131));
          }
          tile_sync(g);
          if (!waited) stop = true;
        }
      }
      if (tile_sync_or(g, stop || *abort_flag)) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();            // the peer's MMAs and loads into this CTA are over
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
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

// Chunk c of a layer holds K columns [32c, 32c + 32) of all N rows as two
// halves (rows [0, N/2) then [N/2, N)), one per CTA of the pair, each in the
// no-swizzle K-major core-matrix layout of an N/2-row operand.
__global__ void tc_pack_kernel(const __nv_bfloat16* __restrict__ blob, PackPlan plan,
                               TcLayout lay, uint8_t* __restrict__ out) {
  const int layer = blockIdx.y;
  const PackLayer& pl = plan.L[layer];
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out);
  const int Nh = pl.N / 2;
  const int64_t total = (int64_t)pl.n_chunks * CHUNK_K * pl.N;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(q / (CHUNK_K * pl.N));
    const int rem = (int)(q % (CHUNK_K * pl.N));
    const int n = rem / CHUNK_K, kl = rem % CHUNK_K;
    const int k = c * CHUNK_K + kl;
    __nv_bfloat16 v = k < pl.K_src ? blob[pl.src_w + (int64_t)n * pl.K_src + k]
                                   : __float2bfloat16(0.0f);
    const int hh = n / Nh, nn = n % Nh;
    const int64_t byte = (int64_t)hh * lay.half_stream_bytes + lay.half_off[pl.chunk0 + c] +
                         (kl >> 3) * (Nh * 16) + (nn >> 3) * 128 + (nn & 7) * 16 + (kl & 7) * 2;
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
  CUtensorMap tmap_unit;    // the stream as rows of 128 B, boxes of one unit's half (GROUP_BYTES)
  CUtensorMap tmap_half;    // boxes of half of that (the direction layer's units)
  int max_clusters = 0;     // co-resident CTA pairs of the kernel on this device
};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t make_stream_map(CUtensorMap* m, void* base, int64_t bytes, int box_rows) {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  const cuuint64_t dims[2] = {64, (cuuint64_t)(bytes / 128)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

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
  // the packed stream (both half-streams) and then the vectors, inside one allocation
  bool units_ok = s->lay.n_units <= 40;
  for (int u = 0; u < s->lay.n_units && units_ok; ++u)
    units_ok = s->lay.unit_bytes[u] == GROUP_BYTES || s->lay.unit_bytes[u] == GROUP_BYTES / 2;
  if (s->lay.vec_off < s->lay.stream_bytes || !units_ok) { delete s; return cudaErrorInvalidValue; }
  cudaError_t e = cudaMalloc(&s->buf, s->lay.vec_off + s->lay.vec_count * sizeof(float));
  if (e == cudaSuccess) e = make_stream_map(&s->tmap_unit, s->buf, s->lay.stream_bytes, GROUP_BYTES / 128);
  if (e == cudaSuccess) e = make_stream_map(&s->tmap_half, s->buf, s->lay.stream_bytes, GROUP_BYTES / 256);
  if (e != cudaSuccess) { cudaFree(s->buf); delete s; return e; }
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaFuncSetAttribute(mlp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(mlp_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
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
  dim3 grid(128, NLAYER);
  tc_pack_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(blob), s->plan, s->lay,
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
  P.n_pairs = (rows + 4 * TM - 1) / (4 * TM);     // two tiles of 256 rows per CTA pair
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (s->max_clusters <= 0) {
    // persistent grid: as many CTA pairs as can be resident at once
    cfg.gridDim = dim3((unsigned)ctx->num_sms & ~1u);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, mlp_tc_kernel, &cfg) != cudaSuccess || n <= 0)
      n = ctx->num_sms / 2;
    s->max_clusters = n;
  }
  const int64_t clusters = P.n_pairs < s->max_clusters ? P.n_pairs : s->max_clusters;
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  return cudaLaunchKernelEx(&cfg, mlp_tc_kernel, P, s->tmap_unit, s->tmap_half);
}

}  // namespace nerfb
