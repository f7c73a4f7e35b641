// qmv on the tensor cores: the NVFP4 weight goes to tcgen05 block-scaled
// MMAs in its stored form (e2m1 codes by TMA, e4m3 block scales through
// tensor memory); nothing is decoded per weight on the SIMT cores.
//
// Same result as k_qmv (qmv.cuh):  y[m, n] = T( sum_b sd[n,b] * sum_{k in b}
// x_hat[m,k] * e2m1(q[n,k]) ),  sd = f8(s) * g_w / 2688.
//
// x_hat is written exactly as two e2m1 "planes" per 16-block:
//   x_hat_k = A_b * e2m1(pA_k) + B_b * e2m1(pB_k),
//   A_b = T(sdx_b), B_b = T(1.5 * sdx_b)  (sdx = f8(sx) * g_x / 2688),
// because T(v * sdx) = 2^i * T(u * sdx) for v = 2^i * u, u in {1, 1.5},
// whenever 0.5 |sdx| and 6 |sdx| lie in T's normal range (rounding to a
// binary format commutes with scaling by a power of two there, and the fp32
// product before the rounding to T scales the same way).  The prologue
// checks that range per block; if any block of x falls outside it (x_hat
// subnormal or overflowing), the CTA computes its rows with the SIMT loop
// instead, from an fp32 x_hat written over the plane tiles.  One MMA (M = 128 weight rows, N = 8 per x row, K = 64)
// per k-step then yields, for each of the k-step's 4 blocks and 2 planes,
//   D[n, (m, b, p)] = sum_{k in b} e2m1(q[n, k]) * e2m1(p_k)
// (unit block scales on both operands), written to fresh TMEM columns; the
// epilogue warps accumulate y[m, n] += U_(b,p) * (f8(sw[n, b]) * D) with U =
// A_b or B_b, and finally scale by g_w / 2688.  f8(sw) * D is exact in fp32
// (a 4-bit by 11-bit significand product: D is a multiple of 1/4 below 2^9),
// so this equals the block-scaled MMA's own output times U; applying the
// weight scales in the epilogue removes every per-stage scale copy from the
// tensor-core instruction stream, which is what bounds a CTA (each tcgen05
// instruction of these N = 8 shapes costs about as much as a small MMA).
//
// CTA = 128 weight rows; warps: 0 TMA producer (codes [128 x 128 B] per
// stage), 1 TMEM allocator + MMA issuer, 4-7 epilogue (TMEM lane quarters;
// each lane reads its weight row's LINEAR scale bytes straight from global
// memory, one ring half ahead).  Warp 0 first copies x into shared memory
// (one bulk copy, ahead of the weight in the memory queues) and then starts
// the weight stream; warps 1-11 compute the x_hat planes from that copy.
// TMEM: a ring of NSEG 128-column segments of MMA outputs, each drained by
// the epilogue as a whole, and one tile of unit scales used by both
// operands.  With three segments a segment is reused only after the
// epilogue has long drained it, so the MMA chain rarely waits on it.
//
// Every mbarrier wait of the MMA thread costs about as much as several of
// these small MMAs (its shared-memory access queues behind the tensor
// core's operand reads), so the MMA thread waits once per group of stages:
// the stages of a group complete on one barrier (the producer posts each
// stage's bytes on it; two such barriers alternate, and the ring holds two
// groups, so a group barrier is not reused before the MMA warp has passed
// its previous phase); segments that were never used are not waited on.
// The first group is small, so the MMAs start as soon as the x planes are
// ready; a stage's slot is released (commit) only when a later stage will
// reuse it.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "qmv.cuh"
#include "qqmm_sm100.cuh"

namespace nvfp4 {
namespace qtc {

constexpr int THREADS = 384;
constexpr int BM = 128;            // weight rows per CTA
constexpr int MAX_STAGES = 12;
constexpr int A_STAGE = BM * 128;  // 16 KiB of codes (256 K)
constexpr int STAGE_BYTES = A_STAGE;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t NSEG = 3;         // 128-column segments of MMA outputs: columns [0, 384)
constexpr uint32_t T_ONES = 384;     // unit block scales (both operands)

// shared memory carve-up (bytes, from a 1024-aligned base)
struct Layout {
  uint32_t stages, M, K;
  uint32_t ring, planes, uplane, ones, xraw, total;
  __host__ __device__ void init(uint32_t st, uint32_t m, uint32_t k, uint32_t esz) {
    stages = st;
    M = m;
    K = k;
    ring = 0;
    planes = stages * STAGE_BYTES;                 // 4 * M * K bytes (fp32 x_hat in the SIMT fallback)
    uplane = planes + 4u * M * K;                  // 2 * (K / 16) * M floats
    ones = uplane + 2u * (K / 16u) * M * 4u;       // 512 bytes of e4m3 1.0
    xraw = ones + 512u;                            // x as stored: M * K elements of esz bytes
    total = xraw + M * K * esz;
  }
};

__host__ __device__ inline uint32_t smem_needed(uint32_t stages, uint32_t M, uint32_t K, uint32_t esz) {
  Layout L;
  L.init(stages, M, K, esz);
  return L.total + 1024u;
}

// Stage groups: group 0 holds the first g0 stages, every later group g
// stages; all stages of a group complete on one barrier.
constexpr uint32_t NGRP = 4;  // group barriers, used round robin
struct Groups {
  uint32_t g0, g;
  __host__ __device__ uint32_t start(uint32_t grp) const { return grp == 0 ? 0u : g0 + (grp - 1u) * g; }
  __host__ __device__ uint32_t of(uint32_t kb) const { return kb < g0 ? 0u : 1u + (kb - g0) / g; }
  __host__ __device__ uint32_t count(uint32_t kb_count) const {
    return kb_count <= g0 ? 1u : 1u + (kb_count - g0 + g - 1u) / g;
  }
};

// Group sizes for a ring of S slots and kb_count stages: half the ring per
// group (on the 14336 x 4096 GEMV this timed 2-3 % faster than a small
// first group of 2 stages, with or without the PDL overlap); the smaller
// first groups are the fallbacks where half-ring groups are not valid.  No
// group may hold more than S stages (its stages are all in the ring before
// the MMA warp consumes any of them).  A group barrier is rearmed by the producer for
// group grp + NGRP only after the slot of a stage that group reuses was
// released, i.e. after the MMA warp consumed stage kb - S, which must lie
// in group grp or later, so that the MMA warp has already waited on group
// grp's phase.
inline Groups pick_groups(uint32_t S, uint32_t kb_count) {
  const uint32_t cand[3][2] = {{S / 2u, S / 2u}, {2u, S / 2u}, {2u, 4u}};
  for (auto& c : cand) {
    Groups gr{c[0], c[1]};
    if (gr.g == 0 || gr.g0 == 0 || gr.g > S || gr.g0 > S) continue;
    bool ok = true;
    for (uint32_t kb = S; kb < kb_count && ok; ++kb) ok = gr.of(kb - S) + NGRP > gr.of(kb);
    if (ok) return gr;
  }
  return Groups{S / 2u, S / 2u};
}

struct Args {
  const void* x;
  const float* g_x;
  const uint32_t* wc;
  const uint8_t* wsc;
  const float* g_w;
  void* y;
  uint32_t M, N, K, stages;
  uint32_t g0, g;  // stage groups (pick_groups)
};

// K-major operand without swizzle: 8-row x 16-byte core matrices, `lbo`
// bytes between core matrices along K, `sbo` between 8-row groups.
__device__ __forceinline__ uint64_t kmajor_plain_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return tc::smem_desc(addr, lbo, sbo, 0);
}

// Normal range of T: the plane form of x_hat is exact for a block whose
// decode scale sdx has 0.5 |sdx| >= kMinNormal and 6 |sdx| <= kMaxFinite.
template <typename T> struct Range;
template <> struct Range<float> {
  static constexpr float kMinNormal = 0x1p-126f, kMaxFinite = 0x1.fffffep127f;
};
template <> struct Range<__half> {
  static constexpr float kMinNormal = 0x1p-14f, kMaxFinite = 65504.0f;
};
template <> struct Range<__nv_bfloat16> {
  static constexpr float kMinNormal = 0x1p-126f, kMaxFinite = 0x1.fep127f;
};

// x_hat = quantize-dequantize(x, g_x) of all M rows as plane codes and
// plane scales (layout in the header comment), from x staged in shared
// memory.  One thread per 16-element block; threads 32.. (warps 1 and up)
// take part, warp 0 streams the weight.  Returns false on a thread that met
// a block outside the exact range.
template <typename T>
__device__ __forceinline__ bool x_planes(const T* xs, float gx, uint32_t M, uint32_t K, uint8_t* planes,
                                         float* uplane) {
  const float E = kGlobalEncode / gx;
  const float d = gx / kGlobalEncode;
  const uint32_t n_blk = M * K / 16u;
  const uint32_t nb = K / 16u;
  bool exact = true;
  const uint32_t nthr = blockDim.x - 32u;  // warps 1 and up
  for (uint32_t blk = threadIdx.x - 32u; threadIdx.x >= 32u && blk < n_blk; blk += nthr) {
    float v[16];
    {
      float lo[8], hi[8];
      load8_shared<T>(xs + (size_t)blk * 16, lo);
      load8_shared<T>(xs + (size_t)blk * 16 + 8, hi);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[j] = lo[j];
        v[8 + j] = hi[j];
      }
    }
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(v[j]));
    const float t = (a / kE2M1Max) * E;
    const float fs = e4m3_to_f32(f32_to_e4m3(t));
    const float sd = fs * d;
    uint32_t w[2] = {0u, 0u};
    if (fs != 0.0f) {
      const float k = E / fs;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = v[8 * hf + j] * k;
        w[hf] = f32x8_to_e2m1x8(q);
      }
    }
    const float asd = fabsf(sd);
    exact = exact && (sd == 0.0f || (0.5f * asd >= Range<T>::kMinNormal && 6.0f * asd <= Range<T>::kMaxFinite));
    // codes of magnitude 1.5, 3, 6 (odd magnitude code >= 3) go to plane B
    // as 1, 2, 4 (the code minus one); all others stay in plane A
    uint32_t pa[2], pbw[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t odd3 = w[hf] & 0x11111111u & ((w[hf] >> 1) | (w[hf] >> 2));
      const uint32_t mask = odd3 * 15u;
      pa[hf] = w[hf] & ~mask;
      pbw[hf] = (w[hf] - odd3) & mask;
    }
    // plane tile of k-step g = k0/64, block bl = (k0/16)%4; the block's two
    // code words are 8 contiguous bytes of its plane row
    const uint32_t m = (blk * 16u) / K, k0 = blk * 16u - m * K;
    const uint32_t g = k0 >> 6, bl = (k0 >> 4) & 3u;
    uint8_t* tile = planes + (size_t)g * 256u * M;  // [h][row group][8 rows][16 B], rows = m*8 + bl*2 + p
    const uint32_t h = bl >> 1, byte = 8u * (bl & 1u);
    const uint32_t rowA = m * 8u + bl * 2u, rowB = rowA + 1u;
    *reinterpret_cast<uint2*>(tile + h * 128u * M + (rowA >> 3) * 128u + (rowA & 7u) * 16u + byte) =
        make_uint2(pa[0], pa[1]);
    *reinterpret_cast<uint2*>(tile + h * 128u * M + (rowB >> 3) * 128u + (rowB & 7u) * 16u + byte) =
        make_uint2(pbw[0], pbw[1]);
    const uint32_t b = k0 >> 4;
    uplane[m * 2u * nb + 2u * b] = Elem<T>::to_f(Elem<T>::from_f(sd));
    uplane[m * 2u * nb + 2u * b + 1u] = Elem<T>::to_f(Elem<T>::from_f(1.5f * sd));
  }
  return exact;
}

// PDL = true: the kernel is launched with programmatic stream serialization
// (qmv_pdl).  Its weight codes, weight scales and g_w are read without
// waiting for the previous kernel of the stream (the caller guarantees that
// no pending work writes them); x, g_x and y only after griddepcontrol.wait
// (all prerequisite grids complete, their writes visible).  Each CTA lets
// the next launch begin at once (launch_dependents), so a chain of calls
// streams the next weight while the previous call drains.
template <typename T, int MM, bool PDL = false>
__global__ void __launch_bounds__(THREADS, 1) k_qmv_tc(const __grid_constant__ CUtensorMap tmap_w, Args a) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t gfull[NGRP];  // all stages of a group landed
  __shared__ __align__(8) uint64_t empty_bar[MAX_STAGES];
  __shared__ __align__(8) uint64_t dfull_bar[NSEG];
  __shared__ __align__(8) uint64_t dempty_bar[NSEG];
  __shared__ __align__(8) uint64_t xbar;  // x landed in shared memory
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;

  float gx = kGlobalEncode;
  if (!PDL) gx = a.g_x ? __ldg(a.g_x) : kGlobalEncode;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Layout L;
  L.init(a.stages, MM, a.K, (uint32_t)sizeof(T));
  const uint32_t xbytes = a.M * a.K * (uint32_t)sizeof(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t row0 = blockIdx.x * BM;
  const uint32_t S = a.stages;
  const uint32_t kb_count = a.K / 256u;   // stages of 256 K
  const uint32_t ksteps = a.K / 64u;      // MMAs
  const uint32_t ncols = 8u * MM;         // MMA N
  const uint32_t steps_per_half = 128u / ncols;
  const uint32_t nb = a.K / 16u;
  const Groups GR{a.g0, a.g};
  const uint32_t groups = GR.count(kb_count);

  // stage kb into ring slot kb % S; its bytes complete on its group's
  // barrier (group grp on gfull[grp % NGRP], phase (grp / NGRP) & 1); the
  // group's last stage (or the last stage of all) also arrives
  auto issue = [&](uint32_t kb) {
    const uint32_t grp = GR.of(kb), bar = smem_u32(&gfull[grp % NGRP]);
    if (kb + 1 == GR.start(grp + 1) || kb + 1 == kb_count) mbar_expect_tx(bar, A_STAGE);
    else asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(A_STAGE) : "memory");
    tma_load_2d(sbase + L.ring + (kb % S) * STAGE_BYTES, &tmap_w, (int)(kb * 128u), (int)row0, bar);
  };
  // the latest phases of the group barriers (all copies still in flight
  // belong to the last NGRP groups issued); after an abort the last group
  // may lack its arriving stage, so the producer arrives for it first
  auto drain = [&](uint32_t issued) {
    if (issued == 0) return;
    const uint32_t last = GR.of(issued - 1);
    if (issued != kb_count && GR.start(last + 1) != issued)
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&gfull[last % NGRP])) : "memory");
    for (uint32_t gr = last + 1 > NGRP ? last + 1 - NGRP : 0; gr <= last; ++gr)
      mbar_wait(smem_u32(&gfull[gr % NGRP]), (gr / NGRP) & 1u);
  };

  uint32_t issued = 0;  // weight stages issued (thread 0)
  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < S; ++s) mbar_init(smem_u32(&empty_bar[s]), 1);
    for (uint32_t i = 0; i < NGRP; ++i) mbar_init(smem_u32(&gfull[i]), 1);
    for (uint32_t h = 0; h < NSEG; ++h) {
      mbar_init(smem_u32(&dfull_bar[h]), 1);
      mbar_init(smem_u32(&dempty_bar[h]), 4);
    }
    mbar_init(smem_u32(&xbar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (PDL) {
      // the weight before the wait for the previous kernel, x after it
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
      for (; issued < S && issued < kb_count; ++issued) issue(issued);
      asm volatile("griddepcontrol.wait;" ::: "memory");
      mbar_expect_tx(smem_u32(&xbar), xbytes);
      bulk_load(sbase + L.xraw, a.x, xbytes, smem_u32(&xbar));
    } else {
      // x first, one bulk copy (the rows are contiguous, 16-byte aligned and
      // a multiple of 512 bytes long), so it does not queue behind the weight
      // stream; then the weight stream, before TMEM allocation and the prologue
      mbar_expect_tx(smem_u32(&xbar), xbytes);
      bulk_load(sbase + L.xraw, a.x, xbytes, smem_u32(&xbar));
      for (; issued < S && issued < kb_count; ++issued) issue(issued);
    }
  }
  if (PDL) {
    // every thread that reads g_x, or later x_hat's inputs or writes y
    asm volatile("griddepcontrol.wait;" ::: "memory");
    gx = a.g_x ? __ldg(a.g_x) : kGlobalEncode;
  }
  // zero the plane tiles (a plane row is nonzero only inside its own
  // 16-block: the prologue writes those bytes alone), fill the unit scale tile
  {
    uint4* z = reinterpret_cast<uint4*>(smem + L.planes);
    const uint32_t nz = (L.uplane - L.planes) / 16u;
    for (uint32_t i = threadIdx.x; i < nz; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    uint4* o = reinterpret_cast<uint4*>(smem + L.ones);
    if (threadIdx.x < 32) o[threadIdx.x] = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to tcgen05.cp
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  bool mine = true;
  if (warp >= 1) {
    mine = mbar_wait(smem_u32(&xbar), 0);
    if (!mine) abort_flag = 1;
    else
      mine = x_planes<T>(reinterpret_cast<const T*>(smem + L.xraw), gx, a.M, a.K, smem + L.planes,
                         reinterpret_cast<float*>(smem + L.uplane));
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // planes are read by the tensor core
  const bool exact = __syncthreads_and(mine) != 0;
  const float dw = a.g_w ? __ldg(a.g_w) / kGlobalEncode : 1.0f;

  if (!exact) {
    // x_hat outside the planes' exact range: fp32 x_hat over the plane tiles
    // and SIMT rows for this CTA, after the loads in flight have landed
    float4* xs4 = reinterpret_cast<float4*>(smem + L.planes);
    qmv_prologue<T>(static_cast<const T*>(a.x), a.g_x, a.M, a.K, xs4, threadIdx.x, blockDim.x);
    if (threadIdx.x == 0) {
      drain(issued);
      mbar_wait(smem_u32(&xbar), 0);  // x's copy has landed (a no-op unless its wait above gave up)
    }
    __syncthreads();
    const uint32_t end = min(row0 + BM, a.N);
    qmv_simt_rows<T, MM>(xs4, a.wc, a.wsc, dw, a.M, a.N, a.K, static_cast<T*>(a.y), row0 + warp,
                         THREADS / 32, end);
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (uint32_t kb = issued; kb < kb_count; ++kb) {
        const uint32_t s = kb % S;
        if (!mbar_wait(smem_u32(&empty_bar[s]), ((kb / S) & 1u) ^ 1u) || *(volatile int*)&abort_flag) {
          abort_flag = 1;
          break;
        }
        issue(kb);
        issued = kb + 1;
      }
      drain(issued);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and one elected lane issues.  The wait
    // for a drained ring half sits at a stage boundary (a half holds a
    // multiple of 4 k-steps), so each stage issues straight-line code.
    const bool leader = elect_one();
    if (leader) tmem_cp_sf(tmem + T_ONES, sf_tile_desc(sbase + L.ones));
    const uint32_t idesc = (1u << 7) | (1u << 10) | ((ncols >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    const uint64_t a_base = kmajor_sw128_desc(sbase + L.ring);
    const uint64_t b_base = kmajor_plain_desc(sbase + L.planes, 128u * MM, 128u);
    const uint32_t a_hi = (uint32_t)(a_base >> 32), b_hi = (uint32_t)(b_base >> 32);
    auto mk = [](uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; };
    uint32_t g = 0;  // global k-step
    bool ok = true;
    for (uint32_t grp = 0; grp < groups && ok; ++grp) {
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&gfull[grp % NGRP]), (grp / NGRP) & 1u)) ||
          *(volatile int*)&abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t kb1 = min(GR.start(grp + 1), kb_count);
      for (uint32_t kb = GR.start(grp); kb < kb1; ++kb) {
        const uint32_t s = kb % S;
        const uint32_t seg = g / steps_per_half;          // segment use number
        const uint32_t hf = seg % NSEG;                   // ring segment of this stage
        const uint32_t use = seg / NSEG;                  // times this segment was used before
        if (g % steps_per_half == 0 && use > 0) {         // reuse: wait until the segment is drained
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&dempty_bar[hf]), (use & 1u) ^ 1u))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (leader) {
          const uint32_t dcol = hf * 128u + (g % steps_per_half) * ncols;
#pragma unroll
          for (uint32_t j = 0; j < 4; ++j)
            mma_block_scaled<kNV>(tmem + dcol + j * ncols,
                                    mk((uint32_t)a_base + ((s * STAGE_BYTES + 32u * j) >> 4), a_hi),
                                    mk((uint32_t)b_base + (((g + j) * 256u * MM) >> 4), b_hi), idesc, tmem + T_ONES,
                                    tmem + T_ONES, 0u);
          if ((g + 4) % steps_per_half == 0 || g + 4 == ksteps) mma_commit(smem_u32(&dfull_bar[hf]));
          if (kb + S < kb_count) mma_commit(smem_u32(&empty_bar[s]));  // the slot is refilled later
        }
        __syncwarp();
        g += 4;
      }
    }
    if (!ok && leader) abort_flag = 1;
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    constexpr int NC = 8 * MM;              // MMA output columns per k-step
    constexpr int SPH = 128 / NC;           // k-steps per ring half (16 or 8)
    const uint32_t q = warp & 3;
    const float* U = reinterpret_cast<const float*>(smem + L.uplane);
    const uint32_t n = row0 + q * 32u + lane;
    // this lane's weight row of LINEAR scales (a row past N reads row N-1:
    // its codes were loaded as zeros, so the products vanish)
    const uint8_t* srow = a.wsc + (size_t)min(n, a.N - 1u) * nb;
    float acc[MM];
#pragma unroll
    for (int m = 0; m < MM; ++m) acc[m] = 0.0f;
    const uint32_t halves = (ksteps + steps_per_half - 1) / steps_per_half;
    auto load_scales = [&](uint32_t h, uint4 (&sc)[SPH / 4]) {
#pragma unroll
      for (int j = 0; j < SPH / 4; ++j) {
        const uint32_t off = 4u * h * (uint32_t)SPH + 16u * (uint32_t)j;  // 4 scale bytes per k-step
        sc[j] = off < nb ? __ldg(reinterpret_cast<const uint4*>(srow + off)) : make_uint4(0, 0, 0, 0);
      }
    };
    uint4 sc[SPH / 4];
    load_scales(0, sc);
    bool ok = true;
    for (uint32_t h = 0; h < halves; ++h) {
      const uint32_t hf = h % NSEG;
      uint4 cur[SPH / 4];
#pragma unroll
      for (int j = 0; j < SPH / 4; ++j) cur[j] = sc[j];
      if (h + 1 < halves) load_scales(h + 1, sc);  // next half's scales in flight
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&dfull_bar[hf]), (h / NSEG) & 1u)) &&
           !*(volatile int*)&abort_flag;
      tc_fence_after();
      if (!ok) break;
      const uint32_t g0 = h * steps_per_half;
      const uint32_t nsteps = min(steps_per_half, ksteps - g0);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {  // 32-column chunks of the half
        if ((uint32_t)(cc * 32) < nsteps * ncols) {
          float v[32];
          tmem_ld32(tmem + ((q * 32u) << 16) + hf * 128u + (uint32_t)(cc * 32), v);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {  // (plane A, plane B) of one block
            const int m = (i % NC) >> 3, bl = (i & 7) >> 1;
            const int kl = cc * 32 / NC + i / NC;  // k-step within the half
            const int byte = 4 * kl + bl;          // its scale byte within the half
            const uint4 w4 = cur[byte >> 4];
            const uint32_t word = ((byte >> 2) & 3) == 0 ? w4.x : ((byte >> 2) & 3) == 1 ? w4.y
                                  : ((byte >> 2) & 3) == 2 ? w4.z : w4.w;
            const float sw = e4m3_to_f32(word >> (8 * (byte & 3)));
            const uint32_t ub = (uint32_t)m * 2u * nb + 8u * (g0 + (uint32_t)kl) + 2u * (uint32_t)bl;
            acc[m] = fmaf(U[ub], v[i] * sw, acc[m]);
            acc[m] = fmaf(U[ub + 1u], v[i + 1] * sw, acc[m]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&dempty_bar[hf])) : "memory");
    }
    if (ok && n < a.N) {
#pragma unroll
      for (int m = 0; m < MM; ++m)
        if ((uint32_t)m < a.M) static_cast<T*>(a.y)[(size_t)m * a.N + n] = Elem<T>::from_f(acc[m] * dw);
    }
  }
  __syncwarp();  // lanes that skipped a one-lane role loop wait for it before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

// Tensor map of the weight codes [N, K/2 bytes] (box 128 B x 128 rows,
// 128-byte swizzle).
inline bool make_map(CUtensorMap* mw, const uint32_t* wc, uint64_t N, uint64_t K) {
  auto fn = tc::encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K / 2, N};
  cuuint64_t strides[1] = {K / 2};
  cuuint32_t box[2] = {128, BM};
  cuuint32_t estr[2] = {1, 1};
  return fn(mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(wc), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stages that fit next to the plane tiles, plane scales and x (elements of
// esz bytes); 0 if the tensor-core path does not apply (then the caller runs
// the SIMT kernel).
inline uint32_t pick_stages(int64_t M, int64_t K, uint32_t esz) {
  if (M < 1 || M > 2 || K % 256 != 0 || K < 256) return 0;
  const uint32_t MM = M == 1 ? 1u : 2u;
  for (uint32_t st = MAX_STAGES; st >= 2; st -= 2)  // even: two groups of st / 2 stages
    if (smem_needed(st, MM, (uint32_t)K, esz) <= 227u * 1024u) return st;
  return 0;
}

}  // namespace qtc
}  // namespace nvfp4
