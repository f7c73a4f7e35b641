// Dense block-scaled quantized matmul on the 5th-generation tensor cores
// (tcgen05), sm_100a.
//
//   y[m, n] = alpha * sum_b sx[m, b] * sw[n, b] * sum_{k in b} qx[m, k] * qw[n, k]
//
// NVFP4: e2m1 codes, ue4m3 scales per 16 elements, alpha = (g_x / 2688) *
// (g_w / 2688) (the device alpha of compute_qqmm_pointers, "mlx 0.30.7.2 ->
// 0.30.7.6" diff, page 7, qqmm_utils.cu).  MXFP8: e4m3 codes, ue8m0 scales per
// 32 elements, alpha = 1.  MXFP4: e2m1 codes, ue8m0 scales per 32 elements
// (kind::mxf4nvf4 .block32: two scale bytes per K = 64 step, picked by the
// scale-factor id), alpha = 1.  Folding the global scales into alpha is exact in
// real arithmetic (sum (c sx dx)(c sw dw) = dx dw sum c sx c sw), and no
// operand is rounded to a narrower type on this path, so it is equivalent to
// decoding each block with its global scale.
//
// Kernel structure (persistent: one CTA per SM loops over 128 x 256 output
// tiles; 352 threads):
//   warp 0   TMA producer: per K stage, A codes [128 rows x 128 B] and B codes
//            [256 rows x 128 B] as 128-byte-swizzled tiles; it also posts
//            the stage's expected bytes, scale tiles included.
//   warp 10  scale producer: the stage's scale tiles as plain bulk copies
//            (the 128x4 scale-tile layout of the operands is already the
//            order the MMA's scale tensor memory expects, so the copies are
//            contiguous 512-byte blocks).  Each TMA issue occupies its thread
//            for on the order of a hundred cycles; with all five copies of a
//            stage on one thread the issue loop, not the tensor core, set the
//            stage rate, so the copies are split over two warps.
//   warp 1   TMEM allocator and MMA issuer: one elected lane of the
//            converged warp moves the stage's
//            scale tiles into tensor memory (tcgen05.cp 32x128b.warpx4) and
//            issues the block-scaled MMAs (M=128, N=256, K=64 NVFP4 and
//            MXFP4 / 32 MXFP8 per instruction) into a 128 x 256 fp32
//            accumulator in TMEM;
//            tcgen05.commit frees the stage when its MMAs are done.
//   warps 2-9 epilogue: two warps per TMEM lane quarter (warp w reads lanes
//            32*(w%4)...), 128 accumulator columns each; they drain the
//            accumulator into registers, release it to the MMA warp at once
//            (so the next tile's MMAs start), then apply alpha, convert and
//            store while the tensor core works on the next tile: 32 rows x
//            32 bytes at a time staged in the warp's shared-memory box and
//            written by a TMA tensor store (direct stores when the output's
//            row pitch is not a multiple of 16 bytes).
// Every mbarrier wait is bounded; on timeout the kernel sets the device
// error word (NVFP4_ERR_TIMEOUT through nvfp4_check_device_errors), drains,
// frees its TMEM and exits.  No cluster multicast is used.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "nvfp4.h"

namespace nvfp4 {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BKB = 128;  // bytes of K per row per stage (256 FP4 / 128 FP8 elements)
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 8;
constexpr int W_SCALES = 2 + EPI_WARPS;         // the scale producer warp
constexpr int THREADS = 96 + 32 * EPI_WARPS;     // producer, MMA, 8 epilogue warps, scale producer
constexpr int A_STAGE = BM * BKB;    // 16 KiB
constexpr int B_STAGE = BN * BKB;    // 32 KiB
constexpr int SFA_STAGE = 4 * 512;   // up to 4 scale tiles (NVFP4)
constexpr int SFB_STAGE = 2 * 4 * 512;
constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_STAGE;
constexpr int SMEM_SFA = SMEM_B + STAGES * B_STAGE;
constexpr int SMEM_SFB = SMEM_SFA + STAGES * SFA_STAGE;
constexpr int SMEM_EPI = SMEM_SFB + STAGES * SFB_STAGE;
constexpr int EPI_BUF = 32 * 32;  // per epilogue warp: 32 rows x 32 bytes of output
constexpr int SMEM_BYTES = SMEM_EPI + EPI_WARPS * EPI_BUF;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_SF = 256;       // scale-factor columns start here
constexpr uint32_t TMEM_SF_STAGE = 48;  // 16 (A) + 32 (B) columns per stage
// Polls of a bounded mbarrier wait before it gives up.  A test build of the
// library lowers it (-DNVFP4_WAIT_LIMIT=...) so that a withheld stage (below)
// times out within milliseconds.
#ifndef NVFP4_WAIT_LIMIT
#define NVFP4_WAIT_LIMIT (1u << 26)
#endif
constexpr uint32_t kWaitLimit = NVFP4_WAIT_LIMIT;

// Test builds only (-DNVFP4_TEST_WITHHOLD_STAGE=s): CTA 0 of the dense GEMM
// issues neither the arrival nor any copy of its stage s, so the MMA warp's
// bounded wait on that stage runs out and the kernel takes its timeout path
// (error word, drain, TMEM freed).  No copy is left in flight: nothing is
// issued for the withheld stage.  The library itself is built without it.
__device__ __forceinline__ bool withheld_stage(uint32_t it) {
#ifdef NVFP4_TEST_WITHHOLD_STAGE
  return blockIdx.x == 0 && it == (uint32_t)(NVFP4_TEST_WITHHOLD_STAGE);
#else
  (void)it;
  return false;
#endif
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false (and the device error word set) if the phase never
// completes.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
  return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Tensor store of a 2-D box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Shared-memory matrix descriptor of tcgen05 (start >> 4 in bits 0-13,
// leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// version 1 in bits 46-47, layout type in 61-63).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// K-major operand tile, 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t addr) { return smem_desc(addr, 16, 1024, 2); }
// A 512-byte scale tile: 32 rows of 16 bytes, no swizzle (8-row core
// matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_tile_desc(uint32_t addr) { return smem_desc(addr, 0, 128, 0); }

// Instruction descriptor of the block-scaled MMA: A/B formats (bits 7-9,
// 10-12), K-major A and B, N >> 3 (bits 17-22), scale format (bit 23:
// 0 = ue4m3, 1 = ue8m0), M >> 4 (bits 24-28), scale-factor byte ids of B
// (bits 4-5) and A (bits 29-30).
__host__ __device__ constexpr uint32_t block_scaled_idesc(uint32_t ab_format, uint32_t scale_ue8m0, uint32_t sf_id,
                                                         uint32_t n = BN) {
  return (sf_id << 4) | (ab_format << 7) | (ab_format << 10) | ((n >> 3) << 17) | (scale_ue8m0 << 23) |
         ((uint32_t)(BM >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Operand kinds of the dense GEMM: NVFP4 (e2m1, ue4m3 per 16), MXFP8 (e4m3,
// ue8m0 per 32), MXFP4 (e2m1, ue8m0 per 32).
enum { kNV = 0, kMX8 = 1, kMX4 = 2 };

template <int KIND>
__device__ __forceinline__ void mma_block_scaled(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if constexpr (KIND == kMX4) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  } else if constexpr (KIND == kMX8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  }
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// One lane of a converged warp, for issuing single-thread tensor-core
// instructions while the whole warp runs the issue loop (so the loop's
// values stay warp-uniform).
__device__ __forceinline__ bool elect_one() {
  uint32_t p = 0;
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.u32 %0, 1, 0, e;\n\t}" : "=r"(p));
  return p != 0;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct Params {
  const uint8_t* sfa;  // SWIZZLED scale buffers
  const uint8_t* sfb;
  const float* g_x;
  const float* g_w;
  void* y;
  int M, N, K;
  int y_dt;             // nvfp4_dtype
  uint32_t kb_count;    // K stages
  uint32_t k_bytes;     // bytes of K per row (K/2 NVFP4, K MXFP8)
  uint32_t sf_groups;   // Cp / 4: scale-tile columns per 128-row block
  uint32_t rows_b_pad;  // ceil128(N)
  int tma_store;        // 1: y is written through tmap_y (row pitch a multiple of 16 bytes)
  uint32_t nfull;       // work units that are whole 128 x 256 tiles
  uint32_t units;       // all work units: nfull + 2 x (tiles split into 128 x 128 halves)
};

template <typename T>
__device__ __forceinline__ void store_out(T* dst, const float* v, int n);

template <>
__device__ __forceinline__ void store_out<float>(float* dst, const float* v, int n) {
  if (n == 32 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  } else {
    for (int i = 0; i < n; ++i) dst[i] = v[i];
  }
}

template <typename T>
__device__ __forceinline__ void store_out_16(T* dst, const float* v, int n) {
  if (n == 32 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = v[i + j];
      store8<T>(dst + i, t);
    }
  } else {
    for (int i = 0; i < n; ++i) dst[i] = Elem<T>::from_f(v[i]);
  }
}

template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* dst, const float* v, int n) {
  store_out_16<__nv_bfloat16>(dst, v, n);
}
template <>
__device__ __forceinline__ void store_out<__half>(__half* dst, const float* v, int n) {
  store_out_16<__half>(dst, v, n);
}

// Epilogue of one warp: its 32 accumulator rows (one per lane, starting at
// row0) x 128 columns (starting at col0), scaled by alpha and rounded to y's
// type.  With p.tma_store the warp stages 32 rows x 32 bytes at a time in
// its 1 KiB shared buffer `buf` and the TMA writes the box (whole sectors;
// rows >= M and columns >= N of the box are clipped by the tensor map); each
// lane writes its row's two 16-byte halves in an order that keeps every
// 8-lane phase of the shared store free of bank conflicts.  Otherwise each
// lane stores its row directly.
__device__ __forceinline__ void epilogue_store(const Params& p, const CUtensorMap* tmap_y, uint32_t buf,
                                               const float (&v)[128], float alpha, int row0, int col0, int lane) {
  if (row0 >= p.M) return;
  if (p.tma_store) {
    const uint32_t rbase = buf + (uint32_t)lane * 32u;
    const bool swap = (lane >> 2) & 1;
    auto put = [&](int col, uint4 h0, uint4 h1) {
      if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      __syncwarp();
      st_shared_v4(rbase + (swap ? 16u : 0u), swap ? h1 : h0);
      st_shared_v4(rbase + (swap ? 0u : 16u), swap ? h0 : h1);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) tma_store_2d(tmap_y, buf, col, row0);
    };
    if (p.y_dt == NVFP4_DT_F32) {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int col = col0 + c * 8;
        if (col >= p.N) break;
        const float* o = v + c * 8;
        put(col,
            make_uint4(__float_as_uint(o[0] * alpha), __float_as_uint(o[1] * alpha), __float_as_uint(o[2] * alpha),
                       __float_as_uint(o[3] * alpha)),
            make_uint4(__float_as_uint(o[4] * alpha), __float_as_uint(o[5] * alpha), __float_as_uint(o[6] * alpha),
                       __float_as_uint(o[7] * alpha)));
      }
    } else {
      const bool bf = p.y_dt == NVFP4_DT_BF16;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int col = col0 + c * 16;
        if (col >= p.N) break;
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float lo = v[c * 16 + 2 * i] * alpha, hi = v[c * 16 + 2 * i + 1] * alpha;
          w[i] = bf ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
        }
        put(col, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
      }
    }
    return;
  }
  const int row = row0 + lane;
  if (row >= p.M) return;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int col = col0 + c * 32;
    if (col < p.N) {
      const int n = min(32, p.N - col);
      float o[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = v[c * 32 + i] * alpha;
      const size_t off = (size_t)row * p.N + col;
      if (p.y_dt == NVFP4_DT_F32) store_out<float>(static_cast<float*>(p.y) + off, o, n);
      else if (p.y_dt == NVFP4_DT_BF16) store_out<__nv_bfloat16>(static_cast<__nv_bfloat16*>(p.y) + off, o, n);
      else store_out<__half>(static_cast<__half*>(p.y) + off, o, n);
    }
  }
}

// Tile t of the persistent schedule -> (m tile, n tile): groups of 8 M tiles
// sweep all N tiles, so the CTAs running at the same time share A and B
// tiles in L2.
__device__ __forceinline__ void tile_coords(uint32_t t, uint32_t mt, uint32_t nt, uint32_t& tm, uint32_t& tn) {
  const uint32_t group = t / (8u * nt);
  const uint32_t first_m = group * 8u;
  const uint32_t gm = min(8u, mt - first_m);
  const uint32_t r = t - group * 8u * nt;
  tm = first_m + r % gm;
  tn = r / gm;
}

// Work unit u of the persistent schedule -> output tile.  Units below
// p.nfull are 128 x 256 tiles in tile_coords order.  The tiles after them
// (the last, partial wave of wide tiles) are split into their two 128 x 128
// halves, one unit each, so that wave runs on up to twice as many SMs for
// about half as long.  n0 is the first output column; false for a half that
// lies wholly beyond N (every role skips it).
__device__ __forceinline__ bool unit_coords(uint32_t u, const Params& p, uint32_t mt, uint32_t nt, uint32_t& tm,
                                            uint32_t& n0, bool& wide) {
  uint32_t tn;
  if (u < p.nfull) {
    tile_coords(u, mt, nt, tm, tn);
    n0 = tn * BN;
    wide = true;
    return true;
  }
  const uint32_t s = u - p.nfull;
  tile_coords(p.nfull + s / 2u, mt, nt, tm, tn);
  n0 = tn * BN + (s & 1u) * 128u;
  wide = false;
  return n0 < (uint32_t)p.N;
}

template <int KIND>
__global__ void __launch_bounds__(THREADS, 1) k_qqmm(const __grid_constant__ CUtensorMap tmap_a,
                                                     const __grid_constant__ CUtensorMap tmap_b,
                                                     const __grid_constant__ CUtensorMap tmap_b128,
                                                     const __grid_constant__ CUtensorMap tmap_y, Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t accum_full;
  __shared__ __align__(8) uint64_t accum_empty;
  __shared__ uint32_t tmem_base_holder;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t mt = ((uint32_t)p.M + BM - 1) / BM, nt = ((uint32_t)p.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&accum_full), 1);
    mbar_init(smem_u32(&accum_empty), EPI_WARPS);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_holder;
  const uint32_t tiles_per_stage = KIND == kNV ? 4u : KIND == kMX8 ? 1u : 2u;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;  // global stage counter across tiles
      for (uint32_t u = blockIdx.x; u < p.units && !*(volatile int*)&abort_flag; u += gridDim.x) {
        uint32_t tm, n0;
        bool wide;
        if (!unit_coords(u, p, mt, nt, tm, n0, wide)) continue;
        const int tile_m = (int)(tm * BM), tile_n = (int)n0;
        const bool b_second = wide && (uint32_t)(tile_n + 128) < p.rows_b_pad;
        for (uint32_t kb = 0; kb < p.kb_count; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / STAGES) & 1u) ^ 1u)) {
            abort_flag = 1;
            break;
          }
          const uint32_t g0 = kb * tiles_per_stage;
          uint32_t ntl = p.sf_groups > g0 ? p.sf_groups - g0 : 0;
          if (ntl > tiles_per_stage) ntl = tiles_per_stage;
          const uint32_t sfa_bytes = ntl * 512u, sfb_bytes = ntl * 512u * (b_second ? 2u : 1u);
          const uint32_t bar = smem_u32(&full_bar[s]);
          if (withheld_stage(it)) continue;
          mbar_expect_tx(bar, A_STAGE + (wide ? B_STAGE : B_STAGE / 2) + sfa_bytes + sfb_bytes);
          tma_load_2d(sbase + SMEM_A + s * A_STAGE, &tmap_a, (int)(kb * BKB), tile_m, bar);
          tma_load_2d(sbase + SMEM_B + s * B_STAGE, wide ? &tmap_b : &tmap_b128, (int)(kb * BKB), tile_n, bar);
        }
      }
      // drain: the last STAGES issued stages must have landed before exit
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
      for (uint32_t i = first; i < it; ++i) mbar_wait(smem_u32(&full_bar[i % STAGES]), (i / STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (its values stay warp-uniform) and one
    // elected lane issues the tensor-core instructions.  The loop is kept
    // lean: descriptors are built once and advanced by adding byte offsets
    // >> 4 to their low 32-bit word (start address field); stage offsets
    // advance incrementally.
    {
      const bool leader = elect_one();
      const uint64_t a_base = kmajor_sw128_desc(sbase + SMEM_A), b_base = kmajor_sw128_desc(sbase + SMEM_B);
      const uint64_t sfa_base = sf_tile_desc(sbase + SMEM_SFA), sfb_base = sf_tile_desc(sbase + SMEM_SFB);
      const uint32_t a_hi = (uint32_t)(a_base >> 32), b_hi = (uint32_t)(b_base >> 32);
      const uint32_t sfa_hi = (uint32_t)(sfa_base >> 32), sfb_hi = (uint32_t)(sfb_base >> 32);
      auto mk = [](uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; };
      uint32_t it = 0, tile_i = 0, s = 0, ph = 0;
      bool ok = true;
      for (uint32_t u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        uint32_t tm, n0;
        bool wide;
        if (!unit_coords(u, p, mt, nt, tm, n0, wide)) continue;
        const bool b_second = wide && (uint32_t)(n0 + 128) < p.rows_b_pad;
        const uint32_t nmma = wide ? (uint32_t)BN : 128u;                 // MMA N of this unit
        const uint32_t idesc_nv = block_scaled_idesc(1u, 0u, 0u, nmma);  // e2m1 x e2m1, ue4m3
        // the epilogue has drained the previous tile's accumulator
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&accum_empty), (tile_i & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        for (uint32_t kb = 0; kb < p.kb_count; ++kb, ++it) {
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full_bar[s]), ph))) {
            abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
          const uint32_t tsfa = tmem + TMEM_SF + s * TMEM_SF_STAGE, tsfb = tsfa + 16;
          const uint32_t sfa_lo = (uint32_t)sfa_base + s * (SFA_STAGE >> 4);
          const uint32_t sfb_lo = (uint32_t)sfb_base + s * (SFB_STAGE >> 4);
          const uint32_t a_lo = (uint32_t)a_base + s * (A_STAGE >> 4), b_lo = (uint32_t)b_base + s * (B_STAGE >> 4);
          const uint32_t g0 = kb * tiles_per_stage;
          if (g0 + tiles_per_stage <= p.sf_groups && p.k_bytes >= (kb + 1) * BKB) {
            // full stage: all scale tiles and all four k-steps present
            if constexpr (KIND == kMX8) {
              tmem_cp_sf(tsfa, mk(sfa_lo, sfa_hi));
              tmem_cp_sf(tsfb, mk(sfb_lo, sfb_hi));
              if (b_second) tmem_cp_sf(tsfb + 4, mk(sfb_lo + (4 * 512 >> 4), sfb_hi));
#pragma unroll
              for (uint32_t j = 0; j < 4; ++j)
                mma_block_scaled<kMX8>(tmem, mk(a_lo + 2 * j, a_hi), mk(b_lo + 2 * j, b_hi),
                                       block_scaled_idesc(0u, 1u, j, nmma), tsfa, tsfb, (kb | j) != 0);
            } else {
              // NVFP4: one scale tile per k-step; MXFP4: one per two k-steps,
              // the k-step's two scale bytes selected by the scale-factor id
              constexpr uint32_t TPS = KIND == kNV ? 4u : 2u;
#pragma unroll
              for (uint32_t u = 0; u < TPS; ++u) {
                tmem_cp_sf(tsfa + 4 * u, mk(sfa_lo + 32 * u, sfa_hi));
                tmem_cp_sf(tsfb + 8 * u, mk(sfb_lo + 32 * u, sfb_hi));
                if (b_second) tmem_cp_sf(tsfb + 8 * u + 4, mk(sfb_lo + (4 * 512 >> 4) + 32 * u, sfb_hi));
              }
#pragma unroll
              for (uint32_t j = 0; j < 4; ++j) {
                if constexpr (KIND == kNV)
                  mma_block_scaled<kNV>(tmem, mk(a_lo + 2 * j, a_hi), mk(b_lo + 2 * j, b_hi), idesc_nv, tsfa + 4 * j,
                                        tsfb + 8 * j, (kb | j) != 0);
                else
                  mma_block_scaled<kMX4>(tmem, mk(a_lo + 2 * j, a_hi), mk(b_lo + 2 * j, b_hi),
                                         block_scaled_idesc(1u, 1u, (j & 1u) * 2u, nmma), tsfa + 4 * (j >> 1),
                                         tsfb + 8 * (j >> 1), (kb | j) != 0);
              }
            }
          } else {
            // ragged last stage: only the scale tiles and k-steps that exist
            uint32_t ntl = p.sf_groups > g0 ? p.sf_groups - g0 : 0;
            if (ntl > tiles_per_stage) ntl = tiles_per_stage;
            for (uint32_t u = 0; u < ntl; ++u) {
              tmem_cp_sf(tsfa + 4 * u, mk(sfa_lo + 32 * u, sfa_hi));
              tmem_cp_sf(tsfb + 8 * u, mk(sfb_lo + 32 * u, sfb_hi));
              if (b_second) tmem_cp_sf(tsfb + 8 * u + 4, mk(sfb_lo + (4 * 512 >> 4) + 32 * u, sfb_hi));
            }
            for (uint32_t j = 0; j < 4; ++j) {
              if (kb * BKB + j * 32u >= p.k_bytes) break;
              if constexpr (KIND == kMX8)
                mma_block_scaled<kMX8>(tmem, mk(a_lo + 2 * j, a_hi), mk(b_lo + 2 * j, b_hi),
                                       block_scaled_idesc(0u, 1u, j, nmma), tsfa, tsfb, (kb | j) != 0);
              else if constexpr (KIND == kMX4)
                mma_block_scaled<kMX4>(tmem, mk(a_lo + 2 * j, a_hi), mk(b_lo + 2 * j, b_hi),
                                       block_scaled_idesc(1u, 1u, (j & 1u) * 2u, nmma), tsfa + 4 * (j >> 1),
                                       tsfb + 8 * (j >> 1), (kb | j) != 0);
              else
                mma_block_scaled<kNV>(tmem, mk(a_lo + 2 * j, a_hi), mk(b_lo + 2 * j, b_hi), idesc_nv, tsfa + 4 * j,
                                      tsfb + 8 * j, (kb | j) != 0);
            }
          }
            mma_commit(smem_u32(&empty_bar[s]));
          }
          __syncwarp();
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (leader) mma_commit(smem_u32(&accum_full));  // arrives when this tile's MMAs are done
        __syncwarp();
        ++tile_i;
      }
    }
  } else if (warp == W_SCALES) {
    // ------------------------------------------------------------ scale producer
    // Same stage sequence as warp 0; its copies complete on the stage's full
    // barrier, whose expected bytes warp 0 has posted (or will post: the
    // phase cannot complete before warp 0's arrival).
    if (lane == 0) {
      uint32_t it = 0;
      for (uint32_t u = blockIdx.x; u < p.units && !*(volatile int*)&abort_flag; u += gridDim.x) {
        uint32_t tm, n0;
        bool wide;
        if (!unit_coords(u, p, mt, nt, tm, n0, wide)) continue;
        const int tile_n = (int)n0;
        const bool b_second = wide && (uint32_t)(tile_n + 128) < p.rows_b_pad;
        for (uint32_t kb = 0; kb < p.kb_count; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((it / STAGES) & 1u) ^ 1u)) {
            abort_flag = 1;
            break;
          }
          const uint32_t g0 = kb * tiles_per_stage;
          uint32_t ntl = p.sf_groups > g0 ? p.sf_groups - g0 : 0;
          if (ntl > tiles_per_stage) ntl = tiles_per_stage;
          if (ntl == 0 || withheld_stage(it)) continue;
          const uint32_t bytes = ntl * 512u, bar = smem_u32(&full_bar[s]);
          bulk_load(sbase + SMEM_SFA + s * SFA_STAGE, p.sfa + ((size_t)tm * p.sf_groups + g0) * 512u, bytes, bar);
          bulk_load(sbase + SMEM_SFB + s * SFB_STAGE, p.sfb + ((size_t)(tile_n / 128) * p.sf_groups + g0) * 512u,
                    bytes, bar);
          if (b_second)
            bulk_load(sbase + SMEM_SFB + s * SFB_STAGE + 4 * 512,
                      p.sfb + ((size_t)(tile_n / 128 + 1) * p.sf_groups + g0) * 512u, bytes, bar);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..9
    const int q = warp & 3;                // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;      // which 128 accumulator columns
    float alpha = 1.0f;
    if (KIND == kNV && p.g_x != nullptr) alpha = (__ldg(p.g_x) / kGlobalEncode) * (__ldg(p.g_w) / kGlobalEncode);
    uint32_t tile_i = 0;
    for (uint32_t u = blockIdx.x; u < p.units; u += gridDim.x) {
      uint32_t tm, n0;
      bool wide;
      if (!unit_coords(u, p, mt, nt, tm, n0, wide)) continue;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&accum_full), tile_i & 1u));
      tc_fence_after();
      ++tile_i;
      if (!ok || *(volatile int*)&abort_flag) break;
      if (!wide && half == 1) {
        // a 128 x 128 unit: the second column half holds nothing
        tc_fence_before();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&accum_empty)) : "memory");
        continue;
      }
      float v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float w32[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128 + c * 32), w32);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[c * 32 + i] = w32[i];
      }
      // accumulator drained into registers: hand TMEM back to the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&accum_empty)) : "memory");
      epilogue_store(p, &tmap_y, sbase + SMEM_EPI + (uint32_t)(warp - 2) * EPI_BUF, v, alpha,
                     (int)(tm * BM) + q * 32, (int)n0 + half * 128, lane);
    }
    // the tensor stores of this warp are complete before the CTA exits
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  __syncwarp();  // lanes that skipped a one-lane role loop wait for it before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D byte tensor [rows, row_bytes] (row stride row_bytes), box [box_rows, 128 B],
// 128-byte swizzle, out-of-range elements read as zero.
inline bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)BKB, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output tensor map for the TMA-store epilogue: boxes of 32 rows x 32 bytes.
// False (direct stores then) unless the row pitch is a multiple of 16 bytes;
// y itself is 16-byte aligned.
inline bool make_y_tmap(CUtensorMap* m, void* y, int y_dt, int64_t M, int64_t N) {
  const uint64_t esz = y_dt == NVFP4_DT_F32 ? 4u : 2u;
  memset(m, 0, sizeof(*m));
  if (((uint64_t)N * esz) % 16u != 0) return false;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)N * esz};
  cuuint32_t box[2] = {(cuuint32_t)(32u / esz), 32u};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = y_dt == NVFP4_DT_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : y_dt == NVFP4_DT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(m, dt, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

inline nvfp4_status qqmm_launch(int kind, int64_t M, int64_t N, int64_t K, const uint32_t* a_codes,
                                const uint8_t* a_scales, const uint32_t* b_codes, const uint8_t* b_scales,
                                const float* g_x, const float* g_w, void* y, int y_dt, int sm_count,
                                cudaStream_t stream, char* msg, size_t msg_len) {
  using namespace tc;
  const bool mx = kind == tc::kMX8;
  const uint64_t k_bytes = mx ? (uint64_t)K : (uint64_t)K / 2;
  CUtensorMap ta, tb, tb128;
  if (!make_tmap(&ta, a_codes, (uint64_t)M, k_bytes, BM) || !make_tmap(&tb, b_codes, (uint64_t)N, k_bytes, BN) ||
      !make_tmap(&tb128, b_codes, (uint64_t)N, k_bytes, 128)) {
    snprintf(msg, msg_len, "[qqmm] cuTensorMapEncodeTiled failed");
    return NVFP4_ERR_CUDA;
  }
  CUtensorMap ty;
  const bool tma_store = make_y_tmap(&ty, y, y_dt, M, N);
  Params p;
  p.tma_store = tma_store ? 1 : 0;
  p.sfa = a_scales;
  p.sfb = b_scales;
  p.g_x = g_x;
  p.g_w = g_w;
  p.y = y;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.y_dt = y_dt;
  p.k_bytes = (uint32_t)k_bytes;
  p.kb_count = (uint32_t)((k_bytes + BKB - 1) / BKB);
  const int64_t sf_cols = kind == tc::kNV ? K / 16 : K / 32;
  p.sf_groups = (uint32_t)((sf_cols + 3) / 4);
  p.rows_b_pad = (uint32_t)((N + 127) / 128 * 128);
  // 128 x 256 tiles; when the last wave is at most half full, its tiles run
  // as 128 x 128 halves (two units each) on up to twice as many SMs
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int64_t rem = tiles % sm_count;
  const bool split = rem != 0 && 2 * rem <= sm_count;
  p.nfull = (uint32_t)(split ? tiles - rem : tiles);
  p.units = (uint32_t)(split ? tiles + rem : tiles);
  dim3 grid((unsigned)(p.units < (uint32_t)sm_count ? p.units : (uint32_t)sm_count));  // persistent: one CTA per SM
  cudaError_t e;
  auto go = [&](auto kern) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e == cudaSuccess) kern<<<grid, THREADS, SMEM_ALLOC, stream>>>(ta, tb, tb128, ty, p);
  };
  if (kind == kMX8) go(k_qqmm<kMX8>);
  else if (kind == kMX4) go(k_qqmm<kMX4>);
  else go(k_qqmm<kNV>);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(msg, msg_len, "[qqmm] launch failed: %s", cudaGetErrorString(e));
    return NVFP4_ERR_CUDA;
  }
  msg[0] = '\0';
  return NVFP4_OK;
}

}  // namespace nvfp4
