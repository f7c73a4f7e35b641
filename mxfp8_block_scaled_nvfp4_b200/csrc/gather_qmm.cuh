// gather_qmm: MoE matmul with per-expert NVFP4 weights and per-expert
// global scales ("[Metal] global scale for qmm", ml-explore/mlx pull 4458:
// the fp32 global scale multiplies each fp8 block scale inside the
// dequantization, before the weight is cast to bf16; weights transposed).
//
//   y[t, j, :] = x[t, :] . w_hat_e^T,   e = idx[t, j]
//   w_hat_e[n, k] = bf16( e2m1(q) * fp32(f8(s) * (g[e] / 2688)) )
//
// Kernels:
//  1. k_route (one CTA): histogram of the T*topk (token, slot) pairs by
//     expert, exclusive prefix sum, a list of 256-pair tiles (expert, first
//     row of the expert's run, rows) and the permutation of pair ids grouped
//     by expert.  Expert ids outside [0, E) set the device error word and
//     their output rows are written as zeros.
//  2. With a staged workspace and weights [E, N, K]: k_stage_x (the routed
//     x rows copied once, grouped by expert) and k_gather_mma_ts, the SM-pair
//     kernel with the dequantized weights in tensor memory (section 2b).
//  3. Otherwise k_gather_mma, persistent (one CTA per SM): work units are (256-pair
//     tile, 256 output columns), handed out round-robin, the column tiles of
//     a pair tile adjacent so that CTAs running together share x rows and the
//     expert's weight in L2.  Each dequantized weight stage feeds the MMAs of
//     both 128-pair halves of the tile (two accumulators), which halves the
//     dequantization per MMA.  Warp roles:
//       warps 0-5  gather the tile's x rows with TMA tile::gather4 (4 rows
//                  per copy, up to 11 copies per warp and k-step: one
//                  issuing warp cannot keep up with the tensor core) into
//                  128-byte-swizzled K-major stages;
//       warp 6     streams the expert's NVFP4 codes [256 rows x 32 B] per
//                  k-step with TMA;
//       warp 7     allocates TMEM and issues tcgen05 kind::f16 MMAs (M = 128
//                  pairs, N = 256 columns, K = 16) from one elected lane, one
//                  fp32 accumulator per 128-pair half;
//       warps 8-15 drain the accumulators (one TMEM lane quarter and one
//                  half each, so the MMA warp waits on half as long a
//                  drain) and scatter each pair row to y[t, j, :];
//       warps 16-31 dequantize the codes to bf16 (two threads per weight
//                  row, block scales from global memory one k-step ahead)
//                  into the swizzled B stages, rounding exactly as the
//                  dequantize kernel does.
// The contraction is on the bf16 tensor pipe: both operands are bf16, as
// the method requires of the materialized weight.  Every wait is bounded.
//
// Decode (T <= kQmvTokens tokens; the pages' "gather_qmv"): few pairs per
// expert, so 256-pair MMA tiles would mostly compute padding.  k_gather_qmv
// instead streams each routed expert's weight rows once per tile of pairs:
// a warp per weight row, 128-bit coalesced code loads, the same bf16
// rounding of the dequantized weight as above, fp32 dot products with up to
// kQmvPairs routed x rows held in shared memory (as bf16) at a time.
#pragma once

#include <cuda.h>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "nvfp4.h"
#include "qmv.cuh"
#include "qqmm_sm100.cuh"

namespace nvfp4 {
namespace gq {

constexpr int BM = 256;            // pairs per tile
constexpr int MMA_M = 128;         // pairs per MMA (one accumulator per half tile)
constexpr int BN = 256;            // output columns per unit
constexpr int BK = 64;             // K elements per k-step (128 bytes of bf16)
constexpr int XS = 3;              // x stages
constexpr int WS = 3;              // bf16 weight stages
constexpr int RS = 4;              // raw code stages
constexpr int GATHER_WARPS = 6;
constexpr int GATHER_LANES = 11;   // lanes of a gather warp that issue (6 x 11 >= 64 four-row copies)
constexpr int DEQ_WARPS = 16;
constexpr int EPI_WARPS = 8;       // two per TMEM lane quarter, one per 128-pair half
constexpr int W_CODES = 6, W_MMA = 7, W_EPI = 8, W_DEQ = 16;  // first warp of each role
constexpr int THREADS = 32 * (W_DEQ + DEQ_WARPS);                  // 1024
constexpr int X_STAGE = BM * 128;  // 32 KiB: two 16 KiB MMA operands
constexpr int W_STAGE = BN * 128;  // 32 KiB
constexpr int R_STAGE = BN * 32;   // 8 KiB of codes
constexpr int SMEM_X = 0;
constexpr int SMEM_W = SMEM_X + XS * X_STAGE;
constexpr int SMEM_R = SMEM_W + WS * W_STAGE;
constexpr int SMEM_BYTES = SMEM_R + RS * R_STAGE;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;  // two 256-column accumulators (one per half tile)

// Workspace: [0] number of tiles, [1] number of routed pairs; then
// tile_expert, tile_row0, tile_rows (max_tiles each) and the permutation
// (P entries), all int32.  The staged form appends, 256-byte aligned, a
// bf16 copy of the routed x rows in permutation order ([P, K]).
struct Workspace {
  int32_t* ntiles;
  int32_t* nrows;
  int32_t* tile_expert;
  int32_t* tile_row0;
  int32_t* tile_rows;
  int32_t* perm;
};

__host__ __device__ inline int64_t max_tiles(int64_t P, int64_t E) { return P / BM + E + 1; }

__host__ __device__ inline size_t workspace_bytes(int64_t T, int64_t topk, int64_t E) {
  const int64_t P = T * topk;
  return (size_t)(16 + 3 * 4 * max_tiles(P, E) + 4 * P + 16);
}

// Byte offset of the staged x rows in a staged workspace, and its size.
__host__ __device__ inline size_t staged_offset(int64_t T, int64_t topk, int64_t E) {
  return (workspace_bytes(T, topk, E) + 255) & ~(size_t)255;
}
__host__ __device__ inline size_t staged_workspace_bytes(int64_t T, int64_t topk, int64_t E, int64_t K) {
  return staged_offset(T, topk, E) + (size_t)(T * topk) * (size_t)K * 2u;
}

__host__ __device__ inline Workspace carve(void* base, int64_t P, int64_t E) {
  Workspace w;
  char* p = static_cast<char*>(base);
  const int64_t mt = max_tiles(P, E);
  w.ntiles = reinterpret_cast<int32_t*>(p);
  w.nrows = w.ntiles + 1;
  w.tile_expert = reinterpret_cast<int32_t*>(p + 16);
  w.tile_row0 = w.tile_expert + mt;
  w.tile_rows = w.tile_row0 + mt;
  w.perm = w.tile_rows + mt;
  return w;
}

// ---------------------------------------------------------------------------
// 1. routing
// ---------------------------------------------------------------------------
constexpr int ROUTE_THREADS = 1024;
constexpr int ROUTE_WARPS = ROUTE_THREADS / 32;
constexpr int ROUTE_CHUNK = 16;  // expert ids each lane loads before it processes them
constexpr int MAX_E = 1024;      // one expert per thread in the scans

// Dynamic shared memory of k_route: per-warp expert histograms [32][E],
// then expert offsets and first tile indices [E] each.
__host__ __device__ inline size_t route_smem_bytes(int64_t E) { return (size_t)(ROUTE_WARPS + 2) * E * 4; }

// Exclusive prefix sum of one value per thread over the CTA (1024 threads);
// also returns the total.  `tmp` holds ROUTE_WARPS ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) tmp[w] = x;
  __syncthreads();
  if (w == 0) {
    int y = tmp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += t;
    }
    tmp[lane] = y;  // inclusive over warps
  }
  __syncthreads();
  total = tmp[ROUTE_WARPS - 1];
  const int r = x - v + (w > 0 ? tmp[w - 1] : 0);
  __syncthreads();  // tmp may be reused by the caller
  return r;
}

// Pass 1 counts the pairs of each expert per warp (shared-memory atomics on
// the warp's own histogram); the per-warp counts become per-warp bases
// inside each expert's run; pass 2 gives every pair a slot with an atomic
// on its warp's base.  The order of the pairs inside an expert's run is not
// part of the result (each output row depends on its own pair only).
__global__ void __launch_bounds__(ROUTE_THREADS) k_route(const int32_t* __restrict__ idx, int P, int E, int N,
                                                         Workspace ws, __nv_bfloat16* __restrict__ y) {
  extern __shared__ int rsm[];
  __shared__ int scan_tmp[ROUTE_WARPS];
  int* whist = rsm;                     // [ROUTE_WARPS][E]
  int* off = rsm + ROUTE_WARPS * E;     // [E] first row of each expert's run
  int* tile0 = off + E;                 // [E] first tile of each expert
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < ROUTE_WARPS * E; i += blockDim.x) whist[i] = 0;
  __syncthreads();
  for (int base0 = w * 32; base0 < P; base0 += ROUTE_THREADS * ROUTE_CHUNK) {
    int ev[ROUTE_CHUNK];
#pragma unroll
    for (int i = 0; i < ROUTE_CHUNK; ++i) {
      const int p = base0 + i * ROUTE_THREADS + lane;
      ev[i] = p < P ? __ldg(idx + p) : -1;
    }
#pragma unroll
    for (int i = 0; i < ROUTE_CHUNK; ++i) {
      const int p = base0 + i * ROUTE_THREADS + lane;
      const int e = ev[i];
      if (e >= 0 && e < E) {
        atomicAdd(&whist[w * E + e], 1);
      } else if (p < P) {
        atomicOr(&g_device_error, (unsigned)kDevErrIndex);
        for (int n = 0; n < N; ++n) y[(size_t)p * N + n] = __float2bfloat16_rn(0.0f);
      }
    }
  }
  __syncthreads();
  // thread e: per-warp bases inside expert e's run, its count and tile count
  int cnt = 0, ntl = 0;
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    for (int k = 0; k < ROUTE_WARPS; ++k) {
      const int c = whist[k * E + e];
      whist[k * E + e] = cnt;
      cnt += c;
    }
    ntl = (cnt + BM - 1) / BM;
  }
  int total_rows, total_tiles;
  const int o = block_exclusive_scan(cnt, scan_tmp, total_rows);
  const int t0 = block_exclusive_scan(ntl, scan_tmp, total_tiles);
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    off[e] = o;
    tile0[e] = t0;
    for (int k = 0; k < ntl; ++k) {
      ws.tile_expert[t0 + k] = e;
      ws.tile_row0[t0 + k] = o + k * BM;
      ws.tile_rows[t0 + k] = min(BM, cnt - k * BM);
    }
  }
  if (threadIdx.x == 0) {
    *ws.ntiles = total_tiles;
    *ws.nrows = total_rows;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ROUTE_WARPS * E; i += blockDim.x) whist[i] += off[i % E];
  __syncthreads();
  for (int base0 = w * 32; base0 < P; base0 += ROUTE_THREADS * ROUTE_CHUNK) {
    int ev[ROUTE_CHUNK];
#pragma unroll
    for (int i = 0; i < ROUTE_CHUNK; ++i) {
      const int p = base0 + i * ROUTE_THREADS + lane;
      ev[i] = p < P ? __ldg(idx + p) : -1;
    }
#pragma unroll
    for (int i = 0; i < ROUTE_CHUNK; ++i) {
      const int p = base0 + i * ROUTE_THREADS + lane;
      const int e = ev[i];
      if (e >= 0 && e < E) ws.perm[atomicAdd(&whist[w * E + e], 1)] = p;
    }
  }
}

// ---------------------------------------------------------------------------
// 2. grouped MMA
// ---------------------------------------------------------------------------
// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled
// K-major tile (rows of 128 bytes, 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) { return r * 128u + ((c ^ (r & 7u)) << 4); }

// kind::f16 instruction descriptor: fp32 accumulate (bits 4-5 = 1), A and B
// bf16 (bits 7-9, 10-12 = 1), K-major, N >> 3 (bits 17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t f16_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(MMA_M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Four rows (r0..r3) of 64 bf16 of x at column c0 into 512 consecutive
// bytes of a 128-byte-swizzled stage.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, int c0, int r0, int r1, int r2,
                                            int r3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Eight e2m1 codes times the fp32 block scale, rounded to bf16 (two per
// 32-bit word): the same arithmetic as the dequantize kernel.
__device__ __forceinline__ uint4 dequant8_bf16(uint32_t w, float sd) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float lo, hi;
    e2m1x2_to_f32((w >> (8 * i)) & 0xFFu, lo, hi);
    // both products in one packed fp32x2 multiply (round-to-nearest per lane)
    uint64_t p;
    asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %3};\n\tmul.rn.f32x2 %0, a, b;\n\t}"
        : "=l"(p)
        : "f"(lo), "f"(hi), "f"(sd));
    o[i] = pack_bf16x2(__uint_as_float((uint32_t)p), __uint_as_float((uint32_t)(p >> 32)));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

struct Args {
  const uint8_t* wsc;
  const float* g;
  __nv_bfloat16* y;
  Workspace ws;
  int N, K, topk;
  int n_tiles_n;  // column tiles per pair tile
  int E;          // experts
};

// Unit u -> (pair tile, first output column).
__device__ __forceinline__ void unit_coords(uint32_t u, uint32_t n_tiles_n, uint32_t& tile, uint32_t& n0) {
  tile = u / n_tiles_n;
  n0 = (u - tile * n_tiles_n) * (uint32_t)BN;
}

// KN = false: w is [E, N, K] (quantized along K, the transposed layout);
// KN = true: w is [E, K, N] (quantized along N).  With KN the bf16 weight
// stage is written N-major (the codes' own order) and the MMA reads B as an
// MN-major operand: 128-byte-swizzled atoms of 8 k-rows x 64 n, LBO 1 KiB
// between the four atoms along N, SBO 4 KiB between 8-row groups along K.
template <bool KN>
__global__ void __launch_bounds__(THREADS, 1) k_gather_mma(const __grid_constant__ CUtensorMap tmap_x,
                                                           const __grid_constant__ CUtensorMap tmap_w, Args a) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t x_full[XS], x_empty[XS];
  __shared__ __align__(8) uint64_t w_full[WS], w_empty[WS];
  __shared__ __align__(8) uint64_t r_full[RS], r_empty[RS];
  __shared__ __align__(8) uint64_t acc_full, acc_empty;
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t units = (uint32_t)(*a.ws.ntiles) * (uint32_t)a.n_tiles_n;
  const uint32_t kb_count = (uint32_t)a.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(smem_u32(&x_full[s]), GATHER_WARPS);
      mbar_init(smem_u32(&x_empty[s]), 1);
    }
    for (int s = 0; s < WS; ++s) {
      mbar_init(smem_u32(&w_full[s]), DEQ_WARPS);
      mbar_init(smem_u32(&w_empty[s]), 1);
    }
    for (int s = 0; s < RS; ++s) {
      mbar_init(smem_u32(&r_full[s]), 1);
      mbar_init(smem_u32(&r_empty[s]), DEQ_WARPS);
    }
    mbar_init(smem_u32(&acc_full), 1);
    mbar_init(smem_u32(&acc_empty), EPI_WARPS);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp < GATHER_WARPS) {
    // ------------------------------------------------------------ x gather
    // lane l < 11 of warp w owns pair rows 4q..4q+3, q = 11w + l < 64; rows
    // past the tile's end gather token 0 (their accumulator rows are never
    // stored)
    const uint32_t q = (uint32_t)GATHER_LANES * warp + (lane < (uint32_t)GATHER_LANES ? lane : 0u);
    const uint32_t nq = min((uint32_t)GATHER_LANES, 64u - (uint32_t)GATHER_LANES * warp);  // copies of this warp
    const bool issues = lane < nq;
    uint32_t it = 0;
    for (uint32_t u = blockIdx.x; u < units; u += gridDim.x) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int row0 = a.ws.tile_row0[tile], nrows = a.ws.tile_rows[tile];
      int tok[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * (int)q + i;
        tok[i] = r < nrows ? a.ws.perm[row0 + r] / a.topk : 0;
      }
      bool ok = true;
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++it) {
        const uint32_t s = it % XS;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&x_empty[s]), ((it / XS) & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        const uint32_t bar = smem_u32(&x_full[s]);
        if (lane == 0) mbar_expect_tx(bar, nq * 512u);  // this warp's share of the stage
        __syncwarp();
        if (issues)
          tma_gather4(sbase + SMEM_X + s * X_STAGE + 512u * q, &tmap_x, (int)(kb * BK), tok[0], tok[1], tok[2], tok[3],
                      bar);
      }
      if (!ok) {
        if (lane == 0) abort_flag = 1;
        break;
      }
    }
    // the last stages must land before the CTA exits
    const uint32_t first = it > (uint32_t)XS ? it - XS : 0;
    for (uint32_t i = first; i < it; ++i) mbar_wait(smem_u32(&x_full[i % XS]), (i / XS) & 1u);
  } else if (warp == W_CODES) {
    // ------------------------------------------------------------ code stream
    const bool leader = elect_one();
    uint32_t it = 0;
    for (uint32_t u = blockIdx.x; u < units; u += gridDim.x) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int wrow = KN ? a.ws.tile_expert[tile] * a.K : a.ws.tile_expert[tile] * a.N + (int)n0;
      bool ok = true;
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++it) {
        const uint32_t s = it % RS;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&r_empty[s]), ((it / RS) & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        if (leader) {
          const uint32_t bar = smem_u32(&r_full[s]);
          mbar_expect_tx(bar, R_STAGE);
          if (KN)  // 64 k-rows x 256 codes along n
            tma_load_2d(sbase + SMEM_R + s * R_STAGE, &tmap_w, (int)(n0 / 2u), wrow + (int)(kb * 64u), bar);
          else     // 256 n-rows x 64 codes along k
            tma_load_2d(sbase + SMEM_R + s * R_STAGE, &tmap_w, (int)(kb * 32u), wrow, bar);
        }
        __syncwarp();
      }
      if (!ok) {
        if (lane == 0) abort_flag = 1;
        break;
      }
    }
    const uint32_t first = it > (uint32_t)RS ? it - RS : 0;
    if (leader)
      for (uint32_t i = first; i < it; ++i) mbar_wait(smem_u32(&r_full[i % RS]), (i / RS) & 1u);
    __syncwarp();
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    const uint32_t idesc = f16_idesc() | (KN ? (1u << 16) : 0u);  // B MN-major for KN
    const uint64_t x_base = kmajor_sw128_desc(sbase + SMEM_X);
    const uint64_t w_base = KN ? smem_desc(sbase + SMEM_W, 1024u, 4096u, 2u /* 128B swizzle */) : kmajor_sw128_desc(sbase + SMEM_W);
    constexpr uint32_t kWStep = KN ? (8192u >> 4) : 2u;  // descriptor advance per K = 16: two 8-row groups, or 32 B
    const uint32_t x_hi = (uint32_t)(x_base >> 32), w_hi = (uint32_t)(w_base >> 32);
    auto mk = [](uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; };
    uint32_t xit = 0, wit = 0, ui = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
      if (ui >= 1) {  // the epilogue has drained the previous unit's accumulators
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_empty), (ui - 1u) & 1u))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++xit, ++wit) {
        const uint32_t xs = xit % XS, ws = wit % WS;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&x_full[xs]), (xit / XS) & 1u) &&
                                         mbar_wait(smem_u32(&w_full[ws]), (wit / WS) & 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
          const uint32_t xl = (uint32_t)x_base + xs * (X_STAGE >> 4), wl = (uint32_t)w_base + ws * (W_STAGE >> 4);
#pragma unroll
          for (uint32_t hh = 0; hh < 2; ++hh)
#pragma unroll
            for (uint32_t j = 0; j < 4; ++j)
              mma_bf16(tmem + hh * 256u, mk(xl + hh * ((MMA_M * 128) >> 4) + 2 * j, x_hi), mk(wl + kWStep * j, w_hi),
                       idesc, (kb | j) != 0);
          mma_commit(smem_u32(&x_empty[xs]));
          mma_commit(smem_u32(&w_empty[ws]));
          if (kb + 1 == kb_count) mma_commit(smem_u32(&acc_full));
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
  } else if (KN && warp >= W_DEQ) {
    // ------------------------------------------------------------ dequantize (w stored [K, N])
    // thread (warp w, lane o) takes code word o (n = n0 + 8o .. +7) of k-rows
    // w, w + 16, w + 32, w + 48 of each k-step: one 16-byte N-major store per
    // word, conflict-free (the 8 lanes of a store phase hit 8 chunks of one
    // 128-byte row)
    const uint32_t o = lane, kr = (uint32_t)(warp - W_DEQ);
    const uint32_t nb16 = (uint32_t)a.N / 16u;
    uint32_t rit = 0, wit = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int e = a.ws.tile_expert[tile];
      const bool valid = n0 + 8u * o < (uint32_t)a.N;  // N % 16 == 0: whole words valid or not
      const float d = a.g ? __ldg(a.g + e) / kGlobalEncode : 1.0f;
      // scale byte of (k-row k of the expert, this word's 16-block)
      const uint8_t* scol = a.wsc + (size_t)e * a.K * nb16 + (n0 + 8u * o) / 16u;
      auto load_sc = [&](uint32_t kb, uint32_t (&sc)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          sc[i] = (valid && kb < kb_count) ? __ldg(scol + (size_t)(kb * 64u + kr + 16u * i) * nb16) : 0u;
      };
      uint32_t sc[4];
      load_sc(0, sc);
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++rit, ++wit) {
        const uint32_t rs = rit % RS, ws = wit % WS;
        uint32_t sc_next[4];
        load_sc(kb + 1, sc_next);  // next k-step's scales in flight
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&r_full[rs]), (rit / RS) & 1u) &&
                                         mbar_wait(smem_u32(&w_empty[ws]), ((wit / WS) & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        uint32_t words[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          words[i] = *reinterpret_cast<const uint32_t*>(smem + SMEM_R + rs * R_STAGE + (kr + 16u * i) * 128u + 4u * o);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&r_empty[rs]));  // codes are in registers
        const uint32_t dst = sbase + SMEM_W + ws * W_STAGE;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t k = kr + 16u * i;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (valid) v = dequant8_bf16(words[i], e4m3_to_f32(sc[i]) * d);
          const uint32_t off = (k >> 3) * 4096u + (o >> 3) * 1024u + (k & 7u) * 128u + (((o & 7u) ^ (k & 7u)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + off), "r"(v.x), "r"(v.y), "r"(v.z),
                       "r"(v.w)
                       : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // st.shared visible to tcgen05.mma
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&w_full[ws]));
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[i] = sc_next[i];
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
  } else if (warp >= W_DEQ) {
    // ------------------------------------------------------------ dequantize
    // thread pair (2t, 2t+1) owns weight row t of the unit; half h takes K
    // elements 32h..32h+31 of each k-step (blocks 2h, 2h+1)
    const uint32_t tt = threadIdx.x - 32u * W_DEQ;
    const uint32_t t = tt >> 1, h = tt & 1u;
    const uint32_t kscales = (uint32_t)a.K / 16u;
    uint32_t rit = 0, wit = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int e = a.ws.tile_expert[tile];
      const bool valid = n0 + t < (uint32_t)a.N;
      const float d = a.g ? __ldg(a.g + e) / kGlobalEncode : 1.0f;
      const unsigned short* srow =
          reinterpret_cast<const unsigned short*>(a.wsc + ((size_t)e * a.N + n0 + t) * kscales) + h;
      uint32_t sc = valid ? __ldg(srow) : 0u;  // this half's two block scales of k-step 0
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++rit, ++wit) {
        const uint32_t rs = rit % RS, ws = wit % WS;
        const uint32_t sc_next = (valid && kb + 1 < kb_count) ? __ldg(srow + 2 * (kb + 1)) : 0u;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&r_full[rs]), (rit / RS) & 1u) &&
                                         mbar_wait(smem_u32(&w_empty[ws]), ((wit / WS) & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        const uint4 c0 = *reinterpret_cast<const uint4*>(smem + SMEM_R + rs * R_STAGE + t * 32u + h * 16u);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&r_empty[rs]));  // codes are in registers
        const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
        const uint32_t dst = sbase + SMEM_W + ws * W_STAGE;
        const float sd0 = e4m3_to_f32(sc & 0xFFu) * d, sd1 = e4m3_to_f32((sc >> 8) & 0xFFu) * d;
#pragma unroll
        for (uint32_t c = 0; c < 4; ++c) {  // chunk 4h + c holds K elements 8(4h+c).. (block 2h + c/2)
          uint4 v = make_uint4(0, 0, 0, 0);
          if (valid) v = dequant8_bf16(words[c], c < 2 ? sd0 : sd1);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + sw128(t, 4u * h + c)), "r"(v.x),
                       "r"(v.y), "r"(v.z), "r"(v.w)
                       : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // st.shared visible to tcgen05.mma
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&w_full[ws]));
        sc = sc_next;
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
  } else if (warp >= W_EPI && warp < W_EPI + EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u;                        // TMEM lane quarter
    const uint32_t hh = (uint32_t)(warp - W_EPI) >> 2;   // 128-pair half (its accumulator)
    uint32_t ui = 0;
    for (uint32_t u = blockIdx.x; u < units; u += gridDim.x, ++ui) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int row0 = a.ws.tile_row0[tile], nrows = a.ws.tile_rows[tile];
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full), ui & 1u));
      tc_fence_after();
      if (!ok || *(volatile int*)&abort_flag) {
        if (lane == 0) abort_flag = 1;
        break;
      }
      {
        const int r = (int)(hh * MMA_M + q * 32u + lane);  // pair row of the tile
        const int pid = r < nrows ? a.ws.perm[row0 + r] : -1;
        for (uint32_t c = 0; c < (uint32_t)BN; c += 32) {
          float v[32];
          tmem_ld32(tmem + ((q * 32u) << 16) + hh * 256u + c, v);
          const int col = (int)(n0 + c);
          if (pid >= 0 && col < a.N) {  // N % 16 == 0: a chunk has 32 or 16 columns
            __nv_bfloat16* dst = a.y + (size_t)pid * a.N + col;
            const uint4 h0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                        pack_bf16x2(v[6], v[7]));
            const uint4 h1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                                        pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
            reinterpret_cast<uint4*>(dst)[0] = h0;
            reinterpret_cast<uint4*>(dst)[1] = h1;
            if (col + 32 <= a.N) {
              const uint4 h2 = make_uint4(pack_bf16x2(v[16], v[17]), pack_bf16x2(v[18], v[19]),
                                          pack_bf16x2(v[20], v[21]), pack_bf16x2(v[22], v[23]));
              const uint4 h3 = make_uint4(pack_bf16x2(v[24], v[25]), pack_bf16x2(v[26], v[27]),
                                          pack_bf16x2(v[28], v[29]), pack_bf16x2(v[30], v[31]));
              reinterpret_cast<uint4*>(dst)[2] = h2;
              reinterpret_cast<uint4*>(dst)[3] = h3;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty));
    }
  }
  __syncwarp();  // lanes that skipped a one-lane role loop wait for it before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

// ---------------------------------------------------------------------------
// 2b. grouped MMA on SM pairs, dequantized weights in tensor memory
// ---------------------------------------------------------------------------
// With a staged workspace, k_stage_x first copies every routed x row once
// into a contiguous [P, K] bf16 buffer in permutation order, so that a
// tile's x rows are consecutive rows there and arrive as 2-D TMA boxes (a
// 4-row tile::gather4 copy moves 512 bytes and was measured at 30-70
// cycles of issue each, which bounds a gathering kernel at about half the
// tensor-core rate).
//
// k_gather_mma_ts (weights [E, N, K]): a cluster of two CTAs computes a
// unit of 256 output columns (weight rows) x 256 pairs with
// tcgen05.mma.cta_group::2 (M = 256 weight rows, N = 256 pairs, K = 16).
// CTA r of the pair holds weight rows 128r..128r+127 of the unit, as the A
// operand, in its own tensor memory: its dequantize warps write the bf16
// weights there with tcgen05.st (one TMEM lane per weight row, two bf16 per
// column), so the dequantized weights never pass through shared memory.
// The x rows are the B operand: CTA r loads pairs 128r..128r+127 of the
// tile (staged rows) into its shared memory and the pair MMA reads both
// halves.  Per SM and 64 K this moves 16 KiB of x and 4 KiB of codes
// through shared memory, against 72 KiB (x, both operand reads of the
// bf16 weights, their stores, codes) per the same FLOPs on one SM.
//
// A pipeline stage covers 128 K (8 MMAs): the MMA warp waits on one
// barrier and commits once per stage.  Measured with 64-K stages and
// separate x and A barriers, the MMA warp's own loop (three satisfied
// waits of ~130 ns each, two commits, four MMAs) took ~0.7 us per stage
// against 0.26 us of tensor-core work.  Four A stages fill the tensor
// memory beside the accumulator; x has four shared-memory slots (an x
// stage was measured to land 1.0-1.6 us after its load was issued).
//
// The accumulator (fp32, 256 columns) holds weight rows on TMEM lanes and
// pairs on columns; the epilogue transposes 32 x 32 blocks through shared
// memory so that each pair row is stored as 16-byte pieces.
//
// Synchronisation.  Stage s of the even CTA's full barrier completes when
// both CTAs' x boxes have landed (the .cta_group::2 form of the TMA load
// counts their bytes there), the even CTA's dequantize warps have arrived
// and the odd CTA's forwarder has arrived; the MMA warp waits on it alone.
// The dequantize warps arrive after tcgen05.wait::st with a CTA-scope
// release; in the odd CTA they arrive on a local barrier that one
// forwarding lane waits on before its remote arrive, which is relaxed:
// measured, a cluster-scope release arrive waits for the issuing thread's
// outstanding memory operations (0.5-1.3 us per remote arrive when one
// forwarder pays it on every stage), and the A stage it announces was
// completed in tensor memory (tcgen05.wait::st) before the CTA-scope
// barrier the forwarder acquired; the MMA that reads it is issued only
// after the even CTA observes the arrive.  Two groups of dequantize warps
// take alternate stages.  The epilogue warps of both CTAs arrive on the
// even CTA's accumulator-empty barrier, relaxed as well, after their last
// tcgen05.ld of the accumulator has completed.  The even CTA's MMA warp
// issues every MMA and its commits arrive on the barriers at the same
// offset in both CTAs (multicast commit).  No TMA load uses cluster
// multicast.  Every wait is bounded; both CTAs reach the closing cluster
// barrier.
namespace ts {
constexpr int P_CTA = 128;           // pairs of the tile in each CTA (its half of B)
constexpr int W_CTA = 128;           // weight rows of the unit in each CTA (its half of A)
constexpr int UNIT_N = 2 * W_CTA;    // output columns per unit
constexpr int BKS = 128;             // K elements per pipeline stage
constexpr int S = 4;                 // pipeline stages: barriers and A stages (tensor memory)
constexpr int SX = 4;                // x slots (shared memory); step it uses slot it % SX
constexpr int RS = 3;                // code stages
constexpr int EPI_WARPS = 8;
constexpr int DEQ_GROUP = 8;         // dequantize warps per stage (4 lane quarters x 2 K halves)
constexpr int DEQ_WARPS = 2 * DEQ_GROUP;  // two groups, alternating stages
constexpr int W_X = 0, W_CODES = 1, W_MMA = 2, W_FWD = 3, W_EPI = 4, W_DEQ = 12;
constexpr int THREADS = 32 * (W_DEQ + DEQ_WARPS);              // 896
constexpr int X_BOX = P_CTA * 128;   // 64 K of 128 pairs (one 128-byte-swizzled box)
constexpr int X_STAGE = 2 * X_BOX;
constexpr int R_STAGE = W_CTA * (BKS / 2);  // 8 KiB of codes
constexpr int EPI_BLOCK = 32 * 64;   // 32 pairs x 32 weight rows of bf16
constexpr int EPI_BUF = 4 * EPI_BLOCK;  // an epilogue warp's four blocks of a unit
constexpr int SMEM_X = 0;
constexpr int SMEM_R = SMEM_X + SX * X_STAGE;
constexpr int SMEM_E = SMEM_R + RS * R_STAGE;
constexpr int SMEM_BYTES = SMEM_E + EPI_WARPS * EPI_BUF;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_A = 256;     // accumulator in columns 0-255, A stages after it
constexpr uint32_t A_COLS = BKS / 2; // tensor-memory columns of an A stage (two bf16 per column)
constexpr int PREFETCH = 4;          // stages of block scales each dequantize thread has in flight
constexpr uint32_t X_AHEAD = 3;      // stages ahead of its loads that the x warp prefetches into L2
static_assert(TMEM_A + S * A_COLS <= TMEM_COLS, "A stages exceed tensor memory");
static_assert(SMEM_ALLOC <= 227 * 1024 - 8 * 1024, "shared memory");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Cluster address of the shared variable at `local` in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// Remote arrive without a release fence (see the forwarder).
__device__ __forceinline__ void arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a barrier that the other CTA of the pair arrives on.
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < tc::kWaitLimit; ++i)
    if (try_wait_cluster(bar, parity)) return true;
  atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
  return false;
}
// Completion of the issuing thread's tcgen05 operations arrives on the
// barrier at the same offset in both CTAs of the pair.
__device__ __forceinline__ void commit_pair(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          bar)
      : "memory");
}
__device__ __forceinline__ void commit_own(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// D (tensor memory) += A (tensor memory) x B (shared memory descriptor).
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// kind::f16, fp32 accumulate, bf16 A and B, both K-major, M = 256, N = 256.
__host__ __device__ constexpr uint32_t idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((256u >> 4) << 24);
}
// 2-D TMA tile load into this CTA's shared memory, completing on a barrier
// of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
// Prefetch of a 2-D box of the tensor into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}
// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
}  // namespace ts

// Staged x rows: xs[r, :] = x[perm[r] / topk, :] for the routed pairs r <
// *ws.nrows, a warp per row, eight 16-byte loads in flight per lane.
constexpr int STAGE_THREADS = 256;
__global__ void __launch_bounds__(STAGE_THREADS) k_stage_x(const __nv_bfloat16* __restrict__ x, Workspace ws, int K,
                                                           int topk, __nv_bfloat16* __restrict__ xs) {
  const int rows = *ws.nrows;
  const int lane = threadIdx.x & 31;
  const uint32_t chunks = (uint32_t)K / 8u;  // 16-byte pieces of a row
  const int warps = gridDim.x * (STAGE_THREADS / 32);
  for (int r = blockIdx.x * (STAGE_THREADS / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int tok = ws.perm[r] / topk;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)tok * K);
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)r * K);
    for (uint32_t c0 = (uint32_t)lane; c0 < chunks; c0 += 8u * 32u) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t c = c0 + 32u * i;
        if (c < chunks) v[i] = __ldg(src + c);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t c = c0 + 32u * i;
        if (c < chunks) dst[c] = v[i];
      }
    }
  }
}

__global__ void __launch_bounds__(ts::THREADS, 1) k_gather_mma_ts(const __grid_constant__ CUtensorMap tmap_x,
                                                                  const __grid_constant__ CUtensorMap tmap_w, Args a) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[ts::S], a_ready[ts::S], empty[ts::S];
  __shared__ __align__(8) uint64_t r_full[ts::RS], r_empty[ts::RS];
  __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_done;
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  __shared__ float g_s[MAX_E];  // per-expert global scales / 2688

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ts::cluster_rank();
  const bool lead = rank == 0;
  const uint32_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t units = (uint32_t)(*a.ws.ntiles) * (uint32_t)a.n_tiles_n;
  const uint32_t kb_count = ((uint32_t)a.K + ts::BKS - 1) / ts::BKS;  // stages per unit (the last may hold 64 K)
  const uint32_t steps = (units > pair ? (units - pair + npairs - 1) / npairs : 0u) * kb_count;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) g_s[e] = a.g ? __ldg(a.g + e) / kGlobalEncode : 1.0f;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ts::S; ++s) {
      // even CTA: its x-load lane (expect-tx), its dequantize group and the odd CTA's forwarder
      mbar_init(smem_u32(&full[s]), 1 + ts::DEQ_GROUP + 1);
      mbar_init(smem_u32(&a_ready[s]), ts::DEQ_GROUP);  // odd CTA: its dequantize group
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int s = 0; s < ts::RS; ++s) {
      mbar_init(smem_u32(&r_full[s]), 1);
      mbar_init(smem_u32(&r_empty[s]), ts::DEQ_GROUP);  // the group that takes the stage
    }
    mbar_init(smem_u32(&acc_full), 1);
    mbar_init(smem_u32(&acc_empty), 2 * ts::EPI_WARPS);  // epilogue warps of both CTAs (even CTA's)
    mbar_init(smem_u32(&mma_done), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == ts::W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(ts::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  ts::cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == ts::W_X) {
    // ------------------------------------------------------------ x rows (this CTA's 128 pairs)
    // two 64 x 128 boxes of the staged rows per stage: tile rows 128 * rank
    // .. + 127; rows past the tile's end are other tiles' rows or past the
    // staged rows (zero fill), K past the end is zero fill, and nothing of
    // either reaches a stored output.  The boxes of the stage X_AHEAD steps
    // later are prefetched into L2 when a stage is loaded (measured: a stage
    // took 1.2-1.6 us from load to landing, longer than the three x slots
    // cover at the tensor-core rate).
    const bool leader = elect_one();
    uint32_t it = 0;
    bool ok = true;
    auto row_of = [&](uint32_t uu) {
      return a.ws.tile_row0[uu / (uint32_t)a.n_tiles_n] + ts::P_CTA * (int)rank;
    };
    int xrow_next = pair + npairs < units ? row_of(pair + npairs) : 0;
    for (uint32_t u = pair; u < units && ok; u += npairs) {
      const int xrow = u == pair ? row_of(u) : xrow_next;
      if (u != pair) xrow_next = u + npairs < units ? row_of(u + npairs) : 0;
      if (u == pair && leader)
        for (uint32_t kp = 0; kp < ts::X_AHEAD && kp < kb_count; ++kp) {  // the first stages
          ts::tma_prefetch_l2(&tmap_x, (int)(kp * ts::BKS), xrow);
          ts::tma_prefetch_l2(&tmap_x, (int)(kp * ts::BKS + 64u), xrow);
        }
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++it) {
        const uint32_t s = it % ts::S;
        // slot it % SX is free once the MMAs of step it - SX have completed
        // (their commit is that step's phase of its empty barrier; step it + 1,
        // the next phase of the same barrier, cannot complete before this load)
        const uint32_t prev = it - ts::SX;
        if (!__all_sync(0xffffffffu,
                        it < (uint32_t)ts::SX || mbar_wait(smem_u32(&empty[prev % ts::S]), (prev / ts::S) & 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        if (leader) {
          const uint32_t bar = ts::peer_addr(smem_u32(&full[s]), 0);
          if (lead) mbar_expect_tx(smem_u32(&full[s]), 2u * ts::X_STAGE);  // both CTAs' boxes
          const uint32_t dst = sbase + ts::SMEM_X + (it % ts::SX) * ts::X_STAGE;
          ts::tma_load_pair(dst, &tmap_x, (int)(kb * ts::BKS), xrow, bar);
          ts::tma_load_pair(dst + ts::X_BOX, &tmap_x, (int)(kb * ts::BKS + 64u), xrow, bar);
          const uint32_t kp = kb + ts::X_AHEAD;  // the stage X_AHEAD steps later
          if (kp < kb_count) {
            ts::tma_prefetch_l2(&tmap_x, (int)(kp * ts::BKS), xrow);
            ts::tma_prefetch_l2(&tmap_x, (int)(kp * ts::BKS + 64u), xrow);
          } else if (u + npairs < units && kp - kb_count < kb_count) {
            ts::tma_prefetch_l2(&tmap_x, (int)((kp - kb_count) * ts::BKS), xrow_next);
            ts::tma_prefetch_l2(&tmap_x, (int)((kp - kb_count) * ts::BKS + 64u), xrow_next);
          }
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
  } else if (warp == ts::W_CODES) {
    // ------------------------------------------------------------ code stream (this CTA's 128 weight rows)
    const bool leader = elect_one();
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t u = pair; u < units && ok; u += npairs) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int wrow = a.ws.tile_expert[tile] * a.N + (int)n0 + ts::W_CTA * (int)rank;
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++it) {
        const uint32_t s = it % ts::RS;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&r_empty[s]), ((it / ts::RS) & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        if (leader) {
          const uint32_t bar = smem_u32(&r_full[s]);
          mbar_expect_tx(bar, ts::R_STAGE);
          tma_load_2d(sbase + ts::SMEM_R + s * ts::R_STAGE, &tmap_w, (int)(kb * (ts::BKS / 2)), wrow, bar);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
    const uint32_t first = it > (uint32_t)ts::RS ? it - ts::RS : 0;
    if (leader)
      for (uint32_t i = first; i < it; ++i) mbar_wait(smem_u32(&r_full[i % ts::RS]), (i / ts::RS) & 1u);
    __syncwarp();
  } else if (warp == ts::W_MMA && lead) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    const bool leader = elect_one();
    const uint64_t x_base = kmajor_sw128_desc(sbase + ts::SMEM_X);
    const uint32_t x_hi = (uint32_t)(x_base >> 32);
    uint32_t it = 0, ui = 0;
    bool ok = true;
    for (uint32_t u = pair; u < units && ok; u += npairs, ++ui) {
      if (ui >= 1) {  // both CTAs' epilogues hold the previous unit's accumulator
        if (!__all_sync(0xffffffffu, ts::wait_cluster(smem_u32(&acc_empty), (ui - 1u) & 1u))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      for (uint32_t kb = 0; kb < kb_count; ++kb, ++it) {
        const uint32_t s = it % ts::S;
        if (!__all_sync(0xffffffffu, ts::wait_cluster(smem_u32(&full[s]), (it / ts::S) & 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
          const uint32_t xl = (uint32_t)x_base + (it % ts::SX) * (ts::X_STAGE >> 4);
          const uint32_t at = tmem + ts::TMEM_A + ts::A_COLS * s;
          const uint32_t nk = min(8u, ((uint32_t)a.K - kb * ts::BKS) / 16u);  // K = 16 slices of the stage
          for (uint32_t j = 0; j < nk; ++j)  // slice j: box j / 4, 32 bytes per slice inside it
            ts::mma_ts(tmem, at + 8u * j, ((uint64_t)x_hi << 32) | (xl + (j >> 2) * (ts::X_BOX >> 4) + 2u * (j & 3u)),
                       ts::idesc(), (kb | j) != 0);
          ts::commit_pair(smem_u32(&empty[s]));
          if (kb + 1 == kb_count) ts::commit_pair(smem_u32(&acc_full));
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
    // every MMA issued here has completed before the pair may release TMEM
    if (leader) ts::commit_own(smem_u32(&mma_done));
    __syncwarp();
    mbar_wait(smem_u32(&mma_done), 0);
  } else if (warp == ts::W_FWD && !lead) {
    // ------------------------------------------------------------ forwarder (odd CTA)
    // each A stage this CTA's dequantize warps completed is announced on
    // the even CTA's full barrier
    if (lane == 0) {
      for (uint32_t it = 0; it < steps; ++it) {
        const uint32_t s = it % ts::S;
        if (!mbar_wait(smem_u32(&a_ready[s]), (it / ts::S) & 1u) || *(volatile int*)&abort_flag) {
          abort_flag = 1;
          break;
        }
        ts::arrive_cluster_relaxed(ts::peer_addr(smem_u32(&full[s]), 0));
      }
    }
  } else if (warp >= ts::W_DEQ) {
    // ------------------------------------------------------------ dequantize into tensor memory
    // group grp takes stages grp, grp + 2, ...; thread (lane quarter qd,
    // lane) owns weight row t = 32 qd + lane of this CTA's half (its TMEM
    // lane); K half h takes elements 64h..64h+63 of the stage (blocks 4h ..
    // 4h+3: TMEM columns 32h..32h+31 of the stage)
    const uint32_t dw = (uint32_t)(warp - ts::W_DEQ);
    const uint32_t qd = (uint32_t)warp & 3u, h = (dw >> 2) & 1u, grp = dw >> 3;
    const uint32_t t = 32u * qd + (uint32_t)lane;
    const uint32_t trow = tmem + ((32u * qd) << 16) + ts::TMEM_A + 32u * h;
    const uint32_t kscales = (uint32_t)a.K / 16u;
    const uint32_t done_bar = lead ? 0u : 1u;  // arrive on full (even CTA) or a_ready (odd CTA)
    // Block scales (four bytes per thread and stage) are loaded PREFETCH of
    // the group's stages ahead, across units, into a fixed slot of a
    // register ring (the loop below is unrolled by PREFETCH, so no register
    // with a load in flight is copied before its use); the expert of the
    // unit after the next is loaded a unit ahead, the global scales come
    // from shared memory.
    uint32_t ua = pair, kba = 0;
    int e_next = pair < units ? a.ws.tile_expert[pair / (uint32_t)a.n_tiles_n] : 0;
    const uint32_t* srow = nullptr;
    float da = 1.0f;
    bool va = false;
    auto enter = [&](uint32_t uu) {
      uint32_t tile, n0;
      unit_coords(uu, (uint32_t)a.n_tiles_n, tile, n0);
      const int e = e_next;
      const uint32_t un = uu + npairs;
      if (un < units) e_next = a.ws.tile_expert[un / (uint32_t)a.n_tiles_n];
      const uint32_t n = n0 + ts::W_CTA * rank + t;
      va = n < (uint32_t)a.N;
      da = g_s[e];
      srow = reinterpret_cast<const uint32_t*>(a.wsc + ((size_t)e * a.N + (va ? n : 0u)) * kscales);
    };
    auto advance = [&]() {  // the cursor to the next stage
      if (ua < units && ++kba == kb_count) {
        kba = 0;
        ua += npairs;
        if (ua < units) enter(ua);
      }
    };
    auto fetch = [&](uint32_t& sc, float& d) {  // the cursor's scales, then the cursor to the group's next stage
      const bool in_k = kba * ts::BKS + 64u * h < (uint32_t)a.K;  // the last stage may hold 64 K
      sc = (ua < units && va && in_k) ? __ldg(srow + 2u * kba + h) : 0u;
      d = da;
      advance();
      advance();
    };
    if (ua < units) enter(ua);
    if (grp == 1) advance();
    uint32_t qsc[ts::PREFETCH];
    float qdd[ts::PREFETCH];
#pragma unroll
    for (int i = 0; i < ts::PREFETCH; ++i) fetch(qsc[i], qdd[i]);
    bool ok = true;
    for (uint32_t it0 = grp; it0 < steps && ok; it0 += 2u * ts::PREFETCH) {
#pragma unroll
      for (int j = 0; j < ts::PREFETCH; ++j) {
        const uint32_t it = it0 + 2u * (uint32_t)j;
        if (it >= steps) break;
        const uint32_t rs = it % ts::RS, s = it % ts::S;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&r_full[rs]), (it / ts::RS) & 1u) &&
                                         mbar_wait(smem_u32(&empty[s]), ((it / ts::S) & 1u) ^ 1u)) ||
            *(volatile int*)&abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();  // the MMAs that read this A stage have completed
        const uint8_t* cp = smem + ts::SMEM_R + rs * ts::R_STAGE + t * (ts::BKS / 2) + h * 32u;
        const uint4 c0 = *reinterpret_cast<const uint4*>(cp), c1 = *reinterpret_cast<const uint4*>(cp + 16);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&r_empty[rs]));  // codes are in registers
        const uint32_t sc = qsc[j];
        const float d = qdd[j];
        fetch(qsc[j], qdd[j]);  // the scales of this group's stage PREFETCH ahead
        uint32_t v[32];
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int b = 0; b < 4; ++b) {  // block 4h + b: words 2b, 2b + 1
          const float sd = e4m3_to_f32((sc >> (8 * b)) & 0xFFu) * d;
          const uint4 p0 = dequant8_bf16(words[2 * b], sd), p1 = dequant8_bf16(words[2 * b + 1], sd);
          v[8 * b + 0] = p0.x;
          v[8 * b + 1] = p0.y;
          v[8 * b + 2] = p0.z;
          v[8 * b + 3] = p0.w;
          v[8 * b + 4] = p1.x;
          v[8 * b + 5] = p1.y;
          v[8 * b + 6] = p1.z;
          v[8 * b + 7] = p1.w;
        }
        ts::tmem_st32(trow + ts::A_COLS * s, v);
        ts::tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(done_bar ? &a_ready[s] : &full[s]));
      }
    }
    if (!ok && lane == 0) abort_flag = 1;
  } else if (warp >= ts::W_EPI && warp < ts::W_EPI + ts::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // warp (quarter qe, pair half ph): weight rows 32 qe + lane of this
    // CTA's half x pairs 128 ph .. 128 ph + 127 of the tile, as four 32 x 32
    // blocks.  Each block is read from tensor memory, rounded to bf16 and
    // written transposed into the warp's buffer; the accumulator is released
    // after the fourth block, and only then are the pair rows stored, each
    // as four 16-byte pieces per block.
    const uint32_t qe = (uint32_t)warp & 3u, ph = (uint32_t)(warp - ts::W_EPI) >> 2;
    const uint32_t buf = sbase + ts::SMEM_E + (uint32_t)(warp - ts::W_EPI) * ts::EPI_BUF;
    const uint32_t empty_addr = ts::peer_addr(smem_u32(&acc_empty), 0);
    uint32_t ui = 0;
    for (uint32_t u = pair; u < units; u += npairs, ++ui) {
      uint32_t tile, n0;
      unit_coords(u, (uint32_t)a.n_tiles_n, tile, n0);
      const int row0 = a.ws.tile_row0[tile], nrows = a.ws.tile_rows[tile];
      int pid[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = (int)(128u * ph + 32u * c) + lane;
        pid[c] = r < nrows ? a.ws.perm[row0 + r] : -1;
      }
      const uint32_t nw = n0 + ts::W_CTA * rank + 32u * qe;  // this warp's first weight row
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full), ui & 1u));
      tc_fence_after();
      if (!ok || *(volatile int*)&abort_flag) {
        if (lane == 0) abort_flag = 1;
        break;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + ((32u * qe) << 16) + 128u * ph + 32u * c, v);
        const uint32_t blk = buf + (uint32_t)c * ts::EPI_BLOCK;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const uint32_t p = pack_bf16x2(v[i], v[i + 1]);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(blk + (uint32_t)i * 64u + 2u * lane), "h"((unsigned short)p)
                       : "memory");
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(blk + (uint32_t)(i + 1) * 64u + 2u * lane),
                       "h"((unsigned short)(p >> 16))
                       : "memory");
        }
      }
      tc_fence_before();
      __syncwarp();
      // the accumulator is free for the next unit: every tcgen05.ld of it has
      // completed (tcgen05.wait::ld) before this relaxed arrive is issued
      if (lane == 0) ts::arrive_cluster_relaxed(empty_addr);
      const uint32_t n = nw + 8u * ((uint32_t)lane & 3u);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t i = 8u * m + ((uint32_t)lane >> 2);  // pair of the block
          uint4 val;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                       : "r"(buf + (uint32_t)c * ts::EPI_BLOCK + i * 64u + 16u * ((uint32_t)lane & 3u)));
          const int p = __shfl_sync(0xffffffffu, pid[c], (int)i);
          if (p >= 0 && n < (uint32_t)a.N)  // N % 16 == 0: eight rows are all valid or none
            *reinterpret_cast<uint4*>(a.y + (size_t)p * a.N + n) = val;
        }
      }
      __syncwarp();  // the buffer is read before the next unit writes it
    }
  }
  __syncwarp();  // lanes that skipped a one-lane role loop wait for it before the CTA barrier
  tc_fence_before();
  __syncthreads();
  ts::cluster_sync();  // the pair's MMAs, copies and remote arrives are finished before TMEM is released
  if (warp == ts::W_MMA) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ts::TMEM_COLS) : "memory");
  }
}

// ---------------------------------------------------------------------------
// 3. decode: gather_qmv
// ---------------------------------------------------------------------------
constexpr int kQmvTokens = 16;   // T at or below which gather_qmm runs k_gather_qmv
constexpr int kQmvPairs = 4;     // routed x rows per pass
constexpr int QV_THREADS = 256;
constexpr int QV_ROWS = 16;      // weight rows per CTA (2 per warp)

// a0 += w.lo * x.lo, a1 += w.hi * x.hi for two bf16x2 words: fp32 fused
// multiply-adds with bf16 operands (each product exact in fp32, one rounding
// per add, as fmaf on the widened operands).
__device__ __forceinline__ void bfma2(float& a0, float& a1, uint32_t w, uint32_t x) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %2;\n\t"
      "mov.b32 {xl, xh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(w), "r"(x));
}

// Byte offset of the 8 bf16 of x starting at k (k % 8 == 0) in routed row q
// of the decode kernel's shared memory: 64-byte chunks of 32 elements, the
// four 16-byte segments of a chunk rotated by chunk / 2, so that the 8 lanes
// of a 128-bit load phase (chunks c .. c+7, one segment) hit 8 distinct
// 4-bank groups.
__device__ __forceinline__ uint32_t xb_offset(uint32_t q, uint32_t K, uint32_t k) {
  const uint32_t c = k >> 5, seg = (k >> 3) & 3u;
  return q * K * 2u + c * 64u + ((seg ^ ((c >> 1) & 3u)) << 4);
}

// Weight row r (< QV_ROWS) of this CTA's block: lane l loads 128-bit code
// chunks g*128 + 32i + l (i < 4) and their two scale bytes.
__device__ __forceinline__ void gqmv_load(const uint32_t* __restrict__ wc, const Args& a, int e, int nr, uint32_t chunks,
                                          int r, uint32_t g, uint4 (&qb)[4], uint32_t (&sb)[4]) {
  const uint32_t lane = threadIdx.x & 31u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t c = g * 128u + (uint32_t)i * 32u + lane;
    if (r < nr && c < chunks) {
      const size_t wrow = (size_t)e * a.N + blockIdx.x * QV_ROWS + r;
      qb[i] = __ldg(reinterpret_cast<const uint4*>(wc + wrow * (size_t)(a.K / 8)) + c);
      sb[i] = __ldg(reinterpret_cast<const unsigned short*>(a.wsc + wrow * (size_t)(a.K / 16)) + c);
    } else {
      qb[i] = make_uint4(0, 0, 0, 0);
      sb[i] = 0;
    }
  }
}

// The rows of one pass against NQ routed x rows held in shared memory: each
// 8-weight word is dequantized once (the bf16 rounding of the tensor-core
// path) and multiplied into NQ pairs of fp32 accumulators by packed fp32x2
// fused multiply-adds.  qb / sb hold the first unit's loads on entry; the
// next unit's loads are issued before the current unit is computed.
template <int NQ>
__device__ __forceinline__ void gqmv_rows(const uint32_t* __restrict__ wc, const Args& a, const uint8_t* xs,
                                          const int* perm, int e, int nr, float d, uint32_t groups, uint32_t chunks,
                                          uint4 (&qb)[4], uint32_t (&sb)[4], int& ur, uint32_t& ug) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t K = (uint32_t)a.K;
  float acc[NQ][2];
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q][0] = acc[q][1] = 0.0f;
  while (ur < nr) {
    uint4 qc[4];
    uint32_t sc4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qc[i] = qb[i];
      sc4[i] = sb[i];
    }
    const int cr = ur;
    const uint32_t cg = ug;
    if (++ug == groups) {
      ug = 0;
      ur += QV_THREADS / 32;
    }
    gqmv_load(wc, a, e, nr, chunks, ur, ug, qb, sb);  // next unit in flight
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t c = cg * 128u + (uint32_t)i * 32u + lane;
      if (c < chunks) {
        const uint32_t words[4] = {qc[i].x, qc[i].y, qc[i].z, qc[i].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // 8 weights per word, block h / 2 of the chunk
          const uint4 wb = dequant8_bf16(words[h], e4m3_to_f32((sc4[i] >> (8 * (h >> 1))) & 0xFFu) * d);
          const uint32_t pw[4] = {wb.x, wb.y, wb.z, wb.w};
          const uint32_t k0 = c * 32u + (uint32_t)h * 8u;
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const uint4 xw = *reinterpret_cast<const uint4*>(xs + xb_offset((uint32_t)q, K, k0));
            bfma2(acc[q][0], acc[q][1], pw[0], xw.x);
            bfma2(acc[q][0], acc[q][1], pw[1], xw.y);
            bfma2(acc[q][0], acc[q][1], pw[2], xw.z);
            bfma2(acc[q][0], acc[q][1], pw[3], xw.w);
          }
        }
      }
    }
    if (cg + 1 == groups) {  // row finished: reduce across the warp and store
      const int n = (int)blockIdx.x * QV_ROWS + cr;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        float t = acc[q][0] + acc[q][1];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0) a.y[(size_t)perm[q] * a.N + n] = __float2bfloat16_rn(t);
        acc[q][0] = acc[q][1] = 0.0f;
      }
    }
  }
}

// CTA (row block, tile): weight rows n0..n0+15 of the tile's expert against
// every pair of the tile, kQmvPairs pairs per pass; x of those pairs in
// shared memory as bf16 [kQmvPairs][K] (xb_offset): lane l reads 16 bytes
// of chunk l per 8 weights, and the swizzle puts the 8 lanes of a 128-bit
// load phase on distinct banks.  Three CTAs per SM (at most 80
// registers a thread): 4 % faster on the 4-token MoE decode than the
// unbounded 127 registers at two CTAs per SM; four (64 registers) spilled
// and was slower.
__global__ void __launch_bounds__(QV_THREADS, 3) k_gather_qmv(const __nv_bfloat16* __restrict__ x,
                                                           const uint32_t* __restrict__ wc, Args a) {
  extern __shared__ __align__(16) uint8_t xs[];  // [kQmvPairs][K] bf16 (xb_offset)
  const int tile = blockIdx.y;
  if (tile >= *a.ws.ntiles) return;  // uniform per CTA
  const int e = a.ws.tile_expert[tile], row0 = a.ws.tile_row0[tile], nrows = a.ws.tile_rows[tile];
  const int warp = threadIdx.x >> 5;
  const int K = a.K, N = a.N;
  const uint32_t chunks = (uint32_t)K / 32u;  // 32 codes (16 bytes) per lane and chunk
  const float d = a.g ? __ldg(a.g + e) / kGlobalEncode : 1.0f;
  // units (row, chunk group): a lane loads chunks g*128 + 32i + lane (i < 4)
  // of a weight row; the next unit's loads are in flight while this one
  // computes, and a pass's first loads are issued before x is staged
  const uint32_t groups = (chunks + 127u) / 128u;
  const int nr = min(QV_ROWS, N - (int)blockIdx.x * QV_ROWS);
  uint4 qb[4];
  uint32_t sb[4];
  for (int q0 = 0; q0 < nrows; q0 += kQmvPairs) {
    const int nq = min(kQmvPairs, nrows - q0);
    int ur = warp;
    uint32_t ug = 0;
    gqmv_load(wc, a, e, nr, chunks, ur, ug, qb, sb);
    __syncthreads();  // the previous pass is done with xs
    for (int q = 0; q < nq; ++q) {
      const int tok = a.ws.perm[row0 + q0 + q] / a.topk;
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)tok * K);
      for (int i = threadIdx.x; i < K / 8; i += blockDim.x)
        *reinterpret_cast<uint4*>(xs + xb_offset((uint32_t)q, (uint32_t)K, (uint32_t)(i * 8))) = __ldg(src + i);
    }
    __syncthreads();
    const int* perm = a.ws.perm + row0 + q0;
    switch (nq) {
      case 1: gqmv_rows<1>(wc, a, xs, perm, e, nr, d, groups, chunks, qb, sb, ur, ug); break;
      case 2: gqmv_rows<2>(wc, a, xs, perm, e, nr, d, groups, chunks, qb, sb, ur, ug); break;
      case 3: gqmv_rows<3>(wc, a, xs, perm, e, nr, d, groups, chunks, qb, sb, ur, ug); break;
      default: gqmv_rows<4>(wc, a, xs, perm, e, nr, d, groups, chunks, qb, sb, ur, ug); break;
    }
  }
}

// x [T, K] bf16: box 64 x 1 rows (tile::gather4 takes four rows of it),
// 128-byte swizzle.  Codes [E*N rows, K/2 bytes]: box 32 B x 256 rows for
// k_gather_mma, 64 B x 128 rows for the SM-pair kernel (`pair`).
inline bool make_maps(CUtensorMap* mx, CUtensorMap* mw, const void* x, const uint32_t* wc, uint64_t T, uint64_t K,
                      uint64_t EN, bool kn = false, uint64_t E = 0, uint64_t N = 0, bool pair = false) {
  auto fn = tc::encode_fn();
  if (!fn) return false;
  {
    cuuint64_t dims[2] = {K, T};
    cuuint64_t strides[1] = {K * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t estr[2] = {1, 1};
    if (fn(mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  if (kn) {  // codes [E * K rows, N/2 bytes], box 128 B (256 n) x 64 k-rows
    cuuint64_t dims[2] = {N / 2, E * K};
    cuuint64_t strides[1] = {N / 2};
    cuuint32_t box[2] = {128, (cuuint32_t)BK};
    cuuint32_t estr[2] = {1, 1};
    return fn(mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(wc), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  {
    cuuint64_t dims[2] = {K / 2, EN};
    cuuint64_t strides[1] = {K / 2};
    cuuint32_t box[2] = {pair ? (cuuint32_t)(ts::BKS / 2) : 32u, pair ? (cuuint32_t)ts::W_CTA : (cuuint32_t)BN};
    cuuint32_t estr[2] = {1, 1};
    if (fn(mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(wc), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

}  // namespace gq

inline size_t gather_workspace_bytes(int64_t T, int64_t topk, int64_t E) { return gq::workspace_bytes(T, topk, E); }
inline size_t gather_staged_workspace_bytes(int64_t T, int64_t topk, int64_t E, int64_t K) {
  return gq::staged_workspace_bytes(T, topk, E, K);
}

// Weights [E, N, K] (kn = false): T <= 16 runs k_gather_qmv; otherwise a
// workspace of gather_staged_workspace_bytes runs k_stage_x and the SM-pair
// kernel, a smaller one (at least gather_workspace_bytes) k_gather_mma.
inline nvfp4_status gather_qmm_launch(const void* x, const uint32_t* w_codes, const uint8_t* w_scales, const float* g,
                                      const int32_t* idx, int64_t T, int64_t topk, int64_t E, int64_t N, int64_t K,
                                      void* y, void* workspace, size_t workspace_bytes, int sm_count,
                                      cudaStream_t stream, char* msg, size_t msg_len, bool kn = false) {
  using namespace gq;
  if (E > MAX_E) {
    snprintf(msg, msg_len, "[gather_qmm] at most %d experts", MAX_E);
    return NVFP4_ERR_UNSUPPORTED;
  }
  const int64_t P = T * topk;
  Workspace ws = carve(workspace, P, E);
  const bool decode = !kn && T <= kQmvTokens && (size_t)kQmvPairs * (size_t)K * sizeof(float) <= 200u * 1024u;
  const bool pair_kernel = !kn && !decode && workspace_bytes >= staged_workspace_bytes(T, topk, E, K);
  CUtensorMap mx, mw;
  if (!make_maps(&mx, &mw, x, w_codes, (uint64_t)T, (uint64_t)K, (uint64_t)(E * N), kn, (uint64_t)E, (uint64_t)N,
                 pair_kernel)) {
    snprintf(msg, msg_len, "[gather_qmm] cuTensorMapEncodeTiled failed");
    return NVFP4_ERR_CUDA;
  }
  const size_t rsmem = route_smem_bytes(E);
  cudaError_t err = cudaFuncSetAttribute(k_route, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem);
  if (err == cudaSuccess) {
    k_route<<<1, ROUTE_THREADS, rsmem, stream>>>(idx, (int)P, (int)E, (int)N, ws, static_cast<__nv_bfloat16*>(y));
    err = cudaGetLastError();
  }
  const size_t qv_smem = (size_t)kQmvPairs * (size_t)K * sizeof(__nv_bfloat16);  // x rows as bf16
  if (err == cudaSuccess && decode) {
    // decode: gather_qmv
    err = cudaFuncSetAttribute(k_gather_qmv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qv_smem);
    if (err == cudaSuccess) {
      Args a;
      a.wsc = w_scales;
      a.g = g;
      a.y = static_cast<__nv_bfloat16*>(y);
      a.ws = ws;
      a.N = (int)N;
      a.K = (int)K;
      a.topk = (int)topk;
      a.E = (int)E;
    a.E = (int)E;
      a.n_tiles_n = 0;
      const int64_t mt = max_tiles(P, E);
      dim3 grid((unsigned)((N + QV_ROWS - 1) / QV_ROWS), (unsigned)(P < mt ? P : mt));  // every tile holds >= 1 pair
      k_gather_qmv<<<grid, QV_THREADS, qv_smem, stream>>>(static_cast<const __nv_bfloat16*>(x), w_codes, a);
      err = cudaGetLastError();
    }
    if (err != cudaSuccess) {
      snprintf(msg, msg_len, "[gather_qmm] launch failed: %s", cudaGetErrorString(err));
      return NVFP4_ERR_CUDA;
    }
    msg[0] = '\0';
    return NVFP4_OK;
  }
  if (err == cudaSuccess && pair_kernel) {
    // staged x rows, then one cluster of two CTAs per SM pair, as many
    // clusters as are resident at once
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(workspace) + staged_offset(T, topk, E));
    CUtensorMap mxs;
    {
      auto fn = tc::encode_fn();
      cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)P};
      cuuint64_t strides[1] = {(cuuint64_t)K * 2};
      cuuint32_t box[2] = {64, (cuuint32_t)ts::P_CTA};
      cuuint32_t estr[2] = {1, 1};
      if (!fn || fn(&mxs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xs, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        snprintf(msg, msg_len, "[gather_qmm] cuTensorMapEncodeTiled failed");
        return NVFP4_ERR_CUDA;
      }
    }
    {
      const int64_t want = (P + STAGE_THREADS / 32 - 1) / (STAGE_THREADS / 32);
      const int64_t cap = (int64_t)sm_count * 8;
      k_stage_x<<<(unsigned)(want < cap ? want : cap), STAGE_THREADS, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(x), ws, (int)K, (int)topk, xs);
      err = cudaGetLastError();
    }
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(k_gather_mma_ts, cudaFuncAttributeMaxDynamicSharedMemorySize, ts::SMEM_ALLOC);
    Args a;
    a.wsc = w_scales;
    a.g = g;
    a.y = static_cast<__nv_bfloat16*>(y);
    a.ws = ws;
    a.N = (int)N;
    a.K = (int)K;
    a.topk = (int)topk;
    a.E = (int)E;
    a.n_tiles_n = (int)((N + ts::UNIT_N - 1) / ts::UNIT_N);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(ts::THREADS);
    cfg.dynamicSmemBytes = ts::SMEM_ALLOC;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static int max_clusters[64] = {0};  // clusters of two resident at once, per device ordinal
    int dev = 0;
    if (err == cudaSuccess) err = cudaGetDevice(&dev);
    const int slot = dev >= 0 && dev < 64 ? dev : 0;
    if (err == cudaSuccess && max_clusters[slot] == 0) {
      cfg.gridDim = dim3(2u * (unsigned)(sm_count / 2));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_gather_mma_ts, &cfg) != cudaSuccess || n < 1) n = sm_count / 2;
      (void)cudaGetLastError();  // a failed query leaves no sticky error; clear the last-error slot
      max_clusters[slot] = n;
    }
    const int64_t max_units = max_tiles(P, E) * a.n_tiles_n;
    const int64_t pairs = max_units < max_clusters[slot] ? max_units : max_clusters[slot];
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    if (err == cudaSuccess) err = cudaLaunchKernelEx(&cfg, k_gather_mma_ts, mxs, mw, a);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) {
      snprintf(msg, msg_len, "[gather_qmm] launch failed: %s", cudaGetErrorString(err));
      return NVFP4_ERR_CUDA;
    }
    msg[0] = '\0';
    return NVFP4_OK;
  }
  auto kern = kn ? k_gather_mma<true> : k_gather_mma<false>;
  if (err == cudaSuccess) err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
  if (err == cudaSuccess) {
    Args a;
    a.wsc = w_scales;
    a.g = g;
    a.y = static_cast<__nv_bfloat16*>(y);
    a.ws = ws;
    a.N = (int)N;
    a.K = (int)K;
    a.topk = (int)topk;
    a.E = (int)E;
    a.n_tiles_n = (int)((N + BN - 1) / BN);
    const int64_t max_units = max_tiles(P, E) * a.n_tiles_n;
    const unsigned grid = (unsigned)(max_units < sm_count ? max_units : sm_count);
    kern<<<grid, THREADS, SMEM_ALLOC, stream>>>(mx, mw, a);
    err = cudaGetLastError();
  }
  if (err != cudaSuccess) {
    snprintf(msg, msg_len, "[gather_qmm] launch failed: %s", cudaGetErrorString(err));
    return NVFP4_ERR_CUDA;
  }
  msg[0] = '\0';
  return NVFP4_OK;
}

}  // namespace nvfp4
