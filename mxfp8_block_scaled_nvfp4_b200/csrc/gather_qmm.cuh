// gather_qmm: MoE matmul with per-expert NVFP4 weights and per-expert
// global scales ("[Metal] global scale for qmm", ml-explore/mlx pull 4458:
// the fp32 global scale multiplies each fp8 block scale inside the
// dequantization, before the weight is cast to bf16; weights transposed).
//
//   y[t, j, :] = x[t, :] . w_hat_e^T,   e = idx[t, j]
//   w_hat_e[n, k] = bf16( e2m1(q) * fp32(f8(s) * (g[e] / 2688)) )
//
// Two kernels:
//  1. k_route (one CTA): histogram of the T*topk (token, slot) pairs by
//     expert, exclusive prefix sum, a list of 128-pair tiles (expert, first
//     row of the expert's run, rows) and the permutation of pair ids grouped
//     by expert.  Expert ids outside [0, E) set the device error word and
//     their output rows are written as zeros.
//  2. k_gather_mma: one CTA per (tile, 256 output columns).  Warps 0-3 gather
//     the tile's 128 x rows with cp.async into the 128-byte-swizzled K-major
//     shared layout and dequantize the expert's weight tile [256 rows x 64 K]
//     to bf16 into the same layout (the weight is rounded to bf16 exactly as
//     the dequantize kernel does); warp 4 issues tcgen05 kind::f16 MMAs
//     (M=128 pairs, N=256 columns, K=16) into a TMEM fp32 accumulator; warps
//     0-3 then read the accumulator and scatter each row to y[t, j, :].
// The contraction is on the bf16 tensor pipe: both operands are bf16, as
// the method requires of the materialized weight.
#pragma once

#include <cstdio>

#include "common.cuh"
#include "nvfp4.h"
#include "qqmm_sm100.cuh"

namespace nvfp4 {
namespace gq {

constexpr int BM = 128;           // pairs per tile
constexpr int BN = 256;           // output columns per CTA
constexpr int BK = 64;            // K elements per stage (128 bytes of bf16)
constexpr int STAGES = 4;
constexpr int PRODUCERS = 128;    // warps 0-3
constexpr int THREADS = 160;      // + MMA warp
constexpr int A_STAGE = BM * 128;  // 16 KiB
constexpr int B_STAGE = BN * 128;  // 32 KiB
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE);
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 256;

// Workspace: [0] number of tiles; then tile_expert, tile_row0, tile_rows
// (max_tiles each) and the permutation (P entries), all int32.
struct Workspace {
  int32_t* ntiles;
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

__host__ __device__ inline Workspace carve(void* base, int64_t P, int64_t E) {
  Workspace w;
  char* p = static_cast<char*>(base);
  const int64_t mt = max_tiles(P, E);
  w.ntiles = reinterpret_cast<int32_t*>(p);
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
constexpr int MAX_E = 1024;

__global__ void __launch_bounds__(ROUTE_THREADS) k_route(const int32_t* __restrict__ idx, int P, int E, int N,
                                                         Workspace ws, __nv_bfloat16* __restrict__ y) {
  __shared__ int cnt[MAX_E];
  __shared__ int cursor[MAX_E];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int e = __ldg(idx + p);
    if (e >= 0 && e < E) {
      atomicAdd(&cnt[e], 1);
    } else {
      atomicOr(&g_device_error, (unsigned)kDevErrIndex);
      for (int n = 0; n < N; ++n) y[(size_t)p * N + n] = __float2bfloat16_rn(0.0f);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0, nt = 0;
    for (int e = 0; e < E; ++e) {
      cursor[e] = off;
      for (int r = 0; r < cnt[e]; r += BM) {
        ws.tile_expert[nt] = e;
        ws.tile_row0[nt] = off + r;
        ws.tile_rows[nt] = min(BM, cnt[e] - r);
        ++nt;
      }
      off += cnt[e];
    }
    *ws.ntiles = nt;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int e = __ldg(idx + p);
    if (e >= 0 && e < E) ws.perm[atomicAdd(&cursor[e], 1)] = p;
  }
}

// ---------------------------------------------------------------------------
// 2. grouped MMA
// ---------------------------------------------------------------------------
// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled
// K-major tile (rows of 128 bytes, 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) { return r * 128u + ((c ^ (r & 7u)) << 4); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  const uint32_t n = pred ? 16u : 0u;  // zero-fill when the source row does not exist
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

// kind::f16 instruction descriptor: fp32 accumulate (bits 4-5 = 1), A and B
// bf16 (bits 7-9, 10-12 = 1), K-major, N >> 3 (bits 17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t f16_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

struct Args {
  const __nv_bfloat16* x;
  const uint32_t* wc;
  const uint8_t* wsc;
  const float* g;
  __nv_bfloat16* y;
  Workspace ws;
  int N, K, topk;
};

__global__ void __launch_bounds__(THREADS, 1) k_gather_mma(Args a) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t accum_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ int rows_pair[BM];

  const int tile = blockIdx.x;
  const int ntiles = *a.ws.ntiles;
  if (tile >= ntiles) return;  // uniform per CTA, before any barrier or TMEM use
  const int e = a.ws.tile_expert[tile], row0 = a.ws.tile_row0[tile], nrows = a.ws.tile_rows[tile];
  const int n0 = blockIdx.y * BN;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < BM) rows_pair[threadIdx.x] = threadIdx.x < nrows ? a.ws.perm[row0 + threadIdx.x] : -1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), PRODUCERS);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(&accum_bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 4) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;
  const int kb_count = a.K / BK;
  bool ok = true;

  if (warp < 4) {
    // ------------------------------------------------------------ producers
    const int t = threadIdx.x;  // 0..127
    const float d = a.g ? __ldg(a.g + e) / kGlobalEncode : 1.0f;
    const uint32_t kwords = (uint32_t)a.K / 8u;    // code words per weight row
    const uint32_t kscales = (uint32_t)a.K / 16u;  // scale bytes per weight row
    const size_t wrow_base = (size_t)e * a.N;
    for (int kb = 0; kb < kb_count && ok; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait(smem_u32(&empty_bar[s]), ((kb / STAGES) & 1) ^ 1)) {
        ok = false;
        break;
      }
      const uint32_t sa = sbase + s * A_STAGE, sb = sbase + STAGES * A_STAGE + s * B_STAGE;
      // x rows of the tile: 128 rows x 8 chunks of 16 bytes
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int u = t + i * PRODUCERS;  // 0..1023
        const int r = u >> 3, c = u & 7;
        const int pid = rows_pair[r];
        const int tok = pid >= 0 ? pid / a.topk : 0;
        const __nv_bfloat16* src = a.x + (size_t)tok * a.K + kb * BK + c * 8;
        cp_async16(sa + sw128(r, c), src, pid >= 0);
      }
      // weight tile: 256 rows x 4 blocks of 16, dequantized to bf16
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int u = t + i * PRODUCERS;  // 0..1023
        const int r = u >> 2, blk = u & 3;
        const int n = n0 + r;
        uint32_t out[8];
        if (n < a.N) {
          const size_t wr = wrow_base + n;
          const uint2 cw = __ldg(reinterpret_cast<const uint2*>(a.wc + wr * kwords + (kb * BK) / 8) + blk);
          const float sd = e4m3_to_f32(__ldg(a.wsc + wr * kscales + (kb * BK) / 16 + blk)) * d;
          const uint32_t words[2] = {cw.x, cw.y};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t c0 = words[h] >> (8 * j), c1 = c0 >> 4;
              out[h * 4 + j] = pack_bf16x2(e2m1_value(c0) * sd, e2m1_value(c1) * sd);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) out[j] = 0u;
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + sw128(r, 2 * blk)), "r"(out[0]),
                     "r"(out[1]), "r"(out[2]), "r"(out[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + sw128(r, 2 * blk + 1)), "r"(out[4]),
                     "r"(out[5]), "r"(out[6]), "r"(out[7])
                     : "memory");
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // make st.shared / cp.async visible to tcgen05
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&full_bar[s])) : "memory");
    }
    // ------------------------------------------------------------ epilogue
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&accum_bar), 0) && ok);
    tc_fence_after();
    if (acc_ok) {
      const int r = warp * 32 + lane;  // TMEM lane = pair row of the tile
      const int pid = rows_pair[r];
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
        const int col = n0 + c;
        if (pid >= 0 && col < a.N) store_out<__nv_bfloat16>(a.y + (size_t)pid * a.N + col, v, min(32, a.N - col));
      }
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = f16_idesc();
      for (int kb = 0; kb < kb_count; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(smem_u32(&full_bar[s]), (kb / STAGES) & 1)) break;
        tc_fence_after();
        const uint32_t sa = sbase + s * A_STAGE, sb = sbase + STAGES * A_STAGE + s * B_STAGE;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_bf16(tmem, kmajor_sw128_desc(sa + 32 * j), kmajor_sw128_desc(sb + 32 * j), idesc, (kb | j) != 0);
        mma_commit(smem_u32(&empty_bar[s]));
      }
      mma_commit(smem_u32(&accum_bar));
    }
  }
  __syncwarp();  // lanes that skipped a one-lane role loop wait for it before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace gq

inline size_t gather_workspace_bytes(int64_t T, int64_t topk, int64_t E) { return gq::workspace_bytes(T, topk, E); }

inline nvfp4_status gather_qmm_launch(const void* x, const uint32_t* w_codes, const uint8_t* w_scales, const float* g,
                                      const int32_t* idx, int64_t T, int64_t topk, int64_t E, int64_t N, int64_t K,
                                      void* y, void* workspace, int sm_count, cudaStream_t stream, char* msg,
                                      size_t msg_len) {
  using namespace gq;
  if (E > MAX_E) {
    snprintf(msg, msg_len, "[gather_qmm] at most %d experts", MAX_E);
    return NVFP4_ERR_UNSUPPORTED;
  }
  const int64_t P = T * topk;
  Workspace ws = carve(workspace, P, E);
  k_route<<<1, ROUTE_THREADS, 0, stream>>>(idx, (int)P, (int)E, (int)N, ws, static_cast<__nv_bfloat16*>(y));
  cudaError_t err = cudaGetLastError();
  if (err == cudaSuccess) err = cudaFuncSetAttribute(k_gather_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
  if (err == cudaSuccess) {
    Args a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.wc = w_codes;
    a.wsc = w_scales;
    a.g = g;
    a.y = static_cast<__nv_bfloat16*>(y);
    a.ws = ws;
    a.N = (int)N;
    a.K = (int)K;
    a.topk = (int)topk;
    dim3 grid((unsigned)max_tiles(P, E), (unsigned)((N + BN - 1) / BN));
    k_gather_mma<<<grid, THREADS, SMEM_ALLOC, stream>>>(a);
    err = cudaGetLastError();
  }
  if (err != cudaSuccess) {
    snprintf(msg, msg_len, "[gather_qmm] launch failed: %s", cudaGetErrorString(err));
    return NVFP4_ERR_CUDA;
  }
  msg[0] = '\0';
  (void)sm_count;
  return NVFP4_OK;
}

}  // namespace nvfp4
