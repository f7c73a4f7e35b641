// libnvfp4.so: the C ABI of include/nvfp4.h.  Host-side argument checks
// (texts after ops.cpp validate_global_scale / validate_qqmm_inputs,
// "mlx 0.30.7.2 -> 0.30.7.6" diff, page 8), launch configuration and the
// device error word.  One translation unit: the kernels live in the .cuh
// files it includes.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "nvfp4.h"
#include "common.cuh"
#include "quantize.cuh"
#include "qmv.cuh"
#include "qmv_tc.cuh"
#include "qqmm_sm100.cuh"
#include "gather_qmm.cuh"

using namespace nvfp4;

// Scratch of gather_qmm_noalloc: a fixed device array that the library owns
// for the life of the process (1 MiB on every GPU that loads the library).
// Host code must not pass the symbol itself to a kernel -- on the host it
// only names the array; the device address comes from
// cudaGetSymbolAddress, looked up once per device (see noalloc_scratch).
static constexpr size_t kNoAllocScratchBytes = (size_t)1 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

thread_local char t_msg[512] = "";

nvfp4_status fail(nvfp4_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
  va_end(ap);
  return s;
}

nvfp4_status ok() {
  t_msg[0] = '\0';
  return NVFP4_OK;
}

nvfp4_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[%s] launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// a * b > limit for a, b >= 0, without forming the (possibly overflowing) product.
bool product_exceeds(int64_t a, int64_t b, int64_t limit) { return b != 0 && a > limit / b; }

struct DeviceInfo {
  int sm_count = 0;
  int cc_major = 0;
  int cc_minor = 0;
  bool ok = false;
};

DeviceInfo g_dev[64];
std::mutex g_dev_mu;

// Current device's properties; the library runs on sm_100 (B200) only.
nvfp4_status device_info(const char* tag, DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[%s] cudaGetDevice: %s", tag, cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(NVFP4_ERR_UNSUPPORTED, "[%s] device ordinal %d", tag, dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ok) {
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return fail(NVFP4_ERR_CUDA, "[%s] cudaDeviceGetAttribute failed", tag);
    d.ok = true;
  }
  if (d.cc_major != 10 || d.cc_minor != 0)
    return fail(NVFP4_ERR_UNSUPPORTED,
                "[%s] this library is built for sm_100a (B200); device has compute capability %d.%d",
                tag, d.cc_major, d.cc_minor);
  *out = d;
  return NVFP4_OK;
}

bool valid_dt(nvfp4_dtype dt) { return dt == NVFP4_DT_F32 || dt == NVFP4_DT_F16 || dt == NVFP4_DT_BF16; }

// CTAs of `fn` (threads per CTA, dynamic shared memory) that fit on one SM
// at once, cached per kernel.
int resident_ctas(const void* fn, int threads, size_t smem) {
  static std::mutex mu;
  static const void* keys[128];
  static int vals[128];
  static int n = 0;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n; ++i)
    if (keys[i] == fn) return vals[i];
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, fn, threads, smem) != cudaSuccess || b < 1) b = 1;
  if (n < 128) {
    keys[n] = fn;
    vals[n] = b;
    ++n;
  }
  return b;
}

// Persistent elementwise grid: every SM filled with as many CTAs of the
// kernel as are resident at once (one wave), never more than the work needs.
unsigned ew_grid(const DeviceInfo& d, uint64_t work_threads, int per_sm) {
  uint64_t want = (work_threads + kEwThreads - 1) / kEwThreads;
  uint64_t cap = (uint64_t)d.sm_count * (uint64_t)per_sm;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return (unsigned)want;
}

template <typename F>
void dispatch_dt(nvfp4_dtype dt, F&& f) {
  switch (dt) {
    case NVFP4_DT_F32: f(float{}); break;
    case NVFP4_DT_F16: f(__half{}); break;
    default: f(__nv_bfloat16{}); break;
  }
}

constexpr int64_t kMaxElems = (int64_t)1 << 34;  // 16 Gi elements: 32-bit half-block indices

}  // namespace

extern "C" {

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
    case NVFP4_ERR_DEVICE_INDEX: return "device-side index out of range";
  }
  return "unknown status";
}

const char* nvfp4_last_error_message(void) { return t_msg; }

nvfp4_status nvfp4_check_device_errors(nvfp4_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[check_device_errors] %s", cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word));
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[check_device_errors] %s", cudaGetErrorString(e));
  if (word != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (word & kDevErrTimeout)
      return fail(NVFP4_ERR_TIMEOUT, "[device] a kernel gave up a bounded wait (word 0x%x)", word);
    return fail(NVFP4_ERR_DEVICE_INDEX, "[device] an index was out of range (word 0x%x)", word);
  }
  return ok();
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t cols, nvfp4_layout layout) {
  if (rows < 0 || cols < 0) return 0;
  if (layout == NVFP4_LAYOUT_LINEAR) return (size_t)(rows * cols);
  return (size_t)(((rows + 127) / 128 * 128) * ((cols + 3) / 4 * 4));
}

static nvfp4_status amax_launch(const char* tag, const nvfp4_amax_item* items, int count, nvfp4_dtype dt,
                                nvfp4_stream_t stream) {
  if (!valid_dt(dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[%s] dtype must be float32, float16 or bfloat16", tag);
  if (!items || count < 1 || count > kAmaxSegs)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] between 1 and %d tensors, got %d", tag, kAmaxSegs, count);
  for (int i = 0; i < count; ++i) {
    const nvfp4_amax_item& it = items[i];
    if (it.n < 0 || it.n > kMaxElems) return fail(NVFP4_ERR_INVALID_ARG, "[%s] bad size %lld", tag, (long long)it.n);
    if (!it.g_out || (it.n > 0 && !it.x)) return fail(NVFP4_ERR_INVALID_ARG, "[%s] null pointer", tag);
    if (!aligned16(it.x) || (reinterpret_cast<uintptr_t>(it.g_out) & 3u))
      return fail(NVFP4_ERR_INVALID_ARG, "[%s] x must be 16-byte aligned, g_out 4-byte aligned", tag);
    for (int j = 0; j < i; ++j)
      if (items[j].g_out == it.g_out) return fail(NVFP4_ERR_INVALID_ARG, "[%s] two tensors share one output", tag);
  }
  DeviceInfo d;
  nvfp4_status st = device_info(tag, &d);
  if (st != NVFP4_OK) return st;
  // outputs start at 0 (max |x| >= 0); one memset when they are consecutive floats
  bool consecutive = true;
  for (int i = 1; i < count; ++i) consecutive = consecutive && items[i].g_out == items[0].g_out + i;
  cudaError_t e = cudaSuccess;
  if (consecutive) {
    e = cudaMemsetAsync(items[0].g_out, 0, sizeof(float) * (size_t)count, stream);
  } else {
    for (int i = 0; i < count && e == cudaSuccess; ++i) e = cudaMemsetAsync(items[i].g_out, 0, sizeof(float), stream);
  }
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[%s] memset: %s", tag, cudaGetErrorString(e));
  AmaxSegs a;
  memset(&a, 0, sizeof(a));
  uint64_t vecs = 0;
  for (int i = 0; i < count; ++i) {
    if (items[i].n == 0) continue;  // its output stays 0
    a.x[a.count] = items[i].x;
    a.n[a.count] = items[i].n;
    a.out[a.count] = items[i].g_out;
    ++a.count;
    vecs += (uint64_t)(items[i].n / 8 + 1);
  }
  if (a.count == 0) return ok();
  dispatch_dt(dt, [&](auto tag_t) {
    using T = decltype(tag_t);
    const unsigned grid = ew_grid(d, (vecs + 3) / 4, resident_ctas((const void*)k_amax<T>, kEwThreads, 0));
    k_amax<T><<<grid, kEwThreads, 0, stream>>>(a);
  });
  return check_launch(tag);
}

nvfp4_status nvfp4_amax(const void* x, nvfp4_dtype dt, int64_t n, float* g_out, nvfp4_stream_t stream) {
  const nvfp4_amax_item it{x, n, g_out};
  return amax_launch("amax", &it, 1, dt, stream);
}

nvfp4_status nvfp4_amax_multi(const nvfp4_amax_item* items, int count, nvfp4_dtype dt, nvfp4_stream_t stream) {
  return amax_launch("amax_multi", items, count, dt, stream);
}

// Argument checks of one row-wise quantize; *empty is set when the output
// has no element.  kind: 0 NVFP4, 1 MXFP8, 2 MXFP4 (the two MX kinds use
// 32-element blocks).
static nvfp4_status check_quantize(const char* tag, int kind, const void* x, nvfp4_dtype dt, int64_t rows,
                                   int64_t K, const float* g, const uint32_t* codes, const uint8_t* scales,
                                   nvfp4_layout layout, bool* empty) {
  const int group = kind ? 32 : 16;
  if (!valid_dt(dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[%s] dtype must be float32, float16 or bfloat16", tag);
  if (layout != NVFP4_LAYOUT_LINEAR && layout != NVFP4_LAYOUT_SWIZZLED)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] unknown scale layout", tag);
  if (rows < 0 || K < 0 || product_exceeds(rows, K, kMaxElems))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] bad shape [%lld, %lld]", tag, (long long)rows, (long long)K);
  if (K % group != 0)
    return fail(NVFP4_ERR_INVALID_ARG,
                "[%s] The last dimension of the matrix needs to be divisible by the quantization group size %d. "
                "However the provided matrix has shape [%lld, %lld]",
                tag, group, (long long)rows, (long long)K);
  if (rows * K > 0 && (!x || !codes || !scales)) return fail(NVFP4_ERR_INVALID_ARG, "[%s] null pointer", tag);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] tensor pointers must be 16-byte aligned", tag);
  *empty = rows * K == 0;
  return NVFP4_OK;
}

static ScaleOut scale_out(uint8_t* scales, int64_t K, int group, nvfp4_layout layout) {
  ScaleOut so;
  so.init(scales, (uint32_t)(K / group), layout == NVFP4_LAYOUT_SWIZZLED);
  return so;
}

// NVFP4 quantize of `count` tensors (those with elements) in one launch.
static nvfp4_status nvfp4_quantize_launch(const char* tag, const nvfp4_quantize_item* items, int count,
                                          nvfp4_dtype dt, nvfp4_stream_t stream, bool sr, uint64_t seed) {
  if (!items || count < 1 || count > kMaxSegs)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] between 1 and %d tensors, got %d", tag, kMaxSegs, count);
  QuantSegs q;
  memset(&q, 0, sizeof(q));
  q.seed = seed;
  bool v8 = true;  // 256-bit loads need every input 32-byte aligned
  for (int i = 0; i < count; ++i) {
    const nvfp4_quantize_item& it = items[i];
    bool empty = false;
    nvfp4_status st = check_quantize(tag, 0, it.x, dt, it.rows, it.K, it.g, it.codes, it.scales, it.layout, &empty);
    if (st != NVFP4_OK) return st;
    if (empty) continue;
    QuantSeg& sg = q.s[q.count++];
    sg.x = it.x;
    sg.g = it.g;
    sg.codes = it.codes;
    sg.so = scale_out(it.scales, it.K, 16, it.layout);
    sg.rows = (uint32_t)it.rows;
    sg.n_blk = (uint32_t)(it.rows * it.K / 16);
    sg.first_unit = q.units;
    q.units += (sg.n_blk + kUnitBlk - 1) / kUnitBlk;
    v8 = v8 && (reinterpret_cast<uintptr_t>(it.x) & 31u) == 0;
  }
  if (q.count == 0) return ok();  // nothing to write: no device work, no device query
  DeviceInfo d;
  nvfp4_status st = device_info(tag, &d);
  if (st != NVFP4_OK) return st;
  dispatch_dt(dt, [&](auto tag_t) {
    using T = decltype(tag_t);
    auto go = [&](auto kern) {
      const unsigned grid = ew_grid(d, (uint64_t)q.units * 32u, resident_ctas((const void*)kern, kEwThreads, 0));
      kern<<<grid, kEwThreads, 0, stream>>>(q);
    };
    if (sr) v8 ? go(k_nvfp4_quantize<T, true, true>) : go(k_nvfp4_quantize<T, true, false>);
    else v8 ? go(k_nvfp4_quantize<T, false, true>) : go(k_nvfp4_quantize<T, false, false>);
  });
  return check_launch(tag);
}

static nvfp4_status mx_quantize(const char* tag, int kind, const void* x, nvfp4_dtype dt, int64_t rows, int64_t K,
                                uint32_t* codes, uint8_t* scales, nvfp4_layout layout, nvfp4_stream_t stream) {
  bool empty = false;
  nvfp4_status st = check_quantize(tag, kind, x, dt, rows, K, nullptr, codes, scales, layout, &empty);
  if (st != NVFP4_OK) return st;
  if (empty) return ok();  // nothing to write: no device work, no device query
  DeviceInfo d;
  st = device_info(tag, &d);
  if (st != NVFP4_OK) return st;
  const ScaleOut so = scale_out(scales, K, 32, layout);
  const uint32_t n_half = (uint32_t)(rows * K / 8);
  dispatch_dt(dt, [&](auto tag_t) {
    using T = decltype(tag_t);
    const void* fn = kind == 1 ? (const void*)k_mxfp8_quantize<T> : (const void*)k_mxfp4_quantize<T>;
    const unsigned grid = ew_grid(d, ((uint64_t)n_half + kUnroll - 1) / kUnroll, resident_ctas(fn, kEwThreads, 0));
    if (kind == 1)
      k_mxfp8_quantize<T><<<grid, kEwThreads, 0, stream>>>(static_cast<const T*>(x), n_half, codes, so,
                                                           (uint32_t)rows);
    else
      k_mxfp4_quantize<T><<<grid, kEwThreads, 0, stream>>>(static_cast<const T*>(x), n_half, codes, so,
                                                           (uint32_t)rows);
  });
  return check_launch(tag);
}

nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K, const float* g,
                            uint32_t* codes, uint8_t* scales, nvfp4_layout layout, nvfp4_stream_t stream) {
  const nvfp4_quantize_item it{x, rows, K, g, codes, scales, layout};
  return nvfp4_quantize_launch("quantize", &it, 1, dt, stream, false, 0);
}

nvfp4_status nvfp4_quantize_multi(const nvfp4_quantize_item* items, int count, nvfp4_dtype dt,
                                  nvfp4_stream_t stream) {
  return nvfp4_quantize_launch("quantize_multi", items, count, dt, stream, false, 0);
}

nvfp4_status nvfp4_quantize_sr(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K, const float* g,
                               uint64_t seed, uint32_t* codes, uint8_t* scales, nvfp4_layout layout,
                               nvfp4_stream_t stream) {
  const nvfp4_quantize_item it{x, rows, K, g, codes, scales, layout};
  return nvfp4_quantize_launch("quantize_sr", &it, 1, dt, stream, true, seed);
}

static nvfp4_status columnwise_launch(const char* tag, const void* x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                                      const float* g, uint32_t* codes, uint8_t* scales, nvfp4_layout layout,
                                      nvfp4_stream_t stream, bool sr, uint64_t seed) {
  if (!valid_dt(dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[%s] dtype must be float32, float16 or bfloat16", tag);
  if (layout != NVFP4_LAYOUT_LINEAR && layout != NVFP4_LAYOUT_SWIZZLED)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] unknown scale layout", tag);
  if (rows < 0 || cols < 0 || rows > (1 << 30) || cols > (1 << 30) || rows * cols > kMaxElems)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] bad shape [%lld, %lld]", tag, (long long)rows, (long long)cols);
  if (rows % 16 != 0)
    return fail(NVFP4_ERR_INVALID_ARG,
                "[%s] The quantized dimension (rows of x, the last dimension of x^T) needs to be divisible by the "
                "quantization group size 16. However the provided matrix has shape [%lld, %lld]",
                tag, (long long)rows, (long long)cols);
  if (rows * cols > 0 && (!x || !codes || !scales)) return fail(NVFP4_ERR_INVALID_ARG, "[%s] null pointer", tag);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] tensor pointers must be 16-byte aligned", tag);
  if (rows * cols == 0) return ok();
  DeviceInfo d;
  nvfp4_status st = device_info(tag, &d);
  if (st != NVFP4_OK) return st;
  ScaleOut so;
  so.init(scales, (uint32_t)(rows / 16), layout == NVFP4_LAYOUT_SWIZZLED);
  dim3 grid((unsigned)((rows + kColR - 1) / kColR), (unsigned)((cols + kColC - 1) / kColC));
  dispatch_dt(dt, [&](auto tag_t) {
    using T = decltype(tag_t);
    if (sr)
      k_nvfp4_quantize_columnwise<T, true><<<grid, kColThreads, 0, stream>>>(static_cast<const T*>(x), (uint32_t)rows,
                                                                            (uint32_t)cols, g, codes, so, seed);
    else
      k_nvfp4_quantize_columnwise<T><<<grid, kColThreads, 0, stream>>>(static_cast<const T*>(x), (uint32_t)rows,
                                                                        (uint32_t)cols, g, codes, so);
  });
  return check_launch(tag);
}

nvfp4_status nvfp4_quantize_columnwise(const void* x, nvfp4_dtype dt, int64_t rows, int64_t cols, const float* g,
                                       uint32_t* codes, uint8_t* scales, nvfp4_layout layout, nvfp4_stream_t stream) {
  return columnwise_launch("quantize_columnwise", x, dt, rows, cols, g, codes, scales, layout, stream, false, 0);
}

nvfp4_status nvfp4_quantize_columnwise_sr(const void* x, nvfp4_dtype dt, int64_t rows, int64_t cols, const float* g,
                                          uint64_t seed, uint32_t* codes, uint8_t* scales, nvfp4_layout layout,
                                          nvfp4_stream_t stream) {
  return columnwise_launch("quantize_columnwise_sr", x, dt, rows, cols, g, codes, scales, layout, stream, true, seed);
}

nvfp4_status mxfp8_quantize(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K, uint32_t* codes,
                            uint8_t* scales, nvfp4_layout layout, nvfp4_stream_t stream) {
  return mx_quantize("mxfp8_quantize", 1, x, dt, rows, K, codes, scales, layout, stream);
}

nvfp4_status mxfp4_quantize(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K, uint32_t* codes,
                            uint8_t* scales, nvfp4_layout layout, nvfp4_stream_t stream) {
  return mx_quantize("mxfp4_quantize", 2, x, dt, rows, K, codes, scales, layout, stream);
}

static nvfp4_status dequantize_common(const char* tag, int kind, const uint32_t* codes, const uint8_t* scales,
                                      nvfp4_layout layout, int64_t rows, int64_t K, const float* g, void* out,
                                      nvfp4_dtype out_dt, nvfp4_stream_t stream) {
  const int group = kind ? 32 : 16;
  if (!valid_dt(out_dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[%s] output dtype must be float32, float16 or bfloat16", tag);
  if (layout != NVFP4_LAYOUT_LINEAR && layout != NVFP4_LAYOUT_SWIZZLED)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] unknown scale layout", tag);
  if (rows < 0 || K < 0 || product_exceeds(rows, K, kMaxElems) || K % group != 0)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] bad shape [%lld, %lld] for group size %d", tag, (long long)rows,
                (long long)K, group);
  if (rows * K > 0 && (!codes || !scales || !out)) return fail(NVFP4_ERR_INVALID_ARG, "[%s] null pointer", tag);
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) || (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] tensor pointers must be 16-byte aligned", tag);
  if (rows * K == 0) return ok();  // nothing to write: no device work, no device query
  DeviceInfo d;
  nvfp4_status st = device_info(tag, &d);
  if (st != NVFP4_OK) return st;
  ScaleIn si;
  si.p = scales;
  si.blocks_per_row = (uint32_t)(K / group);
  si.Cp = (uint32_t)((K / group + 3) / 4 * 4);
  si.swizzled = layout == NVFP4_LAYOUT_SWIZZLED;
  const uint32_t n_half = (uint32_t)(rows * K / 8);
  dispatch_dt(out_dt, [&](auto tag_t) {
    using T = decltype(tag_t);
    const void* fn = kind == 1 ? (const void*)k_mxfp8_dequantize<T>
                     : kind == 2 ? (const void*)k_mxfp4_dequantize<T> : (const void*)k_nvfp4_dequantize<T>;
    const unsigned grid = ew_grid(d, n_half, resident_ctas(fn, kEwThreads, 0));
    if (kind == 1)
      k_mxfp8_dequantize<T><<<grid, kEwThreads, 0, stream>>>(codes, si, n_half, static_cast<T*>(out));
    else if (kind == 2)
      k_mxfp4_dequantize<T><<<grid, kEwThreads, 0, stream>>>(codes, si, n_half, static_cast<T*>(out));
    else
      k_nvfp4_dequantize<T><<<grid, kEwThreads, 0, stream>>>(codes, si, g, n_half, static_cast<T*>(out));
  });
  return check_launch(tag);
}

nvfp4_status nvfp4_dequantize(const uint32_t* codes, const uint8_t* scales, nvfp4_layout layout, int64_t rows,
                              int64_t K, const float* g, void* out, nvfp4_dtype out_dt, nvfp4_stream_t stream) {
  return dequantize_common("dequantize", 0, codes, scales, layout, rows, K, g, out, out_dt, stream);
}

nvfp4_status mxfp8_dequantize(const uint32_t* codes, const uint8_t* scales, nvfp4_layout layout, int64_t rows,
                              int64_t K, void* out, nvfp4_dtype out_dt, nvfp4_stream_t stream) {
  return dequantize_common("mxfp8_dequantize", 1, codes, scales, layout, rows, K, nullptr, out, out_dt, stream);
}

nvfp4_status mxfp4_dequantize(const uint32_t* codes, const uint8_t* scales, nvfp4_layout layout, int64_t rows,
                              int64_t K, void* out, nvfp4_dtype out_dt, nvfp4_stream_t stream) {
  return dequantize_common("mxfp4_dequantize", 2, codes, scales, layout, rows, K, nullptr, out, out_dt, stream);
}

nvfp4_status nvfp4_swizzle_scales(const uint8_t* lin, int64_t rows, int64_t cols, uint8_t* swz,
                                  nvfp4_stream_t stream) {
  if (rows < 0 || cols < 0 || product_exceeds(rows, cols, (int64_t)1 << 31))
    return fail(NVFP4_ERR_INVALID_ARG, "[swizzle_scales] bad shape");
  if (rows * cols > 0 && (!lin || !swz)) return fail(NVFP4_ERR_INVALID_ARG, "[swizzle_scales] null pointer");
  if (!aligned16(lin) || !aligned16(swz))
    return fail(NVFP4_ERR_INVALID_ARG, "[swizzle_scales] Starting addresses must be 16-byte aligned");
  if (rows * cols == 0) return ok();
  DeviceInfo d;
  nvfp4_status st = device_info("swizzle_scales", &d);
  if (st != NVFP4_OK) return st;
  const uint32_t Rp = (uint32_t)((rows + 127) / 128 * 128), Cp = (uint32_t)((cols + 3) / 4 * 4);
  const unsigned grid = ew_grid(d, (uint64_t)Rp * Cp, resident_ctas((const void*)k_swizzle_scales, kEwThreads, 0));
  k_swizzle_scales<<<grid, kEwThreads, 0, stream>>>(lin, (uint32_t)rows, (uint32_t)cols, Rp, Cp, swz);
  return check_launch("swizzle_scales");
}

// Global-scale checks of qqmm ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 8,
// ops.cpp validate_global_scale and validate_qqmm_inputs).
static nvfp4_status check_qqmm_global_scales(nvfp4_mode mode, const float* g_x, const float* g_w) {
  if (mode != NVFP4_MODE_NVFP4 && (g_x || g_w))
    return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] Global scale is only supported for 'nvfp4' quantization mode.");
  if (mode == NVFP4_MODE_NVFP4 && ((g_x == nullptr) != (g_w == nullptr)))
    return fail(NVFP4_ERR_INVALID_ARG,
                "[qqmm] For nvfp4 mode, either both global_scale_x and global_scale_w must be provided, or neither.");
  return NVFP4_OK;
}

nvfp4_status qqmm(nvfp4_mode mode, int64_t M, int64_t N, int64_t K, const uint32_t* a_codes,
                  const uint8_t* a_scales, const uint32_t* b_codes, const uint8_t* b_scales, const float* g_x,
                  const float* g_w, void* y, nvfp4_dtype y_dt, nvfp4_stream_t stream) {
  if (mode != NVFP4_MODE_NVFP4 && mode != NVFP4_MODE_MXFP8 && mode != NVFP4_MODE_MXFP4)
    return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] Only 'nvfp4', 'mxfp8' and 'mxfp4' modes are supported.");
  nvfp4_status st = check_qqmm_global_scales(mode, g_x, g_w);
  if (st != NVFP4_OK) return st;
  if (!valid_dt(y_dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[qqmm] output dtype must be float32, float16 or bfloat16");
  if (M < 0 || N < 0 || K < 0 || M > (1 << 30) || N > (1 << 30) || K > (1 << 30))
    return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] bad shape");
  if (K % 32 != 0)
    return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] K must be a multiple of 32, got %lld", (long long)K);
  if (K == 0 && M * N > 0) return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] K must be positive when M*N > 0");
  if (M * N > 0 && (!a_codes || !a_scales || !b_codes || !b_scales || !y))
    return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] null pointer");
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(g_x) & 3u) || (reinterpret_cast<uintptr_t>(g_w) & 3u))
    return fail(NVFP4_ERR_INVALID_ARG, "[qqmm] tensor pointers must be 16-byte aligned");
  if (M * N == 0) return ok();
  DeviceInfo d;
  st = device_info("qqmm", &d);
  if (st != NVFP4_OK) return st;
  return qqmm_launch((int)mode, M, N, K, a_codes, a_scales, b_codes, b_scales, g_x, g_w, y,
                     (int)y_dt, d.sm_count, stream, t_msg, sizeof(t_msg));
}

// pdl: the tensor-core kernel's PDL form (qmv_pdl); the SIMT kernel always
// launches in plain stream order.
static nvfp4_status qmv_launch(const void* x, nvfp4_dtype x_dt, const float* g_x, const uint32_t* w_codes,
                               const uint8_t* w_scales, const float* g_w, int64_t M, int64_t N, int64_t K, void* y,
                               nvfp4_stream_t stream, bool pdl) {
  if (!valid_dt(x_dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[qmv] dtype must be float32, float16 or bfloat16");
  if ((g_x == nullptr) != (g_w == nullptr))
    return fail(NVFP4_ERR_INVALID_ARG,
                "[qqmm] For nvfp4 mode, either both global_scale_x and global_scale_w must be provided, or neither.");
  if (M < 1 || M > kQmvMaxM) return fail(NVFP4_ERR_INVALID_ARG, "[qmv] M must be in [1, %d], got %lld", kQmvMaxM, (long long)M);
  if (N < 0 || K < 32 || K % 32 != 0 || N > (1 << 30))
    return fail(NVFP4_ERR_INVALID_ARG, "[qmv] bad shape N=%lld K=%lld (K %% 32 == 0)", (long long)N, (long long)K);
  if (M * K * 4 > 160 * 1024)
    return fail(NVFP4_ERR_UNSUPPORTED, "[qmv] M*K*4 bytes of x_hat must fit 160 KiB of shared memory");
  if (N > 0 && (!x || !w_codes || !w_scales || !y)) return fail(NVFP4_ERR_INVALID_ARG, "[qmv] null pointer");
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(g_x) & 3u) || (reinterpret_cast<uintptr_t>(g_w) & 3u))
    return fail(NVFP4_ERR_INVALID_ARG, "[qmv] tensor pointers must be 16-byte aligned");
  if (N == 0) return ok();
  DeviceInfo d;
  nvfp4_status st = device_info("qmv", &d);
  if (st != NVFP4_OK) return st;
  cudaError_t e = cudaSuccess;
  const uint32_t esz = x_dt == NVFP4_DT_F32 ? 4u : 2u;
  const uint32_t stages = qtc::pick_stages(M, K, esz);
  if (stages > 0) {
    // tensor-core path: one CTA per 128 weight rows
    CUtensorMap mw;
    if (!qtc::make_map(&mw, w_codes, (uint64_t)N, (uint64_t)K))
      return fail(NVFP4_ERR_CUDA, "[qmv] cuTensorMapEncodeTiled failed");
    const qtc::Groups gr = qtc::pick_groups(stages, (uint32_t)(K / 256));
    qtc::Args a{x, g_x, w_codes, w_scales, g_w, y, (uint32_t)M, (uint32_t)N, (uint32_t)K, stages, gr.g0, gr.g};
    const uint32_t MM = M == 1 ? 1u : 2u;
    const size_t smem = qtc::smem_needed(stages, MM, (uint32_t)K, esz);
    const unsigned grid = (unsigned)((N + qtc::BM - 1) / qtc::BM);
    dispatch_dt(x_dt, [&](auto tag_t) {
      using T = decltype(tag_t);
      auto go = [&](auto kern) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return;
        if (!pdl) {
          kern<<<grid, qtc::THREADS, smem, stream>>>(mw, a);
          return;
        }
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(qtc::THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, mw, a);
      };
      if (M == 1) pdl ? go(qtc::k_qmv_tc<T, 1, true>) : go(qtc::k_qmv_tc<T, 1>);
      else pdl ? go(qtc::k_qmv_tc<T, 2, true>) : go(qtc::k_qmv_tc<T, 2>);
    });
  } else {
    const size_t smem = (size_t)M * K * sizeof(float);
    // one CTA of 16 warps per SM; each warp owns whole weight rows
    uint64_t grid = ((uint64_t)N + (kQmvThreads / 32) - 1) / (kQmvThreads / 32);
    if (grid > (uint64_t)d.sm_count) grid = d.sm_count;
    dispatch_dt(x_dt, [&](auto tag_t) {
      using T = decltype(tag_t);
      auto x_t = [](const void* p) { return static_cast<const T*>(p); };
      auto y_t = [](void* p) { return static_cast<T*>(p); };
      auto go = [&](auto kern) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
          kern<<<(unsigned)grid, kQmvThreads, smem, stream>>>(x_t(x), g_x, w_codes, w_scales, g_w, (int)M, (int)N,
                                                             (int)K, y_t(y));
      };
      if (M == 1) go(k_qmv<T, 1>);
      else if (M == 2) go(k_qmv<T, 2>);
      else if (M <= 4) go(k_qmv<T, 4>);
      else go(k_qmv<T, 8>);
    });
  }
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[qmv] %s", cudaGetErrorString(e));
  return check_launch("qmv");
}

nvfp4_status qmv(const void* x, nvfp4_dtype x_dt, const float* g_x, const uint32_t* w_codes, const uint8_t* w_scales,
                 const float* g_w, int64_t M, int64_t N, int64_t K, void* y, nvfp4_stream_t stream) {
  return qmv_launch(x, x_dt, g_x, w_codes, w_scales, g_w, M, N, K, y, stream, false);
}

nvfp4_status qmv_mx(nvfp4_mode mode, const void* x, nvfp4_dtype x_dt, const uint32_t* w_codes,
                    const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, void* y, nvfp4_stream_t stream) {
  if (mode != NVFP4_MODE_MXFP8 && mode != NVFP4_MODE_MXFP4)
    return fail(NVFP4_ERR_INVALID_ARG, "[qmv_mx] mode must be mxfp8 or mxfp4 (nvfp4: use qmv)");
  if (!valid_dt(x_dt)) return fail(NVFP4_ERR_UNSUPPORTED, "[qmv_mx] dtype must be float32, float16 or bfloat16");
  if (M < 1 || M > kQmvMaxM)
    return fail(NVFP4_ERR_INVALID_ARG, "[qmv_mx] M must be in [1, %d], got %lld", kQmvMaxM, (long long)M);
  if (N < 0 || K < 32 || K % 32 != 0 || N > (1 << 30))
    return fail(NVFP4_ERR_INVALID_ARG, "[qmv_mx] bad shape N=%lld K=%lld (K %% 32 == 0)", (long long)N, (long long)K);
  if (M * K * 4 > 160 * 1024)
    return fail(NVFP4_ERR_UNSUPPORTED, "[qmv_mx] M*K*4 bytes of x_hat must fit 160 KiB of shared memory");
  if (N > 0 && (!x || !w_codes || !w_scales || !y)) return fail(NVFP4_ERR_INVALID_ARG, "[qmv_mx] null pointer");
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y))
    return fail(NVFP4_ERR_INVALID_ARG, "[qmv_mx] tensor pointers must be 16-byte aligned");
  if (N == 0) return ok();
  DeviceInfo d;
  nvfp4_status st = device_info("qmv_mx", &d);
  if (st != NVFP4_OK) return st;
  const size_t smem = (size_t)M * K * sizeof(float);
  uint64_t grid = ((uint64_t)N + (kQmvThreads / 32) - 1) / (kQmvThreads / 32);
  if (grid > (uint64_t)d.sm_count) grid = d.sm_count;
  cudaError_t e = cudaSuccess;
  dispatch_dt(x_dt, [&](auto tag_t) {
    using T = decltype(tag_t);
    auto go = [&](auto kern) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess)
        kern<<<(unsigned)grid, kQmvThreads, smem, stream>>>(static_cast<const T*>(x), w_codes, w_scales, (int)M,
                                                            (int)N, (int)K, static_cast<T*>(y));
    };
    auto pick = [&](auto mode_tag) {
      constexpr int MD = decltype(mode_tag)::value;
      if (M == 1) go(k_qmv_mx<T, MD, 1>);
      else if (M == 2) go(k_qmv_mx<T, MD, 2>);
      else if (M <= 4) go(k_qmv_mx<T, MD, 4>);
      else go(k_qmv_mx<T, MD, 8>);
    };
    if (mode == NVFP4_MODE_MXFP8) pick(std::integral_constant<int, 1>{});
    else pick(std::integral_constant<int, 2>{});
  });
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[qmv_mx] %s", cudaGetErrorString(e));
  return check_launch("qmv_mx");
}

nvfp4_status qmv_pdl(const void* x, nvfp4_dtype x_dt, const float* g_x, const uint32_t* w_codes,
                     const uint8_t* w_scales, const float* g_w, int64_t M, int64_t N, int64_t K, void* y,
                     nvfp4_stream_t stream) {
  return qmv_launch(x, x_dt, g_x, w_codes, w_scales, g_w, M, N, K, y, stream, true);
}

size_t gather_qmm_workspace_size(int64_t T, int64_t topk, int64_t E) {
  if (T < 0 || topk < 1 || E < 1 || E > gq::MAX_E || product_exceeds(T, topk, 1 << 30)) return 0;
  return gather_workspace_bytes(T, topk, E);
}

size_t gather_qmm_staged_workspace_size(int64_t T, int64_t topk, int64_t E, int64_t K) {
  if (T < 0 || topk < 1 || E < 1 || E > gq::MAX_E || K < 0 || K > (1 << 30) || product_exceeds(T, topk, 1 << 30))
    return 0;
  const int64_t P = T * topk;
  if (K > 0 && P > (int64_t)(SIZE_MAX / 4) / K) return 0;
  return gather_staged_workspace_bytes(T, topk, E, K);
}

// Host checks shared by the gather entries: shapes (K % 64, N % n_mult, K > 0
// when there is output), pointers and, where the caller passes one
// (check_ws), the workspace size.
static nvfp4_status check_gather(const char* tag, bool kn, const void* x, const uint32_t* w_codes,
                                 const uint8_t* w_scales, const float* g, const int32_t* idx, int64_t T,
                                 int64_t topk, int64_t E, int64_t N, int64_t K, const void* y, bool check_ws,
                                 const void* workspace, size_t workspace_bytes) {
  if (T < 0 || topk < 1 || E < 1 || N < 0 || K < 0 || product_exceeds(T, topk, 1 << 30) || N > (1 << 30) ||
      K > (1 << 30))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] bad shape", tag);
  const int n_mult = kn ? 32 : 16;
  if (K % 64 != 0 || N % n_mult != 0)
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] K must be a multiple of 64 and N of %d (K=%lld N=%lld)", tag, n_mult,
                (long long)K, (long long)N);
  if (K == 0 && T * N > 0) return fail(NVFP4_ERR_INVALID_ARG, "[%s] K must be positive when T*N > 0", tag);
  if (E > gq::MAX_E) return fail(NVFP4_ERR_UNSUPPORTED, "[%s] at most %d experts, got %lld", tag, gq::MAX_E, (long long)E);
  // The weight tensor map has E*N rows ([E, N, K]) or E*K rows ([E, K, N]);
  // TMA row coordinates are 32-bit signed.
  const int64_t w_rows = E * (kn ? K : N);
  if (w_rows > INT32_MAX)
    return fail(NVFP4_ERR_UNSUPPORTED, "[%s] the weights span %lld rows; at most %d", tag, (long long)w_rows,
                INT32_MAX);
  if (check_ws && workspace_bytes < gather_workspace_bytes(T, topk, E))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] workspace too small: %zu < %zu", tag, workspace_bytes,
                gather_workspace_bytes(T, topk, E));
  if (T * N > 0 && (!x || !w_codes || !w_scales || !idx || !y || (check_ws && !workspace)))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] null pointer", tag);
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y) || !aligned16(workspace) ||
      !aligned16(idx) || !aligned16(g))
    return fail(NVFP4_ERR_INVALID_ARG, "[%s] tensor pointers must be 16-byte aligned", tag);
  return NVFP4_OK;
}

nvfp4_status gather_qmm(const void* x, const uint32_t* w_codes, const uint8_t* w_scales, const float* g,
                        const int32_t* idx, int64_t T, int64_t topk, int64_t E, int64_t N, int64_t K, void* y,
                        void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  nvfp4_status st = check_gather("gather_qmm", false, x, w_codes, w_scales, g, idx, T, topk, E, N, K, y, true,
                                 workspace, workspace_bytes);
  if (st != NVFP4_OK) return st;
  if (T * N == 0) return ok();
  DeviceInfo d;
  st = device_info("gather_qmm", &d);
  if (st != NVFP4_OK) return st;
  return gather_qmm_launch(x, w_codes, w_scales, g, idx, T, topk, E, N, K, y, workspace, workspace_bytes, d.sm_count,
                           stream, t_msg, sizeof(t_msg));
}

nvfp4_status gather_qmm_kn(const void* x, const uint32_t* w_codes, const uint8_t* w_scales, const float* g,
                        const int32_t* idx, int64_t T, int64_t topk, int64_t E, int64_t N, int64_t K, void* y,
                        void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  nvfp4_status st = check_gather("gather_qmm_kn", true, x, w_codes, w_scales, g, idx, T, topk, E, N, K, y, true,
                                 workspace, workspace_bytes);
  if (st != NVFP4_OK) return st;
  if (T * N == 0) return ok();
  DeviceInfo d;
  st = device_info("gather_qmm_kn", &d);
  if (st != NVFP4_OK) return st;
  return gather_qmm_launch(x, w_codes, w_scales, g, idx, T, topk, E, N, K, y, workspace, workspace_bytes, d.sm_count,
                           stream, t_msg, sizeof(t_msg), true);
}

// Identity of the calling thread's current context (0 if none can be read):
// cuCtxGetCurrent and cuCtxGetId through the runtime's driver entry points,
// so the library needs no link against the driver library.
static unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static bool looked = false;
  if (!looked) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
    looked = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device, resolved with
// that device current and cached per device together with the context it
// belongs to: a new context on the device (after cudaDeviceReset, which
// unloads the library's module and may place the array elsewhere) resolves
// it again.
static nvfp4_status noalloc_scratch(void** out) {
  static void* addr[64] = {nullptr};
  static unsigned long long ctx_of[64] = {0};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(NVFP4_ERR_CUDA, "[gather_qmm_noalloc] cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(NVFP4_ERR_UNSUPPORTED, "[gather_qmm_noalloc] device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(NVFP4_ERR_CUDA, "[gather_qmm_noalloc] cudaGetSymbolAddress of the static scratch failed: %s",
                  cudaGetErrorString(e));
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  *out = addr[dev];
  return NVFP4_OK;
}

nvfp4_status gather_qmm_noalloc(const void* x, const uint32_t* w_codes, const uint8_t* w_scales, const float* g,
                                const int32_t* idx, int64_t T, int64_t topk, int64_t E, int64_t N, int64_t K,
                                void* y, nvfp4_stream_t stream) {
  nvfp4_status st = check_gather("gather_qmm_noalloc", false, x, w_codes, w_scales, g, idx, T, topk, E, N, K, y,
                                 false, nullptr, 0);
  if (st != NVFP4_OK) return st;
  if (T * N == 0) return ok();
  const size_t need = gather_workspace_bytes(T, topk, E);
  if (need > kNoAllocScratchBytes)
    return fail(NVFP4_ERR_UNSUPPORTED,
                "[gather_qmm_noalloc] T=%lld, topk=%lld, E=%lld needs %zu bytes of scratch; the static scratch "
                "holds %zu bytes (use gather_qmm with a caller-provided workspace)",
                (long long)T, (long long)topk, (long long)E, need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != NVFP4_OK) return st;
  // The routing kernel rewrites every scratch entry the grouped kernel reads
  // (tile count, tile list, permutation; the staging kernel the staged rows
  // of every routed pair), so nothing needs clearing between calls.
  return gather_qmm(x, w_codes, w_scales, g, idx, T, topk, E, N, K, y, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
