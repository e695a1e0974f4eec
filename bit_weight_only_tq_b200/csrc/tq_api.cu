// tq_api.cu -- the extern "C" boundary of libtq.so (declared in include/tq.h): argument
// validation, path dispatch, and host utilities (tensor maps, device properties).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/tq.h"
#include "tq_common.cuh"

namespace tq {

bool decode_supported(bool int4, int64_t M, int64_t N, int64_t K);
static bool decode_ok(bool int4, int64_t M, int64_t N, int64_t K) { return decode_supported(int4, M, N, K); }
bool prefill_supported(bool int4, int64_t M, int64_t N, int64_t K);

static constexpr int kMaxDevices = 64;

DeviceInfo current_device_info() {
  // SM count per device, queried once; atomics because calls may come from several host threads
  static std::atomic<int> sms[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  DeviceInfo d{dev, 148};
  if (dev >= 0 && dev < kMaxDevices) {
    int v = sms[dev].load(std::memory_order_relaxed);
    if (v == 0) {
      if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
        sms[dev].store(v, std::memory_order_relaxed);
      else
        v = 0;
    }
    if (v > 0) d.num_sms = v;
  }
  return d;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                  uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                  const uint64_t strides_bytes[2], const uint32_t box[3], CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// An empty kernel launched in plain stream order after every call that writes packed weights,
// scales or zero-points.  The GEMM kernels read those model constants before
// griddepcontrol.wait (programmatic dependent launch lets them start while the previous kernel
// on the stream finishes); after this kernel, the previous kernel is always this one, which
// itself started only once the writer had completed and its writes were visible.
__global__ void constants_written_kernel() {}

cudaError_t after_constants_written(cudaStream_t s) {
  constants_written_kernel<<<1, 32, 0, s>>>();
  return cudaGetLastError();
}

cudaError_t ensure_smem_attr(const void* func, int bytes) {
  struct Entry {
    const void* f;
    int dev;
    int bytes;
  };
  static Entry cache[256];
  static int n = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n; ++i)
      if (cache[i].f == func && cache[i].dev == dev && cache[i].bytes >= bytes) return cudaSuccess;
  }
  const int want = 227 * 1024;  // set the maximum once per (function, device)
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes > want ? bytes : want);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (n < 256) cache[n++] = Entry{func, dev, bytes > want ? bytes : want};
  return cudaSuccess;
}

}  // namespace tq

// =============================================================================================
// extern "C" entry points
// =============================================================================================
namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int to_status(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Checks common to both GEMMs.  Returns TQ_OK, or an error; sets *empty for M == 0 or N == 0.
int check_gemm_args(const void* x, const void* w, const void* sc, const void* y, int64_t M,
                    int64_t N, int64_t K, bool* empty) {
  if (M < 0 || N < 0 || K <= 0) return TQ_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 28))
    return TQ_ERR_SHAPE;
  *empty = (M == 0 || N == 0);
  if (*empty) return TQ_OK;
  if (!x || !w || !sc || !y) return TQ_ERR_NULL;
  return TQ_OK;
}

int resolve_path(int fmt, int path, int64_t M, int64_t N, int64_t K, bool all_aligned) {
  const bool int4 = fmt == TQ_FMT_W4G128;
  switch (path) {
    case TQ_PATH_AUTO:
      return tq_select_path(fmt, M, N, K, all_aligned ? 1 : 0);
    case TQ_PATH_GENERIC:
      return TQ_PATH_GENERIC;
    case TQ_PATH_DECODE:
      if (!tq::decode_ok(int4, M, N, K)) return TQ_ERR_PATH;
      return all_aligned ? static_cast<int>(TQ_PATH_DECODE) : static_cast<int>(TQ_ERR_ALIGN);
    case TQ_PATH_PREFILL:
      if (!tq::prefill_supported(int4, M, N, K)) return TQ_ERR_PATH;
      return all_aligned ? static_cast<int>(TQ_PATH_PREFILL) : static_cast<int>(TQ_ERR_ALIGN);
    default:
      return TQ_ERR_PATH;
  }
}

// Shared driver of the grouped entry points: one decode launch when every matrix takes the
// decode path, one tensor-core launch when every matrix takes the prefill path, otherwise one
// single-matrix GEMM per matrix.
template <bool kInt4, typename WT, typename Single, typename Group>
static int gemm_grouped_impl(const uint16_t* x, int count, const WT* const* w,
                             const uint16_t* const* sc, const uint16_t* const* bias,
                             uint16_t* const* y, const int64_t* N, int64_t M, int64_t K,
                             void* stream, Single single, Group group) {
  if (count < 1 || count > 4) return TQ_ERR_SHAPE;
  if (!w || !sc || !y || !N) return TQ_ERR_NULL;
  if (M < 0 || K <= 0 || K > (int64_t(1) << 28) || M > (int64_t(1) << 31)) return TQ_ERR_SHAPE;
  if (kInt4 && K % 128 != 0) return TQ_ERR_SHAPE;
  bool all_decode = M >= 1 && M <= (kInt4 ? tq::kDecodeAutoMaxM_W4g : tq::kDecodeAutoMaxM_Ternary) && x &&
                    aligned16(x);
  for (int g = 0; g < count; ++g) {
    if (N[g] < 0 || N[g] > (int64_t(1) << 31)) return TQ_ERR_SHAPE;
    if (M > 0 && N[g] > 0 && (!w[g] || !sc[g] || !y[g])) return TQ_ERR_NULL;
    if (N[g] == 0) { all_decode = false; continue; }
    all_decode = all_decode && tq::decode_supported(kInt4, M, N[g], K) && aligned16(w[g]) &&
                 aligned16(y[g]) && (!kInt4 || aligned16(sc[g]));
  }
  if (M == 0) return TQ_OK;
  if (!x) return TQ_ERR_NULL;
  if (all_decode) {
    const __half* bh[4] = {nullptr, nullptr, nullptr, nullptr};
    for (int g = 0; g < count; ++g) bh[g] = bias ? reinterpret_cast<const __half*>(bias[g]) : nullptr;
    return to_status(group(reinterpret_cast<const __half*>(x), count, w,
                           reinterpret_cast<const __half* const*>(sc), bh,
                           reinterpret_cast<__half* const*>(y), N, M, K, as_stream(stream)));
  }
  // every non-empty matrix on the tensor-core path: one launch over all their row tiles
  {
    const int fmt = kInt4 ? TQ_FMT_W4G128 : TQ_FMT_TERNARY;
    int n = 0;
    const void* gw[4];
    const __half* gs[4];
    const __half* gb[4];
    __half* gy[4];
    int64_t gn[4];
    bool all_prefill = true;
    for (int g = 0; g < count && all_prefill; ++g) {
      if (N[g] == 0) continue;
      const bool al = aligned16(x) && aligned16(w[g]) && aligned16(y[g]) && (!kInt4 || aligned16(sc[g]));
      all_prefill = tq_select_path(fmt, M, N[g], K, al ? 1 : 0) == TQ_PATH_PREFILL;
      gw[n] = w[g];
      gs[n] = reinterpret_cast<const __half*>(sc[g]);
      gb[n] = bias ? reinterpret_cast<const __half*>(bias[g]) : nullptr;
      gy[n] = reinterpret_cast<__half*>(y[g]);
      gn[n] = N[g];
      ++n;
    }
    if (all_prefill && n > 1 && tq::prefill_grouping_pays(M, gn, n))
      return to_status(tq::launch_gemm_prefill_grouped(kInt4, reinterpret_cast<const __half*>(x), n, gw, gs, gb, gy,
                                                       gn, M, K, as_stream(stream)));
  }
  for (int g = 0; g < count; ++g) {
    const int st = single(x, w[g], sc[g], bias ? bias[g] : nullptr, y[g], M, N[g], K, stream);
    if (st != TQ_OK) return st;
  }
  return TQ_OK;
}

}  // namespace

extern "C" {

int tq_version(void) { return (1 << 16) | 0; }

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "ok";
    case TQ_ERR_NULL: return "a required pointer is NULL";
    case TQ_ERR_SHAPE: return "invalid shape";
    case TQ_ERR_ALIGN: return "misaligned pointer for the requested path";
    case TQ_ERR_DTYPE: return "unknown dtype";
    case TQ_ERR_CUDA: return "CUDA runtime or launch error";
    case TQ_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case TQ_ERR_INVALID_CODE: return "packed data holds the invalid ternary code 0b11";
    case TQ_ERR_PATH: return "unknown path, or the forced path cannot take this shape";
    default: return "unknown status";
  }
}

int tq_select_path(int fmt, int64_t M, int64_t N, int64_t K, int aligned) {
  if (fmt != TQ_FMT_TERNARY && fmt != TQ_FMT_W4G128) return TQ_ERR_PATH;
  const bool int4 = fmt == TQ_FMT_W4G128;
  if (M < 0 || N < 0 || K <= 0) return TQ_ERR_SHAPE;
  if (int4 && K % 128 != 0) return TQ_ERR_SHAPE;
  if (M == 0 || N == 0 || !aligned) return TQ_PATH_GENERIC;
  // Around the ridge of the fp16 tensor-core roofline the faster path was picked by measurement:
  // the decode kernel for skinny M, the tensor-core prefill kernel above the crossover.
  const int64_t dmax = int4 ? tq::kDecodeAutoMaxM_W4g : tq::kDecodeAutoMaxM_Ternary;
  if (M <= dmax && tq::decode_ok(int4, M, N, K)) return TQ_PATH_DECODE;
  if (tq::prefill_supported(int4, M, N, K)) return TQ_PATH_PREFILL;
  return TQ_PATH_GENERIC;
}

int tq_quantize_pack(const void* w, int w_dtype, uint8_t* packed, uint16_t* scale, int64_t N,
                     int64_t K, void* stream) {
  if (w_dtype != TQ_F32 && w_dtype != TQ_F16) return TQ_ERR_DTYPE;
  if (N < 0 || K <= 0 || K > (int64_t(1) << 28)) return TQ_ERR_SHAPE;
  if (N == 0) return TQ_OK;
  if (!w || !packed || !scale) return TQ_ERR_NULL;
  const cudaError_t e = tq::launch_tq_pack(w, w_dtype == TQ_F16, packed, scale, N, K, as_stream(stream));
  return to_status(e != cudaSuccess ? e : tq::after_constants_written(as_stream(stream)));
}

int w4g_quantize_pack(const void* w, int w_dtype, int32_t* qweight, uint16_t* scales, int64_t N,
                      int64_t K, void* stream) {
  if (w_dtype != TQ_F32 && w_dtype != TQ_F16) return TQ_ERR_DTYPE;
  if (N < 0 || K <= 0 || K % 128 != 0 || K > (int64_t(1) << 28)) return TQ_ERR_SHAPE;
  if (N == 0) return TQ_OK;
  if (!w || !qweight || !scales) return TQ_ERR_NULL;
  const cudaError_t e = tq::launch_w4g_pack(w, w_dtype == TQ_F16, qweight, scales, N, K, as_stream(stream));
  return to_status(e != cudaSuccess ? e : tq::after_constants_written(as_stream(stream)));
}

int tq_gemm_ex(const uint16_t* x, const uint8_t* packed, const uint16_t* scale,
               const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int path,
               void* stream) {
  bool empty = false;
  int st = check_gemm_args(x, packed, scale, y, M, N, K, &empty);
  if (st != TQ_OK) return st;
  if (path < TQ_PATH_AUTO || path > TQ_PATH_GENERIC) return TQ_ERR_PATH;
  if (empty) return TQ_OK;
  const bool al = aligned16(x) && aligned16(packed) && aligned16(y);
  const int p = resolve_path(TQ_FMT_TERNARY, path, M, N, K, al);
  if (p < 0) return p;
  const __half* xh = reinterpret_cast<const __half*>(x);
  const __half* sh = reinterpret_cast<const __half*>(scale);
  const __half* bh = reinterpret_cast<const __half*>(bias);
  __half* yh = reinterpret_cast<__half*>(y);
  cudaStream_t s = as_stream(stream);
  switch (p) {
    case TQ_PATH_DECODE: return to_status(tq::launch_tq_gemm_decode(xh, packed, sh, bh, yh, M, N, K, s));
    case TQ_PATH_PREFILL: return to_status(tq::launch_tq_gemm_prefill(xh, packed, sh, bh, yh, M, N, K, s));
    default: return to_status(tq::launch_tq_gemm_generic(xh, packed, sh, bh, yh, M, N, K, s));
  }
}

int tq_gemm(const uint16_t* x, const uint8_t* packed, const uint16_t* scale, const uint16_t* bias,
            uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream) {
  return tq_gemm_ex(x, packed, scale, bias, y, M, N, K, TQ_PATH_AUTO, stream);
}

}  // extern "C"

namespace {

int w4_gemm_impl(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, const uint8_t* zeros,
                 const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int path, void* stream) {
  bool empty = false;
  int st = check_gemm_args(x, qweight, scales, y, M, N, K, &empty);
  if (st != TQ_OK) return st;
  if (K % 128 != 0) return TQ_ERR_SHAPE;
  if (path < TQ_PATH_AUTO || path > TQ_PATH_GENERIC) return TQ_ERR_PATH;
  if (empty) return TQ_OK;
  const bool al = aligned16(x) && aligned16(qweight) && aligned16(y) && aligned16(scales);
  const int p = resolve_path(TQ_FMT_W4G128, path, M, N, K, al);
  if (p < 0) return p;
  const __half* xh = reinterpret_cast<const __half*>(x);
  const __half* sh = reinterpret_cast<const __half*>(scales);
  const __half* bh = reinterpret_cast<const __half*>(bias);
  __half* yh = reinterpret_cast<__half*>(y);
  cudaStream_t s = as_stream(stream);
  switch (p) {
    case TQ_PATH_DECODE: return to_status(tq::launch_w4g_gemm_decode(xh, qweight, sh, zeros, bh, yh, M, N, K, s));
    case TQ_PATH_PREFILL: return to_status(tq::launch_w4g_gemm_prefill(xh, qweight, sh, zeros, bh, yh, M, N, K, s));
    default: return to_status(tq::launch_w4g_gemm_generic(xh, qweight, sh, zeros, bh, yh, M, N, K, s));
  }
}

}  // namespace

extern "C" {

int w4g_gemm_ex(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
                const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int path,
                void* stream) {
  return w4_gemm_impl(x, qweight, scales, nullptr, bias, y, M, N, K, path, stream);
}

int w4g_gemm_zp_ex(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, const uint8_t* zeros,
                   const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int path, void* stream) {
  if (!zeros && M > 0 && N > 0) return TQ_ERR_NULL;
  return w4_gemm_impl(x, qweight, scales, zeros, bias, y, M, N, K, path, stream);
}

int w4g_gemm_zp(const uint16_t* x, const int32_t* qweight, const uint16_t* scales, const uint8_t* zeros,
                const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream) {
  return w4g_gemm_zp_ex(x, qweight, scales, zeros, bias, y, M, N, K, TQ_PATH_AUTO, stream);
}

int w4g_quantize_pack_ex(const void* w, int w_dtype, const int32_t* perm, int32_t* qweight, uint16_t* scales,
                         uint8_t* zeros, int32_t* g_idx, int64_t N, int64_t K, void* stream) {
  if (w_dtype != TQ_F32 && w_dtype != TQ_F16) return TQ_ERR_DTYPE;
  if (N < 0 || K <= 0 || K % 128 != 0 || K > (int64_t(1) << 28)) return TQ_ERR_SHAPE;
  if (N == 0) {
    if (g_idx && perm) return TQ_ERR_SHAPE;  // g_idx of an empty matrix in act order: nothing defines it
    return g_idx ? to_status(tq::launch_iota_groups(g_idx, K, as_stream(stream))) : TQ_OK;
  }
  if (!w || !qweight || !scales) return TQ_ERR_NULL;
  const cudaError_t e =
      tq::launch_w4g_pack_ex(w, w_dtype == TQ_F16, perm, qweight, scales, zeros, g_idx, N, K, as_stream(stream));
  return to_status(e != cudaSuccess ? e : tq::after_constants_written(as_stream(stream)));
}

int tq_permute_columns(const uint16_t* x, const int32_t* perm, uint16_t* out, int64_t M, int64_t K, void* stream) {
  if (M < 0 || K <= 0) return TQ_ERR_SHAPE;
  if (M == 0) return TQ_OK;
  if (!x || !perm || !out) return TQ_ERR_NULL;
  return to_status(tq::launch_permute_cols(x, perm, out, M, K, as_stream(stream)));
}

int w4g_repack_act_order(const int32_t* qweight, const int32_t* perm, int32_t* out, int64_t N, int64_t K,
                         void* stream) {
  if (N < 0 || K <= 0 || K % 8 != 0) return TQ_ERR_SHAPE;
  if (N == 0) return TQ_OK;
  if (!qweight || !perm || !out) return TQ_ERR_NULL;
  const cudaError_t e = tq::launch_repack_act_order(qweight, perm, out, N, K, as_stream(stream));
  return to_status(e != cudaSuccess ? e : tq::after_constants_written(as_stream(stream)));
}

int w4g_gemm(const uint16_t* x, const int32_t* qweight, const uint16_t* scales,
             const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, void* stream) {
  return w4g_gemm_ex(x, qweight, scales, bias, y, M, N, K, TQ_PATH_AUTO, stream);
}

int tq_gemm_grouped(const uint16_t* x, int count, const uint8_t* const* packed,
                    const uint16_t* const* scale, const uint16_t* const* bias, uint16_t* const* y,
                    const int64_t* N, int64_t M, int64_t K, void* stream) {
  return gemm_grouped_impl<false>(x, count, packed, scale, bias, y, N, M, K, stream, tq_gemm,
                                  tq::launch_tq_gemm_decode_group);
}

int w4g_gemm_grouped(const uint16_t* x, int count, const int32_t* const* qweight,
                     const uint16_t* const* scales, const uint16_t* const* bias,
                     uint16_t* const* y, const int64_t* N, int64_t M, int64_t K, void* stream) {
  return gemm_grouped_impl<true>(x, count, qweight, scales, bias, y, N, M, K, stream, w4g_gemm,
                                 tq::launch_w4g_gemm_decode_group);
}

int tq_debug_set_wait_limit(long long cycles) {
  const long long v = cycles > 0 ? cycles : tq::kWaitLimitCycles;
  return to_status(cudaMemcpyToSymbol(tq::g_tq_wait_limit, &v, sizeof(v)));
}

int tq_debug_skip_activation_loads(int on) {
  const int v = on ? 1 : 0;
  return to_status(cudaMemcpyToSymbol(tq::g_tq_skip_x_loads, &v, sizeof(v)));
}

size_t tq_batch_workspace_size(void) { return static_cast<size_t>(tq::batch_workspace_bytes()); }

}  // extern "C"

namespace {

template <bool kInt4>
int gemm_batch_impl(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                    int variant, void* stream, const tq_linear* next = nullptr, int next_count = 0,
                    int64_t next_M = 0) {
  if (count < 1 || count > tq::kBatchMaxItems) return TQ_ERR_SHAPE;
  if (next_count < 0 || next_count > tq::kBatchMaxItems || next_M < 0 || next_M > tq::kBatchMaxM) return TQ_ERR_SHAPE;
  if (next_count > 0 && !next) return TQ_ERR_NULL;
  tq::BatchLinear nlin[tq::kBatchMaxItems];
  int nn = 0;
  for (int i = 0; i < next_count; ++i) {
    const tq_linear& it = next[i];
    if (it.N < 0 || it.N > (int64_t(1) << 31) || it.K <= 0 || it.K > (int64_t(1) << 28)) return TQ_ERR_SHAPE;
    if (kInt4 ? (it.K % 128 != 0) : (it.K % 64 != 0)) return TQ_ERR_SHAPE;
    if (it.N == 0) continue;
    if (!it.w) return TQ_ERR_NULL;
    if (!aligned16(it.w)) return TQ_ERR_ALIGN;
    nlin[nn++] = tq::BatchLinear{nullptr, it.w, nullptr, nullptr, nullptr, it.N, it.K, nullptr};
  }
  tq::BatchNext nx;
  nx.items = nlin;
  nx.count = nn;
  nx.M = next_M;
  const bool il = (variant & TQ_BATCH_INTERLEAVED) != 0;  // ternary weights in the interleaved layout
  variant &= ~TQ_BATCH_INTERLEAVED;
  if (variant < TQ_BATCH_AUTO || variant > TQ_BATCH_TENSOR_CORE) return TQ_ERR_PATH;
  if (M < 0 || M > tq::kBatchMaxM) return TQ_ERR_SHAPE;
  if (variant == TQ_BATCH_AUTO) variant = M <= 16 ? TQ_BATCH_MMA_SYNC : TQ_BATCH_TENSOR_CORE;
  if (variant == TQ_BATCH_MMA_SYNC && M > 16) return TQ_ERR_PATH;
  if (il && (kInt4 || variant != TQ_BATCH_MMA_SYNC)) return TQ_ERR_PATH;
  if (!items) return TQ_ERR_NULL;
  tq::BatchLinear lin[tq::kBatchMaxItems];
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const tq_linear& it = items[i];
    if (it.N < 0 || it.N > (int64_t(1) << 31) || it.K <= 0 || it.K > (int64_t(1) << 28)) return TQ_ERR_SHAPE;
    if (kInt4 ? (it.K % 128 != 0) : (it.K % 64 != 0)) return TQ_ERR_SHAPE;
    if (it.N == 0) continue;
    if (!it.x || !it.w || !it.scale || !it.y) return TQ_ERR_NULL;
    if (!aligned16(it.x) || !aligned16(it.w)) return TQ_ERR_ALIGN;
    lin[n++] = tq::BatchLinear{reinterpret_cast<const __half*>(it.x), it.w, reinterpret_cast<const __half*>(it.scale),
                               reinterpret_cast<const __half*>(it.bias), reinterpret_cast<__half*>(it.y), it.N, it.K,
                               kInt4 ? it.zeros : nullptr};
  }
  if (M == 0 || n == 0) return TQ_OK;
  if (!workspace) return TQ_ERR_NULL;
  if (!aligned16(workspace)) return TQ_ERR_ALIGN;
  if (static_cast<int64_t>(workspace_bytes) < tq::batch_workspace_bytes()) return TQ_ERR_SHAPE;
  const int64_t wb = static_cast<int64_t>(workspace_bytes);
  cudaError_t e;
  if (variant == TQ_BATCH_TENSOR_CORE)
    e = tq::launch_gemm_batch_tc(kInt4, lin, n, M, workspace, wb, as_stream(stream));
  else
    e = kInt4 ? tq::launch_w4g_gemm_batch(lin, n, M, workspace, wb, as_stream(stream), nx)
              : tq::launch_tq_gemm_batch(lin, n, M, workspace, wb, as_stream(stream), il, nx);
  return to_status(e);
}

}  // namespace

extern "C" {

int tq_gemm_batch(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                  void* stream) {
  return gemm_batch_impl<false>(items, count, M, workspace, workspace_bytes, TQ_BATCH_AUTO, stream);
}

int w4g_gemm_batch(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                   void* stream) {
  return gemm_batch_impl<true>(items, count, M, workspace, workspace_bytes, TQ_BATCH_AUTO, stream);
}

int tq_gemm_batch_ex(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                     int variant, void* stream) {
  return gemm_batch_impl<false>(items, count, M, workspace, workspace_bytes, variant, stream);
}

int w4g_gemm_batch_ex(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                      int variant, void* stream) {
  return gemm_batch_impl<true>(items, count, M, workspace, workspace_bytes, variant, stream);
}

int tq_gemm_batch_next(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                       int variant, const tq_linear* next, int next_count, int64_t next_M, void* stream) {
  return gemm_batch_impl<false>(items, count, M, workspace, workspace_bytes, variant, stream, next, next_count,
                                next_M);
}

int w4g_gemm_batch_next(const tq_linear* items, int count, int64_t M, void* workspace, size_t workspace_bytes,
                        int variant, const tq_linear* next, int next_count, int64_t next_M, void* stream) {
  return gemm_batch_impl<true>(items, count, M, workspace, workspace_bytes, variant, stream, next, next_count,
                               next_M);
}

int tq_interleave_packed(const uint8_t* packed, uint8_t* out, int64_t N, int64_t K, void* stream) {
  if (N < 0 || K <= 0 || K % 16 != 0 || N > (int64_t(1) << 31) || K > (int64_t(1) << 28)) return TQ_ERR_SHAPE;
  if (N == 0) return TQ_OK;
  if (!packed || !out) return TQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(packed) | reinterpret_cast<uintptr_t>(out)) & 3u) return TQ_ERR_ALIGN;
  cudaError_t e = tq::launch_tq_interleave(reinterpret_cast<const uint32_t*>(packed), reinterpret_cast<uint32_t*>(out),
                                           N * (K / 16), as_stream(stream));
  if (e == cudaSuccess) e = tq::after_constants_written(as_stream(stream));
  return to_status(e);
}

int tq_shard_plan(int fmt, int mode, int64_t N, int64_t K, int world, int rank, tq_shard* out) {
  if (!out) return TQ_ERR_NULL;
  if (fmt != TQ_FMT_TERNARY && fmt != TQ_FMT_W4G128) return TQ_ERR_PATH;
  if (mode != TQ_SHARD_ROWS && mode != TQ_SHARD_K) return TQ_ERR_PATH;
  if (world < 1 || rank < 0 || rank >= world || N < 0 || K <= 0) return TQ_ERR_SHAPE;
  const bool int4 = fmt == TQ_FMT_W4G128;
  if (int4 && K % 128 != 0) return TQ_ERR_SHAPE;
  const int64_t pf = int4 ? 8 : 4;  // packed factor: elements per byte (ternary) / per int32 word
  tq_shard r{};
  if (mode == TQ_SHARD_ROWS) {
    r.row0 = N * rank / world;
    r.rows = N * (rank + 1) / world - r.row0;
    r.k0 = 0;
    r.cols = K;
    r.packed0 = 0;
    r.packed = (K + pf - 1) / pf;
    r.group0 = 0;
    r.groups = int4 ? K / 128 : 0;
    r.scale_full = 0;
  } else {
    const int64_t unit = int4 ? 128 : 4;
    if (K % world != 0 || (K / world) % unit != 0) return TQ_ERR_SHAPE;
    r.row0 = 0;
    r.rows = N;
    r.cols = K / world;
    r.k0 = r.cols * rank;
    r.packed0 = r.k0 / pf;
    r.packed = r.cols / pf;
    r.group0 = int4 ? r.k0 / 128 : 0;
    r.groups = int4 ? r.cols / 128 : 0;
    r.scale_full = int4 ? 0 : 1;
  }
  *out = r;
  return TQ_OK;
}

int tq_validate_packed(const uint8_t* packed, int64_t N, int64_t K, int* bad_count, void* stream) {
  if (N < 0 || K <= 0) return TQ_ERR_SHAPE;
  if (!bad_count) return TQ_ERR_NULL;
  if (N > 0 && !packed) return TQ_ERR_NULL;
  if (N == 0) return to_status(cudaMemsetAsync(bad_count, 0, sizeof(int), as_stream(stream)));
  return to_status(tq::launch_tq_validate(packed, N, K, bad_count, as_stream(stream)));
}

int tq_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return TQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_tq_device_status, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(tq::g_tq_device_status, &zero, sizeof(int)) != cudaSuccess)
    return TQ_ERR_CUDA;
  return v == 0 ? TQ_OK : TQ_ERR_TIMEOUT;
}

}  // extern "C"
