// tq_generic.cu -- shape- and alignment-agnostic GEMM kernels (CUDA cores, fp32 accumulation)
// and the packed-data validator.
//
// These take any M, N, K (including K % 4 != 0 with the ceil(K/4) row stride of [TQ] §3.2) and
// any pointer alignment.  They are the device path for shapes the fast kernels do not cover;
// they are correct, not fast.  One warp per output column n, MT tokens per warp.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

constexpr int kGenWarps = 8;
constexpr int kGenMT = 4;

__global__ void __launch_bounds__(kGenWarps * 32)
    tq_gemm_generic_kernel(const __half* __restrict__ x, const uint8_t* __restrict__ packed,
                           const __half* __restrict__ scale, const __half* __restrict__ bias,
                           __half* __restrict__ y, int64_t M, int64_t N, int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kGenWarps + (threadIdx.x >> 5);
  if (n >= N) return;
  const int64_t KB = (K + 3) >> 2;
  const uint8_t* prow = packed + n * KB;
  for (int64_t m0 = static_cast<int64_t>(blockIdx.y) * kGenMT; m0 < M;
       m0 += static_cast<int64_t>(gridDim.y) * kGenMT) {
    float acc[kGenMT];
#pragma unroll
    for (int i = 0; i < kGenMT; ++i) acc[i] = 0.0f;
    for (int64_t j = lane; j < KB; j += 32) {
      const uint32_t b = prow[j];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t k = 4 * j + i;
        if (k >= K) break;
        const float v = static_cast<float>(static_cast<int>((b >> (2 * i)) & 3u) - 1);
#pragma unroll
        for (int mm = 0; mm < kGenMT; ++mm)
          if (m0 + mm < M) acc[mm] = fmaf(v, __half2float(x[(m0 + mm) * K + k]), acc[mm]);
      }
    }
#pragma unroll
    for (int mm = 0; mm < kGenMT; ++mm) acc[mm] = warp_sum(acc[mm]);
    if (lane == 0) {
      const float sc = __half2float(scale[n]);
      const float bs = bias ? __half2float(bias[n]) : 0.0f;
#pragma unroll
      for (int mm = 0; mm < kGenMT; ++mm)
        if (m0 + mm < M) y[(m0 + mm) * N + n] = __float2half_rn(fmaf(sc, acc[mm], bs));
    }
  }
}

__global__ void __launch_bounds__(kGenWarps * 32)
    w4g_gemm_generic_kernel(const __half* __restrict__ x, const int32_t* __restrict__ qweight,
                            const __half* __restrict__ scales, const uint8_t* __restrict__ zeros,
                            const __half* __restrict__ bias, __half* __restrict__ y, int64_t M, int64_t N,
                            int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kGenWarps + (threadIdx.x >> 5);
  if (n >= N) return;
  const int64_t KW = K >> 3, G = K >> 7;
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qweight) + n * KW;
  for (int64_t m0 = static_cast<int64_t>(blockIdx.y) * kGenMT; m0 < M;
       m0 += static_cast<int64_t>(gridDim.y) * kGenMT) {
    float acc[kGenMT];
#pragma unroll
    for (int i = 0; i < kGenMT; ++i) acc[i] = 0.0f;
    for (int64_t j = lane; j < KW; j += 32) {
      const uint32_t wd = qrow[j];
      const float s = __half2float(scales[n * G + (j >> 4)]);
      const int z = zeros ? static_cast<int>(zeros[n * G + (j >> 4)]) : 8;  // symmetric: u - 8
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t k = 8 * j + i;
        const float v = s * static_cast<float>(static_cast<int>((wd >> (4 * i)) & 0xFu) - z);
#pragma unroll
        for (int mm = 0; mm < kGenMT; ++mm)
          if (m0 + mm < M) acc[mm] = fmaf(v, __half2float(x[(m0 + mm) * K + k]), acc[mm]);
      }
    }
#pragma unroll
    for (int mm = 0; mm < kGenMT; ++mm) acc[mm] = warp_sum(acc[mm]);
    if (lane == 0) {
      const float bs = bias ? __half2float(bias[n]) : 0.0f;
#pragma unroll
      for (int mm = 0; mm < kGenMT; ++mm)
        if (m0 + mm < M) y[(m0 + mm) * N + n] = __float2half_rn(acc[mm] + bs);
    }
  }
}

// Count bytes holding code 0b11 among the first K codes of their row.
__global__ void tq_validate_kernel(const uint8_t* __restrict__ packed, int64_t N, int64_t K,
                                   int* __restrict__ bad) {
  const int64_t KB = (K + 3) >> 2;
  const int64_t total = N * KB;
  int local = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = i % KB;
    const uint32_t b = packed[i];
    const int64_t valid = (K - 4 * j) < 4 ? (K - 4 * j) : 4;
    bool isbad = false;
    for (int c = 0; c < valid; ++c) isbad |= ((b >> (2 * c)) & 3u) == 3u;
    local += isbad ? 1 : 0;
  }
  local = warp_sum(local);
  if ((threadIdx.x & 31) == 0 && local) atomicAdd(bad, local);
}

// ---------------------------------------------------------------------------------------------
// Activation order ([VQ] §5 g_idx; [VQ] §4.3: the Marlin path reorders the weights once after
// loading).  With the columns of each group scattered over K, the product is taken in the
// processing order instead: x . What^T = (x P) . (What P)^T for the column permutation P.
// ---------------------------------------------------------------------------------------------
// out[m, j] = x[m, perm[j]] (fp16).
__global__ void permute_cols_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                                    uint16_t* __restrict__ out, int64_t M, int64_t K) {
  const int64_t total = M * K;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / K, j = i - m * K;
    const int64_t c = __ldg(perm + j);
    out[i] = (c >= 0 && c < K) ? x[m * K + c] : static_cast<uint16_t>(0);  // guard: perm not a permutation
  }
}

// Output word j of row n holds, in nibble i, the input nibble of column perm[8j + i].
__global__ void repack_act_order_kernel(const int32_t* __restrict__ qweight, const int32_t* __restrict__ perm,
                                        int32_t* __restrict__ out, int64_t N, int64_t K) {
  const int64_t KW = K >> 3, total = N * KW;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / KW, j = i - n * KW;
    const uint32_t* row = reinterpret_cast<const uint32_t*>(qweight) + n * KW;
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int64_t c = __ldg(perm + 8 * j + q);
      if (c < 0 || c >= K) continue;  // guard: perm not a permutation
      word |= ((__ldg(row + (c >> 3)) >> (4 * (c & 7))) & 0xFu) << (4 * q);
    }
    out[i] = static_cast<int32_t>(word);
  }
}

__global__ void iota_groups_kernel(int32_t* __restrict__ g_idx, int64_t K) {
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < K;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x)
    g_idx[k] = static_cast<int32_t>(k >> 7);
}

static unsigned elementwise_grid(int64_t total) {
  const DeviceInfo di = current_device_info();
  int64_t grid = (total + 255) / 256;
  if (grid > int64_t(di.num_sms) * 16) grid = int64_t(di.num_sms) * 16;
  return static_cast<unsigned>(grid < 1 ? 1 : grid);
}

cudaError_t launch_permute_cols(const uint16_t* x, const int32_t* perm, uint16_t* out, int64_t M, int64_t K,
                                cudaStream_t s) {
  permute_cols_kernel<<<elementwise_grid(M * K), 256, 0, s>>>(x, perm, out, M, K);
  return cudaGetLastError();
}

cudaError_t launch_repack_act_order(const int32_t* qweight, const int32_t* perm, int32_t* out, int64_t N,
                                    int64_t K, cudaStream_t s) {
  repack_act_order_kernel<<<elementwise_grid(N * (K >> 3)), 256, 0, s>>>(qweight, perm, out, N, K);
  return cudaGetLastError();
}

cudaError_t launch_iota_groups(int32_t* g_idx, int64_t K, cudaStream_t s) {
  iota_groups_kernel<<<elementwise_grid(K), 256, 0, s>>>(g_idx, K);
  return cudaGetLastError();
}

static unsigned gen_grid_y(int64_t M) {
  int64_t gy = (M + kGenMT - 1) / kGenMT;
  if (gy > 64) gy = 64;
  return static_cast<unsigned>(gy < 1 ? 1 : gy);
}

cudaError_t launch_tq_gemm_generic(const __half* x, const uint8_t* packed, const __half* scale,
                                   const __half* bias, __half* y, int64_t M, int64_t N, int64_t K,
                                   cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((N + kGenWarps - 1) / kGenWarps), gen_grid_y(M));
  tq_gemm_generic_kernel<<<grid, kGenWarps * 32, 0, s>>>(x, packed, scale, bias, y, M, N, K);
  return cudaGetLastError();
}

cudaError_t launch_w4g_gemm_generic(const __half* x, const int32_t* qweight, const __half* scales,
                                    const uint8_t* zeros, const __half* bias, __half* y, int64_t M, int64_t N,
                                    int64_t K, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((N + kGenWarps - 1) / kGenWarps), gen_grid_y(M));
  w4g_gemm_generic_kernel<<<grid, kGenWarps * 32, 0, s>>>(x, qweight, scales, zeros, bias, y, M, N, K);
  return cudaGetLastError();
}

cudaError_t launch_tq_validate(const uint8_t* packed, int64_t N, int64_t K, int* bad,
                               cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(bad, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  const DeviceInfo di = current_device_info();
  const int64_t total = N * ((K + 3) >> 2);
  int64_t grid = (total + 255) / 256;
  if (grid > int64_t(di.num_sms) * 8) grid = int64_t(di.num_sms) * 8;
  if (grid < 1) grid = 1;
  tq_validate_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(packed, N, K, bad);
  return cudaGetLastError();
}

}  // namespace tq
