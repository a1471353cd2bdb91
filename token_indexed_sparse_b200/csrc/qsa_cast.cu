// FP32 -> BF16 rounding (round to nearest, ties to even) of a contiguous array:
// the final cast of FP32 dK / dV sums that were added up outside a single call
// (context parallelism reduces each rank's FP32 partials across ranks first),
// the same rounding the dK/dV kernel applies in its epilogue ("Selection and
// components" of the "Query Sparse Attention (QSA)" page: FP32 accumulation,
// BF16 gradients).
#include <cuda_bf16.h>

#include "qsa.h"
#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace qsa {
namespace {

// Grid-stride over 8-element groups: two 16-byte loads, one 16-byte store.
__global__ void __launch_bounds__(256) cast_f32_bf16_kernel(const float4* __restrict__ x, uint4* __restrict__ y,
                                                            int64_t n8) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = __ldcs(x + 2 * i), b = __ldcs(x + 2 * i + 1);
    __stcs(y + i, make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w)));
  }
}

// The last n % 8 elements, one thread each.
__global__ void cast_f32_bf16_tail_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, int64_t i0,
                                          int64_t n) {
  const int64_t i = i0 + threadIdx.x;
  if (i < n) y[i] = __float2bfloat16_rn(x[i]);
}

}  // namespace

cudaError_t launch_cast_f32_bf16(const float* x, void* y, int64_t n, cudaStream_t s) {
  const int64_t n8 = n / 8;
  if (n8 > 0) {
    const int64_t want = (n8 + 255) / 256;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    cast_f32_bf16_kernel<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, s>>>(
        reinterpret_cast<const float4*>(x), static_cast<uint4*>(y), n8);
  }
  if (n % 8 != 0)
    cast_f32_bf16_tail_kernel<<<1, 32, 0, s>>>(x, static_cast<__nv_bfloat16*>(y), n8 * 8, n);
  return cudaGetLastError();
}

}  // namespace qsa

extern "C" qsa_status_t qsa_cast_f32_to_bf16(const float* x, void* y, int64_t n, qsa_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return QSA_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0 || (reinterpret_cast<uintptr_t>(y) & 15) != 0)
    return QSA_ERR_MISALIGNED;
  if (n == 0) return QSA_OK;
  return qsa::launch_cast_f32_bf16(x, y, n, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? QSA_OK
                                                                                                    : QSA_ERR_CUDA;
}
