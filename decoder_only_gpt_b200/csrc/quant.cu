// e4m3 quantization of the forward block projections' operands (the page's
// "--fp8" option, "ChatGPT'nizi 50 Dolara Nasil Egitirsiniz?", section
// "Temel Komutlar").  Every scale is a power of two: 2^k with k the largest
// integer such that amax * 2^k <= 448 (e4m3's largest finite value; k = 0
// for an all-zero row or tensor), so scaling and the epilogue's unscaling
// are exact; the code is the e4m3 value nearest to x * 2^k (ties to even,
// the hardware conversion).  Activations get one scale per row (token),
// weights one per tensor.  Dequantization factors 2^-k are written as fp32.
#include <cuda_fp8.h>

#include "device_common.cuh"

namespace gpt {
namespace {

constexpr float kE4m3Max = 448.f;

// the largest k with amax * 2^k <= 448 (exact comparisons; 0 for amax == 0)
__device__ __forceinline__ int pow2_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int k = int(floorf(log2f(kE4m3Max / amax)));
  if (ldexpf(amax, k) > kE4m3Max) --k;
  if (ldexpf(amax, k + 1) <= kE4m3Max) ++k;
  return k;
}

__device__ __forceinline__ float amax8(const uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return m;
}

// 8 bf16 -> 8 e4m3 codes of x * 2^k
__device__ __forceinline__ uint2 quant8(const uint4 u, int k) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    const __nv_fp8x2_storage_t c =
        __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(f.x, k), ldexpf(f.y, k)), __NV_SATFINITE, __NV_E4M3);
    out[i >> 1] |= uint32_t(c) << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

// One warp per row of [rows, cols] bf16 (cols % 8 == 0): amax, k, codes.
__global__ void quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int cols,
                                  uint8_t* __restrict__ q, float* __restrict__ deq) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * cols);
  const int nv = cols / 8;
  float m = 0.f;
  for (int v = lane; v < nv; v += 32) m = fmaxf(m, amax8(src[v]));
  m = warp_max(m);
  const int k = pow2_exponent(m);
  uint2* dst = reinterpret_cast<uint2*>(q + row * cols);
  for (int v = lane; v < nv; v += 32) dst[v] = quant8(src[v], k);
  if (lane == 0) deq[row] = ldexpf(1.f, -k);
}

// Per-tensor amax of `n_mat` matrices of n elements each, matrix i starting
// at x + i * stride: the float bits of |x| order like unsigned integers, so an
// atomic max of the bits is exact and independent of the order.
__global__ void amax_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t stride,
                            unsigned* __restrict__ amax_bits) {
  const __nv_bfloat16* base = x + int64_t(blockIdx.y) * stride;
  float m = 0.f;
  for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < n / 8;
       v += int64_t(gridDim.x) * blockDim.x)
    m = fmaxf(m, amax8(reinterpret_cast<const uint4*>(base)[v]));
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + blockIdx.y, __float_as_uint(m));
}

__global__ void quant_tensor_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t stride,
                                    const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ q,
                                    float* __restrict__ deq) {
  const int k = pow2_exponent(__uint_as_float(amax_bits[blockIdx.y]));
  const int64_t off = int64_t(blockIdx.y) * stride;
  for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < n / 8;
       v += int64_t(gridDim.x) * blockDim.x)
    reinterpret_cast<uint2*>(q + off)[v] = quant8(reinterpret_cast<const uint4*>(x + off)[v], k);
  if (blockIdx.x == 0 && threadIdx.x == 0) deq[blockIdx.y] = ldexpf(1.f, -k);
}

}  // namespace

int launch_quant_rows(const void* x, int64_t rows, int cols, void* q, float* deq, void* stream) {
  if (cols % 8) return 1;
  quant_rows_kernel<<<int(ceil_div(rows, 8)), 256, 0, (cudaStream_t)stream>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, static_cast<uint8_t*>(q), deq);
  return last_launch_rc();
}

int launch_quant_tensors(const void* x, int64_t n, int64_t stride, int n_mat, void* q, float* deq,
                         unsigned* amax_bits, void* stream) {
  if (n % 8 || stride % 8 || n_mat <= 0) return 1;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(amax_bits, 0, sizeof(unsigned) * n_mat, st) != cudaSuccess) return 1;
  const int64_t want = ceil_div(n / 8, 256);
  const dim3 grid(unsigned(want < 148 ? want : 148), unsigned(n_mat));
  amax_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), n, stride, amax_bits);
  quant_tensor_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), n, stride, amax_bits,
                                            static_cast<uint8_t*>(q), deq);
  return last_launch_rc();
}

}  // namespace gpt
