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

// the largest k with amax * 2^k <= 448 (0 for a zero or non-finite amax).
// For a normal amax = m 2^e (1 <= m < 2) and 448 = 1.75 2^8 that is 8 - e
// when m <= 1.75 and 7 - e otherwise, read off the float's bits; a subnormal
// amax takes the same comparisons through ldexpf.
__device__ __forceinline__ int pow2_exponent(float amax) {
  if (!(amax > 0.f) || !(amax <= 3.40282347e38f)) return 0;
  const uint32_t b = __float_as_uint(amax);
  const int ef = int(b >> 23);
  if (ef != 0) return ((b & 0x7FFFFFu) <= 0x600000u ? 8 : 7) - (ef - 127);
  int k = int(floorf(log2f(kE4m3Max / amax)));
  if (ldexpf(amax, k) > kE4m3Max) --k;
  if (ldexpf(amax, k + 1) <= kE4m3Max) ++k;
  return k;
}

// 2^k as a float multiplier: exact for -126 <= k <= 127, where x * 2^k is
// x scaled exactly (or rounded once into the subnormals, as ldexpf would)
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float(uint32_t(127 + k) << 23); }

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
  const bool fast = k >= -126 && k <= 127;
  const float s = fast ? pow2f(k) : 1.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    if (fast) {
      f.x *= s;
      f.y *= s;
    } else {
      f.x = ldexpf(f.x, k);
      f.y = ldexpf(f.y, k);
    }
    const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
    out[i >> 1] |= uint32_t(c) << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

// One warp per row of [rows, cols] bf16 with cols = 256 * PER (PER 16-byte
// units per lane, held in registers, so the row is read once): amax, k, codes.
// Only for rows narrow enough that several blocks still fit an SM (PER <= 8);
// wider rows take the two-pass kernel below, whose second read hits L1.
// blocks of 256 threads per SM that the row's registers (4 per unit) leave room for
constexpr int reg_blocks(int per) { return per <= 4 ? 4 : per <= 6 ? 3 : 2; }

template <int PER>
__global__ void __launch_bounds__(256, reg_blocks(PER)) quant_rows_reg_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                      uint8_t* __restrict__ q, float* __restrict__ deq) {
  constexpr int cols = 256 * PER;
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * cols);
  uint4 v[PER];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    v[i] = src[lane + 32 * i];
    m = fmaxf(m, amax8(v[i]));
  }
  m = warp_max(m);
  const int k = pow2_exponent(m);
  uint2* dst = reinterpret_cast<uint2*>(q + row * cols);
#pragma unroll
  for (int i = 0; i < PER; ++i) dst[lane + 32 * i] = quant8(v[i], k);
  if (lane == 0) deq[row] = ldexpf(1.f, -k);
}

// One block of 192 threads (6 warps) per row of [rows, cols] bf16 with cols =
// 8 * 192 * PER: the row in registers (PER 16-byte units per thread), its
// amax reduced across the warps through shared memory, so it is read once.
// For the wide rows (q|k|v columns, d_ff) at full occupancy.
constexpr int kRowThreads = 192;
template <int PER>
__global__ void __launch_bounds__(kRowThreads, PER <= 4 ? 6 : 4) quant_rows_block_kernel(const __nv_bfloat16* __restrict__ x,
                                                                       uint8_t* __restrict__ q,
                                                                       float* __restrict__ deq) {
  constexpr int cols = 8 * kRowThreads * PER;
  __shared__ float wmax[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * cols);
  uint4 v[PER];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    v[i] = src[t + kRowThreads * i];
    m = fmaxf(m, amax8(v[i]));
  }
  m = warp_max(m);
  if ((t & 31) == 0) wmax[t >> 5] = m;
  __syncthreads();
  m = wmax[0];
#pragma unroll
  for (int w = 1; w < kRowThreads / 32; ++w) m = fmaxf(m, wmax[w]);
  const int k = pow2_exponent(m);
  uint2* dst = reinterpret_cast<uint2*>(q + row * cols);
#pragma unroll
  for (int i = 0; i < PER; ++i) dst[t + kRowThreads * i] = quant8(v[i], k);
  if (t == 0) deq[row] = ldexpf(1.f, -k);
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

// The per-tensor codes of W^T: matrix i of `n_mat` (at x + i * stride) is
// [R, C] bf16; its codes are written transposed, [C, R], at q + i * stride,
// with the scale of the amax already in amax_bits[i] (the forward's).  A block
// moves one 64 x 64 tile through shared memory: coalesced 16-byte loads of W's
// rows, 16-byte stores of the codes' rows.
__global__ void quant_tensor_t_kernel(const __nv_bfloat16* __restrict__ x, int R, int C, int64_t stride,
                                      const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ q) {
  __shared__ uint16_t tile[64][66];  // [r][c] bf16 bits; rows padded to 33 words
  const int64_t off = int64_t(blockIdx.z) * stride;
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
  const int t = threadIdx.x;
  {  // load: thread t takes row t / 4, columns 16 (t % 4) .. + 15
    const int r = t >> 2, c = (t & 3) * 16;
    const uint4* src = reinterpret_cast<const uint4*>(x + off + int64_t(r0 + r) * C + c0 + c);
    const uint4 a = src[0], b = src[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      tile[r][c + 2 * i] = uint16_t(w[i] & 0xFFFFu);
      tile[r][c + 2 * i + 1] = uint16_t(w[i] >> 16);
    }
  }
  __syncthreads();
  const int k = pow2_exponent(__uint_as_float(amax_bits[blockIdx.z]));
  const bool fast = k >= -126 && k <= 127;
  const float sc = fast ? pow2f(k) : 1.f;
  // store: thread t takes code row c = t / 4 (W's column), entries 16 (t % 4) .. + 15 (W's rows)
  const int c = t >> 2, rb = (t & 3) * 16;
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    float2 f = make_float2(__uint_as_float(uint32_t(tile[rb + i][c]) << 16),
                           __uint_as_float(uint32_t(tile[rb + i + 1][c]) << 16));
    if (fast) {
      f.x *= sc;
      f.y *= sc;
    } else {
      f.x = ldexpf(f.x, k);
      f.y = ldexpf(f.y, k);
    }
    const __nv_fp8x2_storage_t cc = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
    out[i >> 2] |= uint32_t(cc) << (16 * ((i >> 1) & 1));
  }
  *reinterpret_cast<uint4*>(q + off + int64_t(c0 + c) * R + r0 + rb) = make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace

int launch_quant_tensors_t(const void* x, int rows, int cols, int64_t stride, int n_mat,
                           const unsigned* amax_bits, void* q, void* stream) {
  if (rows % 64 || cols % 64 || stride % 16 || n_mat <= 0) return 1;
  const dim3 grid(unsigned(cols / 64), unsigned(rows / 64), unsigned(n_mat));
  quant_tensor_t_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(static_cast<const __nv_bfloat16*>(x), rows, cols,
                                                                 stride, amax_bits, static_cast<uint8_t*>(q));
  return last_launch_rc();
}

int launch_quant_rows(const void* x, int64_t rows, int cols, void* q, float* deq, void* stream) {
  if (cols % 8) return 1;
  cudaStream_t st = (cudaStream_t)stream;
  const int grid = int(ceil_div(rows, 8));
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* qb = static_cast<uint8_t*>(q);
  const unsigned nb = unsigned(rows);
  switch (cols) {  // the model's widths: warp per row up to 2048, block per row above
    case 512: quant_rows_reg_kernel<2><<<grid, 256, 0, st>>>(xb, rows, qb, deq); break;
    case 768: quant_rows_reg_kernel<3><<<grid, 256, 0, st>>>(xb, rows, qb, deq); break;
    case 1024: quant_rows_reg_kernel<4><<<grid, 256, 0, st>>>(xb, rows, qb, deq); break;
    case 1536: quant_rows_reg_kernel<6><<<grid, 256, 0, st>>>(xb, rows, qb, deq); break;
    case 2048: quant_rows_reg_kernel<8><<<grid, 256, 0, st>>>(xb, rows, qb, deq); break;
    case 3072: quant_rows_block_kernel<2><<<nb, kRowThreads, 0, st>>>(xb, qb, deq); break;
    case 4608: quant_rows_block_kernel<3><<<nb, kRowThreads, 0, st>>>(xb, qb, deq); break;
    case 6144: quant_rows_block_kernel<4><<<nb, kRowThreads, 0, st>>>(xb, qb, deq); break;
    case 9216: quant_rows_block_kernel<6><<<nb, kRowThreads, 0, st>>>(xb, qb, deq); break;
    default: quant_rows_kernel<<<grid, 256, 0, st>>>(xb, rows, cols, qb, deq);
  }
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
