// mxfp8.cu -- MXFP8 quantisation of a cache tensor (the zhichai.net summary
// of "MiniMax Sparse Attention": an MXFP8 KV cache).
//
// Format (OCP Microscaling formats v1.0, MXFP8 E4M3): blocks of 32
// consecutive elements along the last dimension share one E8M0 scale 2^e,
// e = floor(log2 max|x|) - 8 (8: the exponent of the largest E4M3 normal,
// 448 = 1.75 * 2^8), clamped to [-127, 127] (a block of zeros takes -127);
// each element is x / 2^e rounded to the E4M3 grid, nearest even, saturated at
// +-448.  The scale byte is e + 127.  The division by a power of two is exact
// in fp32, and cvt.rn.satfinite rounds and saturates as the format asks.
#include <cstdint>
#include <cuda_runtime.h>

#include "msa_internal.h"
#include "ptx.cuh"

namespace msa {
namespace {

constexpr int kQuantThreads = 256;

// One thread per 32-element block: 64 bytes of bf16 in, 32 + 1 bytes out.
__global__ void __launch_bounds__(kQuantThreads) quantize_mxfp8_kernel(const uint16_t* __restrict__ x,
                                                                       long long n_blocks, uint8_t* __restrict__ q,
                                                                       uint8_t* __restrict__ scales) {
  const long long blk = static_cast<long long>(blockIdx.x) * kQuantThreads + threadIdx.x;
  if (blk >= n_blocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + blk * 32);
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = src[i];
  const uint32_t* w = reinterpret_cast<const uint32_t*>(v);
  uint32_t amax_bits = 0;   // |x| as fp32 bits: the largest is the largest magnitude
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    amax_bits = max(amax_bits, (w[i] << 16) & 0x7fffffffu);
    amax_bits = max(amax_bits, w[i] & 0x7fff0000u);
  }
  const int exp_field = static_cast<int>(amax_bits >> 23);
  const int e = exp_field == 0 ? -127 : max(exp_field - 127 - 8, -127);   // floor(log2 amax) - 8, clamped
  const float inv = __int_as_float((127 - e) << 23);                        // 2^-e, exact (e >= -127)
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float f0 = __uint_as_float(w[2 * i] << 16) * inv, f1 = __uint_as_float(w[2 * i] & 0xffff0000u) * inv;
    const float f2 = __uint_as_float(w[2 * i + 1] << 16) * inv, f3 = __uint_as_float(w[2 * i + 1] & 0xffff0000u) * inv;
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(f1), "f"(f0));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(f3), "f"(f2));
    out[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(q + blk * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  scales[blk] = static_cast<uint8_t>(e + 127);
}

}  // namespace

int run_quantize_mxfp8(const void* x, long long rows, int cols, void* q, void* scales, cudaStream_t stream) {
  const long long n_blocks = rows * (cols / 32);
  if (n_blocks == 0) return MSA_OK;
  const long long grid = (n_blocks + kQuantThreads - 1) / kQuantThreads;
  quantize_mxfp8_kernel<<<static_cast<unsigned>(grid), kQuantThreads, 0, stream>>>(
      static_cast<const uint16_t*>(x), n_blocks, static_cast<uint8_t*>(q), static_cast<uint8_t*>(scales));
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

}  // namespace msa

extern "C" MSA_API int msa_quantize_mxfp8(const void* x, long long rows, int cols, void* q, void* scales,
                                          void* stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return MSA_ERR_INVALID;
  if (rows > (1ll << 40) / cols) return MSA_ERR_UNSUPPORTED;
  if (rows > 0 && (!x || !q || !scales)) return MSA_ERR_INVALID;
  if (rows > 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q)) & 15u) != 0)
    return MSA_ERR_MISALIGNED;
  return msa::run_quantize_mxfp8(x, rows, cols, q, scales, static_cast<cudaStream_t>(stream));
}
