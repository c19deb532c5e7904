// fp8_qk.cu — Q and K in 8-bit E4M3 for the FP8 variant of the attention logits (the attention
// of crisp_sparse_prefill_fp8qk computes S = Q K^T on E4M3 operands; P, V and O stay as in the
// bf16 kernel). The format is the OCP 8-bit floating point E4M3 (bias 7, 3 mantissa bits, no
// infinities, largest finite value 448).
//
// Per head and 128-row block: amax = max |x| (fp32), inv = 448 / amax and scale = amax / 448,
// both rounded to fp32; each value is stored as E4M3(x * inv), the product rounded to fp32 and
// then to the nearest E4M3 value (ties to even, saturating at 448). An all-zero block gets codes
// 0 and scale 1. The dequantised value is E4M3 * scale; the attention folds the two blocks'
// scales into its logit scale.
#include <cuda_fp8.h>

#include "crisp_internal.h"

namespace crisp {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kChunks = kB * kD / 8;                 // 16-byte chunks of 8 values in a block
constexpr int kPerThread = kChunks / kQuantThreads;  // 8

// One CTA per (head, 128-row block). The block's rows are contiguous (kD values each), so thread
// i takes the 16-byte chunks i, i + 256, ... of the block: every load and every 8-byte code store
// of a warp covers one contiguous span. Chunk c holds row c / 16, values 8 (c % 16) .. +7; rows
// past n are neither read nor stored.
__global__ void __launch_bounds__(kQuantThreads) fp8_quant_kernel(const __nv_bfloat16* x, int n, int ld, int nb,
                                                                  uint8_t* out, float* scales) {
  const int b = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  const int rows = min(kB, n - b * kB);  // rows of this block below n
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)h * ld + (size_t)b * kB) * kD);
  uint4 u[kPerThread];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int c = t + i * kQuantThreads;
    u[i] = c / (kD / 8) < rows ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p2[j]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float wmax[kQuantThreads / 32];
  if ((t & 31) == 0) wmax[t >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, wmax[w]);
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  if (t == 0) scales[(size_t)h * nb + b] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const uint32_t keep = amax > 0.f ? 0xffffffffu : 0u;  // an all-zero block (signed zeros too): codes 0
  uint2* dst = reinterpret_cast<uint2*>(out + ((size_t)h * n + (size_t)b * kB) * kD);  // n rows per head
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int c = t + i * kQuantThreads;
    if (c / (kD / 8) >= rows) continue;
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u[i]);
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 f0 = __bfloat1622float2(p2[2 * j]);
      const float2 f1 = __bfloat1622float2(p2[2 * j + 1]);
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv)),
                                                              __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv)),
                                                              __NV_SATFINITE, __NV_E4M3);
      w[j] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    dst[c] = make_uint2(w[0] & keep, w[1] & keep);
  }
}

}  // namespace

cudaError_t launch_fp8_quant(const __nv_bfloat16* x, int heads, int n, int ld, uint8_t* out, float* scales,
                             cudaStream_t st) {
  const int nb = (n + kB - 1) / kB;
  fp8_quant_kernel<<<dim3(nb, heads), kQuantThreads, 0, st>>>(x, n, ld, nb, out, scales);
  return cudaGetLastError();
}

}  // namespace crisp
