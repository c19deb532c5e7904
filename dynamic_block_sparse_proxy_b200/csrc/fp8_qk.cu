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

// One CTA per (head, 128-row block), thread t owns row t of the block (rows past n are skipped).
__global__ void __launch_bounds__(kB) fp8_quant_kernel(const __nv_bfloat16* x, int n, int ld, int nb,
                                                       uint8_t* out, float* scales) {
  const int b = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  const int row = b * kB + t;
  const bool live = row < n;
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)h * ld + (live ? row : 0)) * kD);
  uint4 u[kD / 8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kD / 8; ++i) {
    u[i] = live ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p2[j]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float wmax[kB / 32];
  if ((t & 31) == 0) wmax[t >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  if (t == 0) scales[(size_t)h * nb + b] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  if (!live) return;
  uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)h * n + row) * kD);  // n rows per head
#pragma unroll
  for (int i = 0; i < kD / 16; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // 4 values: bf16 pairs 2j and 2j+1 of the 16 in u[2i], u[2i+1]
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u[2 * i + (j >> 1)]);
      const float2 f0 = __bfloat1622float2(p2[(j & 1) * 2]);
      const float2 f1 = __bfloat1622float2(p2[(j & 1) * 2 + 1]);
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv)),
                                                              __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv)),
                                                              __NV_SATFINITE, __NV_E4M3);
      w[j] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_fp8_quant(const __nv_bfloat16* x, int heads, int n, int ld, uint8_t* out, float* scales,
                             cudaStream_t st) {
  const int nb = (n + kB - 1) / kB;
  fp8_quant_kernel<<<dim3(nb, heads), kB, 0, st>>>(x, n, ld, nb, out, scales);
  return cudaGetLastError();
}

}  // namespace crisp
