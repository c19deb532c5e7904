// proxy_pass.cu — the proxy attention of CRISP reduced on the fly (CRISP paper §2: proxy
// attention A_hat = softmax(Q_hat K^T / sqrt(d)) over a representative query subset, here the
// last query block; §4: vertical = column means, slash = diagonal means, pooled into blocks).
//
// One CTA handles one q-head and a chunk of kProxyChunk key blocks. TMA streams the key blocks
// of the head's kv-head through a 2-stage ring; one thread issues S = Q_last K_blk^T (128x128x128,
// bf16 -> fp32) with tcgen05 into a double-buffered TMEM tile; four softmax warps (one query
// row per thread) read S back, apply the causal mask on the last key block, and accumulate
// exp2(x - m) with a running row maximum m into two sums per key block: keys at or below the
// row's diagonal offset (t <= r) and keys above it (t > r). A key at offset t of block kb seen by
// proxy row r lies on diagonal offset (N_b-1-kb)*B + (r - t), so the first sum belongs to slash
// block N_b-1-kb and the second to N_b-2-kb; their total is the block's vertical mass. The
// normalisation by the row's global max and sum happens in the routing kernel.
//
// A seventh warp (only in the CTA of the first q-head of each GQA group) sums each K block's
// rows into the mean-pooled key K_bar used by the Pooled-Estimation path, so K is read once.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

constexpr int NS = 2;
constexpr int THREADS = 224;
constexpr uint32_t TILE_BYTES = kB * kD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr float kScaleLog2 = 0.12751743074380045f;  // log2(e) / sqrt(128)

struct __align__(1024) ProxySmem {
  __nv_bfloat16 q[kB * kD];       // two 128-byte-swizzled halves [128 rows][64 cols]
  __nv_bfloat16 k[NS][kB * kD];
  uint64_t q_full;
  uint64_t k_full[NS];
  uint64_t k_empty[NS];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail(ProxySmem& sm, int* status) {
  record_status(status, CRISP_ERR_DEVICE_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

__global__ void __launch_bounds__(THREADS, 2)
    proxy_pass_kernel(const __grid_constant__ CUtensorMap q_map,
                      const __grid_constant__ CUtensorMap k_map, const SelectArgs a) {
  extern __shared__ uint8_t smem_raw[];
  ProxySmem& sm = *reinterpret_cast<ProxySmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const volatile int* abort = &sm.abort;

  const Shape& s = a.s;
  const int h = blockIdx.x % s.h_q;
  const int chunk = blockIdx.x / s.h_q;
  const int kv = h / s.G;
  const int kb0 = chunk * kProxyChunk;
  const int nblk = min(kProxyChunk, s.nb - kb0);
  const bool pool = (h % s.G) == 0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], pool ? 2 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 4);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&q_map);
      tma_prefetch_desc(&k_map);
      const int qrow = h * s.n + s.n - kB;
      mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES);
      tma_load_2d(&q_map, &sm.q_full, sm.q, 0, qrow);
      tma_load_2d(&q_map, &sm.q_full, sm.q + kB * 64, 64, qrow);
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int st = j % NS;
        if (!mbar_wait(&sm.k_empty[st], ((j / NS) & 1) ^ 1, abort)) {
          fail(sm, a.status);
          break;
        }
        const int krow = kv * s.n + (kb0 + j) * kB;
        mbar_arrive_expect_tx(&sm.k_full[st], TILE_BYTES);
        tma_load_2d(&k_map, &sm.k_full[st], sm.k[st], 0, krow);
        tma_load_2d(&k_map, &sm.k_full[st], sm.k[st] + kB * 64, 64, krow);
        ++issued;
      }
      // Never leave with copies in flight: wait (bounded) for the last load of each stage.
      mbar_wait(&sm.q_full, 0, nullptr);
      for (int j = max(0, issued - NS); j < issued; ++j) mbar_wait(&sm.k_full[j % NS], (j / NS) & 1, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      bool ok = mbar_wait(&sm.q_full, 0, abort);
      if (!ok) fail(sm, a.status);
      for (int j = 0; ok && j < nblk; ++j) {
        const int st = j % NS, b = j & 1;
        if (!mbar_wait(&sm.k_full[st], (j / NS) & 1, abort) ||
            !mbar_wait(&sm.s_free[b], ((j >> 1) & 1) ^ 1, abort)) {
          fail(sm, a.status);
          break;
        }
        tc_fence_after();
        const uint32_t qa = smem_u32(sm.q), ka = smem_u32(sm.k[st]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          umma_ss(tmem + b * 128, desc_kmajor_sw128(qa + off), desc_kmajor_sw128(ka + off), idesc,
                  kk > 0);
        }
        umma_commit(&sm.s_full[b]);
        umma_commit(&sm.k_empty[st]);
      }
      // Never release TMEM under a running MMA: wait (bounded) for all issued work.
      umma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0, nullptr);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ softmax rows
    const int grp = warp & 3;
    const int r = grp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    float m = -INFINITY;
    float plo[kProxyChunk], phi[kProxyChunk];
#pragma unroll
    for (int jj = 0; jj < kProxyChunk; ++jj) plo[jj] = phi[jj] = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      if (!warp_wait(&sm.s_full[b], (j >> 1) & 1, abort)) {
        fail(sm, a.status);
        ok = false;
        break;
      }
      tc_fence_after();
      const bool last = (kb0 + j) == s.nb - 1;
      float lo = 0.f, hi = 0.f;
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + b * 128 + sl * 32, v);
        tmem_ld_wait();
        if (sl == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_free[b]);
        }
        float x[32];
        float xm = -INFINITY;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          x[t] = __uint_as_float(v[t]);
          if (last && (sl * 32 + t) > r) x[t] = -INFINITY;
          xm = fmaxf(xm, x[t]);
        }
        xm *= kScaleLog2;
        if (xm > m) {
          const float f = fast_exp2(m - xm);
#pragma unroll
          for (int jj = 0; jj < kProxyChunk; ++jj) {
            plo[jj] *= f;
            phi[jj] *= f;
          }
          lo *= f;
          hi *= f;
          m = xm;
        }
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float e = fast_exp2(fmaf(x[t], kScaleLog2, -m));
          if (sl * 32 + t <= r) lo += e; else hi += e;
        }
      }
#pragma unroll
      for (int jj = 0; jj < kProxyChunk; ++jj)
        if (jj == j) {
          plo[jj] = lo;
          phi[jj] = hi;
        }
    }
    if (ok) {
      float tot = 0.f;
#pragma unroll
      for (int jj = 0; jj < kProxyChunk; ++jj) {
        if (jj < nblk) {
          a.part[((size_t)h * s.nb + kb0 + jj) * kB + r] = make_float2(plo[jj], phi[jj]);
          tot += plo[jj] + phi[jj];
        }
      }
      const size_t ci = ((size_t)h * s.n_chunks + chunk) * kB + r;
      a.chunk_max[ci] = m;
      a.chunk_tot[ci] = tot;
    }
  } else if (pool) {
    // ------------------------------------------------------------------ K block mean (PE path)
    const int c16 = lane & 15, half = c16 >> 3, ch = c16 & 7, rp = lane >> 4;
    for (int j = 0; j < nblk; ++j) {
      const int st = j % NS;
      if (!warp_wait(&sm.k_full[st], (j / NS) & 1, abort)) {
        fail(sm, a.status);
        break;
      }
      const uint8_t* base = reinterpret_cast<const uint8_t*>(sm.k[st]) + half * HALF_BYTES;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
      for (int rr = 0; rr < 64; ++rr) {
        const int row = 2 * rr + rp;
        const uint4 u = *reinterpret_cast<const uint4*>(base + sw128_offset(row, ch));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(p2[i]);
          acc[2 * i] += f.x;
          acc[2 * i + 1] += f.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
      if (lane < 16) {
        float4* dst = reinterpret_cast<float4*>(a.kbar + ((size_t)kv * s.nb + kb0 + j) * kD + c16 * 8);
        const float inv = 1.f / kB;
        dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.k_empty[st]);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_proxy_pass(const CUtensorMap& q_map, const CUtensorMap& k_map, const SelectArgs& a,
                              cudaStream_t st) {
  const size_t smem = sizeof(ProxySmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(proxy_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.s.h_q * a.s.n_chunks);
  proxy_pass_kernel<<<grid, THREADS, smem, st>>>(q_map, k_map, a);
  return cudaGetLastError();
}

}  // namespace crisp
