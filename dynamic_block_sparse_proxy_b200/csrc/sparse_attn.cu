// sparse_attn.cu — block-sparse causal attention on tcgen05 (CRISP paper §2: attention
// restricted to an index set, softmax(QK^T/sqrt(d) + M_S) V; the CRISP summary's final step,
// sparse_attention(Q, K, V, S)).
//
// One CTA computes one 128-row query block of one q-head against the key blocks of its list:
//   warp 0      TMA producer: the Q tile once, then K and V blocks chosen by the list through
//               a 2-stage ring (128-byte swizzle, two 64-column boxes per 128x128 tile);
//   warp 1      one thread issues the UMMAs: S_b = Q K^T into one of two TMEM buffers, then
//               O += P V once the softmax warps published P; commits release the ring slots;
//   warps 2-5   one query row per thread: read S from TMEM, mask the diagonal block (key j is
//               visible to query i iff j <= i), online softmax in the exp2 domain with a lazy
//               maximum (O and the row sum are rescaled only when the maximum grows by more
//               than 2^8), write bf16 P into swizzled shared memory for the PV UMMA; at the end
//               scale O by 1/l and store bf16 O and the natural-log LSE.
// GQA: q-head h reads kv-head h / (h_q / h_kv).
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

constexpr int NS = 2;
constexpr int THREADS = 192;
constexpr uint32_t TILE_BYTES = kB * kD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr float kLazyRescale = 8.0f;   // log2 units
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(1024) AttnSmem {
  __nv_bfloat16 q[kB * kD];
  __nv_bfloat16 k[NS][kB * kD];
  __nv_bfloat16 v[NS][kB * kD];
  __nv_bfloat16 p[kB * kD];
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS];
  uint64_t v_full[NS], v_empty[NS];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, p_free;
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail(AttnSmem& sm, int* status, int code) {
  record_status(status, code);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

struct List {
  const int32_t* cols;
  int len;
  int qb;
  bool dense;
  __device__ __forceinline__ int at(int i) const {
    if (dense) return i;
    const int kb = __ldg(cols + i);
    return (kb < 0 || kb > qb) ? qb : kb;  // invalid entries are reported and replaced
  }
};

__global__ void __launch_bounds__(THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                       const __grid_constant__ CUtensorMap v_map, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const volatile int* abort = &sm.abort;
  const Shape& s = a.s;
  const int h = blockIdx.x % s.h_q;
  const int qb = s.nb - 1 - (int)(blockIdx.x / s.h_q);
  const int kv = h / s.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  List list;
  list.qb = qb;
  list.dense = a.dense != 0;
  if (list.dense) {
    list.cols = nullptr;
    list.len = qb + 1;
  } else {
    const int32_t* rp = a.row_ptr + (size_t)h * (s.nb + 1);
    const int beg = __ldg(rp + qb);
    list.len = __ldg(rp + qb + 1) - beg;
    list.cols = a.cols + (size_t)h * s.cap + beg;
  }
  const int L = list.len;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 4);
    }
    mbar_init(&sm.p_full, 4);
    mbar_init(&sm.p_free, 1);
    mbar_init(&sm.o_done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if (lane == 0) trace_mark(a.trace, 0, 6, 1, 0);
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
    if (lane == 0) trace_mark(a.trace, 0, 6, 2, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_o = tmem + 256;

  if (L <= 0 || L > qb + 1) {
    // Malformed row: report it and emit nothing for this block.
    if (threadIdx.x == 0) record_status(a.status, CRISP_ERR_DEVICE_CHECK);
  } else if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&q_map);
      tma_prefetch_desc(&k_map);
      tma_prefetch_desc(&v_map);
      const int qrow = h * s.n + qb * kB;
      mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES);
      tma_load_2d(&q_map, &sm.q_full, sm.q, 0, qrow);
      tma_load_2d(&q_map, &sm.q_full, sm.q + kB * 64, 64, qrow);
      int issued = 0;
      for (int i = 0; i < L; ++i) {
        const int st = i % NS;
        const uint32_t par = ((i / NS) & 1) ^ 1;
        trace_mark(a.trace, 0, 0, 1, i);
        if (!list.dense) {
          const int raw = __ldg(list.cols + i);
          if (raw < 0 || raw > qb) record_status(a.status, CRISP_ERR_DEVICE_CHECK);
        }
        const int krow = kv * s.n + list.at(i) * kB;
        if (!mbar_wait(&sm.k_empty[st], par, abort)) { fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT); break; }
        mbar_arrive_expect_tx(&sm.k_full[st], TILE_BYTES);
        tma_load_2d(&k_map, &sm.k_full[st], sm.k[st], 0, krow);
        tma_load_2d(&k_map, &sm.k_full[st], sm.k[st] + kB * 64, 64, krow);
        trace_mark(a.trace, 0, 0, 2, i);
        if (!mbar_wait(&sm.v_empty[st], par, abort)) { fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT); issued = i + 1; break; }
        mbar_arrive_expect_tx(&sm.v_full[st], TILE_BYTES);
        tma_load_2d(&v_map, &sm.v_full[st], sm.v[st], 0, krow);
        tma_load_2d(&v_map, &sm.v_full[st], sm.v[st] + kB * 64, 64, krow);
        issued = i + 1;
      }
      // Never leave with copies in flight (bounded waits on the last use of each slot).
      trace_mark(a.trace, 0, 0, 4, issued);
      mbar_wait(&sm.q_full, 0, nullptr);
      for (int i = max(0, issued - NS); i < issued; ++i) {
        mbar_wait(&sm.k_full[i % NS], (i / NS) & 1, nullptr);
        mbar_wait(&sm.v_full[i % NS], (i / NS) & 1, nullptr);
      }
      trace_mark(a.trace, 0, 0, 5, issued);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      bool ok = mbar_wait(&sm.q_full, 0, abort);
      if (!ok) fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
      const uint32_t qa = smem_u32(sm.q), pa = smem_u32(sm.p);
      for (int i = 0; ok && i <= L; ++i) {
        if (i < L) {
          const int st = i % NS, b = i & 1;
          trace_mark(a.trace, 0, 1, 1, i);
          if (!mbar_wait(&sm.k_full[st], (i / NS) & 1, abort) ||
              !mbar_wait(&sm.s_free[b], ((i >> 1) & 1) ^ 1, abort)) {
            fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
            break;
          }
          tc_fence_after();
          const uint32_t ka = smem_u32(sm.k[st]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            umma_ss(tmem + b * 128, desc_kmajor_sw128(qa + off), desc_kmajor_sw128(ka + off), idesc_qk,
                    kk > 0);
          }
          umma_commit(&sm.s_full[b]);
          umma_commit(&sm.k_empty[st]);
        }
        if (i >= 1) {
          const int j = i - 1, st = j % NS;
          trace_mark(a.trace, 0, 1, 3, j);
          if (!mbar_wait(&sm.p_full, j & 1, abort) || !mbar_wait(&sm.v_full[st], (j / NS) & 1, abort)) {
            fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
            break;
          }
          tc_fence_after();
          const uint32_t va = smem_u32(sm.v[st]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            umma_ss(tmem_o, desc_kmajor_sw128(pa + aoff), desc_mnmajor_sw128(va + kk * 2048, HALF_BYTES),
                    idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&sm.p_free);
          umma_commit(&sm.v_empty[st]);
        }
      }
      trace_mark(a.trace, 0, 1, 6, L);
      umma_commit(&sm.o_done);
      mbar_wait(&sm.o_done, 0, nullptr);
      trace_mark(a.trace, 0, 1, 7, L);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int grp = warp & 3;
    const int r = grp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    const float sc = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    uint8_t* prow = reinterpret_cast<uint8_t*>(sm.p);
    for (int i = 0; i < L; ++i) {
      const int b = i & 1;
      const int kb = list.at(i);
      if (lane == 0) trace_mark(a.trace, 0, 2 + grp, 1, i);
      if (!warp_wait(&sm.s_full[b], (i >> 1) & 1, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + b * 128 + c * 32, v[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free[b]);

      const bool diag = kb == qb;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if (diag && (c * 32 + t) > r) v[c][t] = __float_as_uint(-INFINITY);
          mx = fmaxf(mx, __uint_as_float(v[c][t]));
        }
      mx *= sc;
      float m_new = m;
      bool rescale = false;
      if (mx > m + kLazyRescale || m == -INFINITY) {
        m_new = mx;
        rescale = (m != -INFINITY);
      }
      const float alpha = fast_exp2(m - m_new);  // 0 on the first block (m = -inf)
      l *= alpha;
      float rs = 0.f;
      uint32_t pk[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float e0 = fast_exp2(fmaf(__uint_as_float(v[c][2 * t]), sc, -m_new));
          const float e1 = fast_exp2(fmaf(__uint_as_float(v[c][2 * t + 1]), sc, -m_new));
          rs += e0 + e1;
          pk[c][t] = pack_bf16(e0, e1);
        }
      l += rs;
      m = m_new;

      // PV of the previous block must be complete before P is overwritten or O rescaled.
      if (lane == 0) trace_mark(a.trace, 0, 2 + grp, 2, i);
      if (i >= 1 && !warp_wait(&sm.p_free, (i - 1) & 1, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      // The O update is warp-collective (tcgen05.ld/st): run it on the whole warp when any row
      // needs it; rows that keep their maximum have alpha == 1.
      if (__any_sync(0xffffffffu, rescale)) {
        if (lane == 0) trace_mark(a.trace, 0, 2 + grp, 3, i);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
          tmem_st32(tmem_o + lane_off + c * 32, o);
        }
        tmem_st_wait();
      }
      // P row r: 16 chunks of 8 keys; chunk cc lives in half cc/8 at swizzled slot cc%8.
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const int c = cc >> 2, t0 = (cc & 3) * 4;
        uint4 u = make_uint4(pk[c][t0], pk[c][t0 + 1], pk[c][t0 + 2], pk[c][t0 + 3]);
        *reinterpret_cast<uint4*>(prow + (cc >> 3) * HALF_BYTES + sw128_offset(r, cc & 7)) = u;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.p_full);
        trace_mark(a.trace, 0, 2 + grp, 4, i);
      }
      __syncwarp();
    }
    if (ok) {
      if (lane == 0) trace_mark(a.trace, 0, 2 + grp, 5, L);
      if (!warp_wait(&sm.o_done, 0, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
      } else {
        tc_fence_after();
        const float inv = 1.f / l;
        const size_t row = (size_t)h * s.n + (size_t)qb * kB + r;
        uint4* dst = reinterpret_cast<uint4*>(a.o + row * kD);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            dst[c * 4 + t] = make_uint4(
                pack_bf16(__uint_as_float(o[8 * t + 0]) * inv, __uint_as_float(o[8 * t + 1]) * inv),
                pack_bf16(__uint_as_float(o[8 * t + 2]) * inv, __uint_as_float(o[8 * t + 3]) * inv),
                pack_bf16(__uint_as_float(o[8 * t + 4]) * inv, __uint_as_float(o[8 * t + 5]) * inv),
                pack_bf16(__uint_as_float(o[8 * t + 6]) * inv, __uint_as_float(o[8 * t + 7]) * inv));
          }
        }
        if (a.lse != nullptr) a.lse[row] = (m + __log2f(l)) * kLn2;
        if (lane == 0) trace_mark(a.trace, 0, 2 + grp, 6, L);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (lane == 0) trace_mark(a.trace, 0, 6, 4, 0);
    __syncwarp();
    tmem_dealloc(tmem, 512);
    if (lane == 0) trace_mark(a.trace, 0, 6, 5, 0);
  }
}

}  // namespace

cudaError_t launch_sparse_attn(const CUtensorMap& q_map, const CUtensorMap& k_map, const CUtensorMap& v_map,
                               const AttnArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(AttnSmem) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  sparse_attn_kernel<<<a.s.h_q * a.s.nb, THREADS, smem, st>>>(q_map, k_map, v_map, a);
  return cudaGetLastError();
}

}  // namespace crisp
