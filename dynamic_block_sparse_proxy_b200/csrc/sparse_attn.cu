// sparse_attn.cu — block-sparse causal attention on tcgen05 (CRISP paper §2: attention
// restricted to an index set, softmax(QK^T/sqrt(d) + M_S) V; the CRISP summary's final step,
// sparse_attention(Q, K, V, S)).
//
// One CTA computes one 128-row query block qb for two q-heads of the same GQA group (two
// "tiles"); both read the same kv-head, so one K/V stream serves both. The CTA walks the union
// of the two heads' key-block lists in ascending order; a tile takes part in a step only if the
// block is in its own list.
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1 (one query row per thread):
//               read S from TMEM, mask the diagonal block (key j visible to query i iff j <= i),
//               online softmax in the exp2 domain with a lazy maximum (O and the row sum are
//               rescaled only when the maximum grows by more than 2^8), write bf16 P back into
//               the tile's S columns; at the end scale O by 1/l, store bf16 O and the LSE;
//   warp 8      TMA producer: both Q tiles once, then K and V blocks of the union through a
//               2-stage ring (128-byte swizzle, two 64-column boxes per 128x128 tile);
//   warp 9      one thread issues the UMMAs in ping-pong order: for each tile, O_t += P_t V of
//               the previous step (A operand read from TMEM), then S_t = Q_t K^T of this step,
//               so the tensor core works on one tile while the other tile's softmax runs.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P_t is packed bf16 over S_t.
// tcgen05 MMAs issued by one thread execute in order, so S_t is overwritten only after the PV
// that read P_t from the same columns, and the commit that signals S_t also covers that PV.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

constexpr int NS = 2;
constexpr int THREADS = 320;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr uint32_t TILE_BYTES = kB * kD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr float kLazyRescale = 8.0f;  // log2 units
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(1024) AttnSmem {
  __nv_bfloat16 q[2][kB * kD];
  __nv_bfloat16 k[NS][kB * kD];
  __nv_bfloat16 v[NS][kB * kD];
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS];
  uint64_t v_full[NS], v_empty[NS];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail(AttnSmem& sm, int* status, int code) {
  record_status(status, code);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

// One tile's key-block list: either explicit CSR columns or every block <= qb (dense mode).
struct TileList {
  const int32_t* cols;
  int len;
  __device__ __forceinline__ int at(int i, bool dense, int qb) const {
    if (dense) return i;
    const int kb = __ldg(cols + i);
    return (kb < 0 || kb > qb) ? qb : kb;  // invalid entries are reported and replaced
  }
};

// Ascending merge of the two tiles' lists; mask bit t says whether tile t takes part.
struct UnionWalk {
  TileList l[2];
  int i[2];
  bool dense;
  int qb;
  __device__ __forceinline__ bool next(int& kb, int& mask) {
    const bool h0 = i[0] < l[0].len, h1 = i[1] < l[1].len;
    if (!h0 && !h1) return false;
    const int a = h0 ? l[0].at(i[0], dense, qb) : 0x7fffffff;
    const int b = h1 ? l[1].at(i[1], dense, qb) : 0x7fffffff;
    kb = min(a, b);
    mask = (a == kb ? 1 : 0) | (b == kb ? 2 : 0);
    i[0] += mask & 1;
    i[1] += (mask >> 1) & 1;
    return true;
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
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: (pair of q-heads of one GQA group, query block), longest rows first
  const int pairs_per_group = (s.G + 1) / 2;
  const int n_pairs = s.h_kv * pairs_per_group;
  const int pair = blockIdx.x % n_pairs;
  const int qb = s.nb - 1 - (int)(blockIdx.x / n_pairs);
  const int kv = pair / pairs_per_group;
  const int h0 = kv * s.G + 2 * (pair % pairs_per_group);
  const int ntiles = (2 * (pair % pairs_per_group) + 1 < s.G) ? 2 : 1;
  const bool dense = a.dense != 0;

  TileList tl[2];
  bool bad = false;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (t >= ntiles) {
      tl[t].cols = nullptr;
      tl[t].len = 0;
    } else if (dense) {
      tl[t].cols = nullptr;
      tl[t].len = qb + 1;
    } else {
      const int h = h0 + t;
      const int32_t* rp = a.row_ptr + (size_t)h * (s.nb + 1);
      const int beg = __ldg(rp + qb);
      tl[t].len = __ldg(rp + qb + 1) - beg;
      tl[t].cols = a.cols + (size_t)h * s.cap + beg;
      bad |= tl[t].len <= 0 || tl[t].len > qb + 1;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], 4);
    }
    mbar_init(&sm.o_done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (bad) {
    // Malformed row: report it and emit nothing for this block.
    if (threadIdx.x == 0) record_status(a.status, CRISP_ERR_DEVICE_CHECK);
  } else if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&q_map);
      tma_prefetch_desc(&k_map);
      tma_prefetch_desc(&v_map);
      mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES * ntiles);
      for (int t = 0; t < ntiles; ++t) {
        const int qrow = (h0 + t) * s.n + qb * kB;
        tma_load_2d(&q_map, &sm.q_full, sm.q[t], 0, qrow);
        tma_load_2d(&q_map, &sm.q_full, sm.q[t] + kB * 64, 64, qrow);
      }
      if (!dense) {
        for (int t = 0; t < ntiles; ++t)
          for (int i = 0; i < tl[t].len; ++i) {
            const int raw = __ldg(tl[t].cols + i);
            if (raw < 0 || raw > qb) record_status(a.status, CRISP_ERR_DEVICE_CHECK);
          }
      }
      UnionWalk u{{tl[0], tl[1]}, {0, 0}, dense, qb};
      int kb, mask, nk = 0, nv = 0;
      for (int step = 0; u.next(kb, mask); ++step) {
        const int st = step % NS;
        const uint32_t par = ((step / NS) & 1) ^ 1;
        const int krow = kv * s.n + kb * kB;
        trace_mark(a.trace, 0, 0, 1, step);
        if (!mbar_wait(&sm.k_empty[st], par, abort)) { fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT); break; }
        mbar_arrive_expect_tx(&sm.k_full[st], TILE_BYTES);
        tma_load_2d(&k_map, &sm.k_full[st], sm.k[st], 0, krow);
        tma_load_2d(&k_map, &sm.k_full[st], sm.k[st] + kB * 64, 64, krow);
        nk = step + 1;
        trace_mark(a.trace, 0, 0, 2, step);
        if (!mbar_wait(&sm.v_empty[st], par, abort)) { fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT); break; }
        mbar_arrive_expect_tx(&sm.v_full[st], TILE_BYTES);
        tma_load_2d(&v_map, &sm.v_full[st], sm.v[st], 0, krow);
        tma_load_2d(&v_map, &sm.v_full[st], sm.v[st] + kB * 64, 64, krow);
        nv = step + 1;
      }
      // Never leave with copies in flight (bounded waits on the last use of each slot).
      trace_mark(a.trace, 0, 0, 4, 0);
      mbar_wait(&sm.q_full, 0, nullptr);
      for (int i = max(0, nk - NS); i < nk; ++i) mbar_wait(&sm.k_full[i % NS], (i / NS) & 1, nullptr);
      for (int i = max(0, nv - NS); i < nv; ++i) mbar_wait(&sm.v_full[i % NS], (i / NS) & 1, nullptr);
      trace_mark(a.trace, 0, 0, 5, 0);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      bool ok = mbar_wait(&sm.q_full, 0, abort);
      if (!ok) fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
      UnionWalk u{{tl[0], tl[1]}, {0, 0}, dense, qb};
      int pv_n[2] = {0, 0};  // PV_t issued so far
      int prev_mask = 0, prev_st = 0, kb = 0, mask = 0, step = 0;
      while (ok) {
        const bool more = u.next(kb, mask);
        if (!more) mask = 0;
        const int st = step % NS;
        bool v_ready = false, k_ready = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok) continue;
          if (prev_mask & (1 << t)) {
            // O_t += P_t V of the previous step; P_t sits in the S_t columns
            trace_mark(a.trace, 0, 1, 3, step);
            if (!mbar_wait(&sm.p_full[t], pv_n[t] & 1, abort) ||
                (!v_ready && !mbar_wait(&sm.v_full[prev_st], ((step - 1) / NS) & 1, abort))) {
              fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
              ok = false;
              continue;
            }
            v_ready = true;
            tc_fence_after();
            const uint32_t va = smem_u32(sm.v[prev_st]);
            const uint32_t p_tmem = tmem + t * 128;
            const uint32_t o_tmem = tmem + 256 + t * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(o_tmem, p_tmem + kk * 8, desc_mnmajor_sw128(va + kk * 2048, HALF_BYTES), idesc_pv,
                      (pv_n[t] > 0 || kk > 0) ? 1u : 0u);
            ++pv_n[t];
          }
          if (mask & (1 << t)) {
            // S_t = Q_t K^T of this step
            trace_mark(a.trace, 0, 1, 1, step);
            if (!k_ready && !mbar_wait(&sm.k_full[st], (step / NS) & 1, abort)) {
              fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
              ok = false;
              continue;
            }
            k_ready = true;
            tc_fence_after();
            const uint32_t qa = smem_u32(sm.q[t]), ka = smem_u32(sm.k[st]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
              umma_ss(tmem + t * 128, desc_kmajor_sw128(qa + off), desc_kmajor_sw128(ka + off), idesc_qk,
                      kk > 0);
            }
            umma_commit(&sm.s_full[t]);
          }
        }
        if (!ok) break;
        if (prev_mask) umma_commit(&sm.v_empty[prev_st]);
        if (mask) umma_commit(&sm.k_empty[st]);
        if (!more) break;
        prev_mask = mask;
        prev_st = st;
        ++step;
      }
      trace_mark(a.trace, 0, 1, 6, step);
      // Never release TMEM under a running MMA: the epilogue and teardown wait for this.
      umma_commit(&sm.o_done);
      mbar_wait(&sm.o_done, 0, nullptr);
      trace_mark(a.trace, 0, 1, 7, step);
    }
    __syncwarp();
  } else if (warp < 4 * ntiles) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int grp = warp & 3;
    const int r = grp * 32 + lane;
    const int role = 2 + t;                     // traced by the first warp of each tile
    const bool tracer = grp == 0 && lane == 0;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    const uint32_t s_tmem = tmem + t * 128 + lane_off;
    const uint32_t o_tmem = tmem + 256 + t * 128 + lane_off;
    const float sc = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    const TileList my = t ? tl[1] : tl[0];
    const int L = my.len;
    for (int i = 0; i < L; ++i) {
      const int kb = my.at(i, dense, qb);
      if (tracer) trace_mark(a.trace, 0, role, 1, i);
      if (!warp_wait(&sm.s_full[t], i & 1, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      // S row: all four 32-column loads in flight, one wait (a TMEM round trip is expensive
      // while the tensor core works on the other tile)
      uint32_t v[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_tmem + c * 32, v[c]);
      tmem_ld_wait();
      if (kb == qb) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j > r) v[c][j] = __float_as_uint(-INFINITY);
      }
      // row maximum over eight independent chains
      float mx8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mx8[j] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(v[c][j]));
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mx *= sc;
      float m_new = m;
      bool rescale = false;
      if (mx > m + kLazyRescale || m == -INFINITY) {
        m_new = mx;
        rescale = (m != -INFINITY);
      }
      const float alpha = fast_exp2(m - m_new);  // 0 on the first block (m = -inf), 1 if kept
      // P = exp2(x*sc - m), packed to bf16 pairs in place (pair j of a chunk overwrites register
      // j, already read) and stored over the S columns: keys 32c..32c+31 -> columns 16c..16c+15.
      const float nm = -m_new;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float e0 = fast_exp2(fmaf(__uint_as_float(v[c][2 * j]), sc, nm));
          const float e1 = fast_exp2(fmaf(__uint_as_float(v[c][2 * j + 1]), sc, nm));
          acc[j & 3] += e0 + e1;
          v[c][j] = pack_bf16(e0, e1);
        }
        tmem_st16(s_tmem + c * 16, v[c]);
      }
      // The O update is warp-collective (tcgen05.ld/st): run it on the whole warp when any row
      // needs it. The PV of the previous step completed before S_t was signalled, and the PV of
      // this step waits for p_full below.
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tmem + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(o_tmem + c * 32, o);
        }
      }
      l = l * alpha + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[t]);
      if (tracer) trace_mark(a.trace, 0, role, 4, i);
      __syncwarp();
    }
    if (ok) {
      if (tracer) trace_mark(a.trace, 0, role, 5, L);
      if (!warp_wait(&sm.o_done, 0, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
      } else {
        tc_fence_after();
        const float inv = 1.f / l;
        const int h = h0 + t;
        const size_t row = (size_t)h * s.n + (size_t)qb * kB + r;
        uint4* dst = reinterpret_cast<uint4*>(a.o + row * kD);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tmem + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dst[c * 4 + j] = make_uint4(
                pack_bf16(__uint_as_float(o[8 * j + 0]) * inv, __uint_as_float(o[8 * j + 1]) * inv),
                pack_bf16(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv),
                pack_bf16(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv),
                pack_bf16(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv));
          }
        }
        if (a.lse != nullptr) a.lse[row] = (m + __log2f(l)) * kLn2;
        if (tracer) trace_mark(a.trace, 0, role, 6, L);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_sparse_attn(const CUtensorMap& q_map, const CUtensorMap& k_map, const CUtensorMap& v_map,
                               const AttnArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(AttnSmem) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_pairs = a.s.h_kv * ((a.s.G + 1) / 2);
  sparse_attn_kernel<<<n_pairs * a.s.nb, THREADS, smem, st>>>(q_map, k_map, v_map, a);
  return cudaGetLastError();
}

}  // namespace crisp
