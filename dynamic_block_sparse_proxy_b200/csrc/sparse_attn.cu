// sparse_attn.cu — block-sparse causal attention on tcgen05 (CRISP paper §2: attention
// restricted to an index set, softmax(QK^T/sqrt(d) + M_S) V; the CRISP summary's final step,
// sparse_attention(Q, K, V, S)).
//
// One CTA computes two "tiles", each a 128-row query block of one q-head: the same query block
// of two q-heads of a GQA group that were routed alike, or two adjacent query blocks of one
// head. Both tiles read the same kv-head, so one K/V stream serves both. The CTA
// walks the union of the two tiles' key-block lists in ascending order; a tile takes part in a
// step only if the block is in its own list.
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1 (one query row per thread):
//               read S from TMEM, mask the diagonal block (key j visible to query i iff j <= i),
//               online softmax in the exp2 domain against a lagging row reference (O and the
//               row sum are rescaled only when a block's exponentials would leave [0, 2^64]),
//               write bf16 P back into the tile's S columns; at the end scale O by 1/l, store
//               bf16 O and the LSE;
//   warp 8      TMA producer of both Q tiles once, then the K blocks of the union through a
//               2-stage ring (128-byte swizzle, two 64-column boxes per 128x128 tile);
//   warp 11     TMA producer of the V blocks through a 3-stage ring (a V block is consumed a
//               step after its K block, so it gets the deeper ring);
//   warps 9-10  one thread per tile issues that tile's UMMAs: O_t += P_t V of the previous step
//               (A operand read from TMEM), then S_t = Q_t K^T of this step; the two tiles run
//               out of phase, so the tensor core works on one while the other's softmax runs.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P_t is packed bf16 over S_t.
// Q, K and V are read through per-head 3D tensor maps: when n is not a multiple of 128 the last
// block's rows past n arrive as zeros; the causal mask already hides keys past n from every
// real query (key j <= query i < n), and output rows past n are not stored.
// tcgen05 MMAs issued by one thread execute in order, so S_t is overwritten only after the PV
// that read P_t from the same columns, and the commit that signals S_t also covers that PV.
// Both tiles' MMAs run on the same tensor core, interleaved as their issuers go.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

constexpr int NSK = 2;  // K ring depth
constexpr int NSV = 3;  // V ring depth (V is consumed a step after K)
constexpr int THREADS = 384;
constexpr int PRODUCER_WARP = 8;     // Q and K
constexpr int V_PRODUCER_WARP = 11;  // V
constexpr int MMA_WARP = 9;  // and 10: one issuing warp per tile
constexpr uint32_t TILE_BYTES = kB * kD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(1024) AttnSmem {
  __nv_bfloat16 q[2][kB * kD];
  __nv_bfloat16 k[NSK][kB * kD];
  __nv_bfloat16 v[NSV][kB * kD];
  uint64_t q_full;
  uint64_t k_full[NSK], k_empty[NSK];
  uint64_t v_full[NSV], v_empty[NSV];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done[2];
  uint64_t turn[2][4];  // softmax turn handoff between the tiles, per sub-partition
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
};

// Ascending merge of the two tiles' lists; mask bit t says whether tile t takes part. Each
// list's next entry is loaded one step ahead, so its latency hides behind the step. An entry
// outside [0, qb] or not above its predecessor sets `bad` (the producer reports it) and an
// out-of-range one is replaced by qb, so every walker stays in bounds and ends after at most
// len0 + len1 steps; all walkers see the same sequence.
struct UnionWalk {
  TileList l[2];
  int pos[2], head[2], last[2];
  bool dense, bad;
  int qb[2];
  __device__ __forceinline__ UnionWalk(const TileList (&tl)[2], bool dense_, const int (&qb_)[2])
      : dense(dense_), bad(false) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      l[t] = tl[t];
      qb[t] = qb_[t];
      pos[t] = 0;
      last[t] = -1;
      head[t] = load(t, 0);
    }
  }
  __device__ __forceinline__ int load(int t, int i) const {
    if (i >= l[t].len) return 0x7fffffff;
    return dense ? i : __ldg(l[t].cols + i);
  }
  __device__ __forceinline__ bool next(int& kb, int& mask) {
    int h[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      h[t] = head[t];
      if (h[t] != 0x7fffffff) {
        if (h[t] < 0 || h[t] > qb[t] || h[t] <= last[t]) bad = true;
        if (h[t] < 0 || h[t] > qb[t]) h[t] = qb[t];
      }
    }
    if (h[0] == 0x7fffffff && h[1] == 0x7fffffff) return false;
    kb = min(h[0], h[1]);
    mask = (h[0] == kb ? 1 : 0) | (h[1] == kb ? 2 : 0);
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if ((mask >> t) & 1) {
        last[t] = head[t];
        head[t] = load(t, ++pos[t]);
      }
    return true;
  }
};

// F8: Q and K arrive as E4M3 tiles (one 128x128-byte box each) and S = Q K^T runs as kind::f8f6f4
// MMAs; the logit scale of a step folds in the two blocks' dequantisation scales.
template <bool F8>
__global__ void __launch_bounds__(THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                       const __grid_constant__ CUtensorMap v_map, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const volatile int* abort = &sm.abort;
  const Shape& s = a.s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: two tiles (q-head, query block) that read the same kv-head. kv-heads run one
  // after another and, within one, the longest rows first: the CTAs resident at a time stream
  // the same kv-head's K and V, which then stay in L2 instead of all heads competing for it.
  // Per kv-head the query blocks go in rows of two (qa = nb-1-2i, qa-1), G CTAs per row. The
  // group's heads are taken Vertical-Slash first, then Pooled-Estimation (by `route`, when
  // given), each in ascending order; consecutive heads of one class form a pair that gets two
  // CTAs (one per query block), and a class's leftover head gets one CTA holding both of its
  // query blocks. Heads of one class select alike, so a CTA's two lists overlap and most steps
  // feed both tiles; either way the G heads fill exactly G slots per row.
  const int per_kv = s.G * ((s.nb + 1) / 2);
  const int kv = (int)(blockIdx.x / per_kv);
  const int rem = (int)(blockIdx.x % per_kv);
  const int row_i = rem / s.G, slot = rem % s.G;
  const int qa = s.nb - 1 - 2 * row_i;  // qa - 1 is -1 past the first query block
  int tile_h[2] = {0, 0}, tile_qb[2] = {qa, qa}, ntiles = 0;
  {
    int next_slot = 0, pending = -1;
    bool found = false;
    for (int cls = 1; cls >= 0 && !found; --cls) {
      for (int x = 0; x < s.G && !found; ++x) {
        const int h = kv * s.G + x;
        const int c = a.route != nullptr ? (__ldg(a.route + h) != 0 ? 1 : 0) : 1;
        if (c != cls) continue;
        if (pending < 0) {
          pending = h;
          continue;
        }
        if (slot == next_slot || slot == next_slot + 1) {  // head pair, one query block each
          tile_h[0] = pending;
          tile_h[1] = h;
          tile_qb[0] = tile_qb[1] = qa - (slot - next_slot);
          ntiles = tile_qb[0] >= 0 ? 2 : 0;
          found = true;
        }
        next_slot += 2;
        pending = -1;
      }
      if (!found && pending >= 0) {
        if (slot == next_slot) {  // leftover head: two adjacent query blocks of it
          tile_h[0] = tile_h[1] = pending;
          tile_qb[0] = qa;
          tile_qb[1] = qa - 1;
          ntiles = qa - 1 >= 0 ? 2 : 1;
          found = true;
        }
        next_slot += 1;
        pending = -1;
      }
    }
  }
  if (ntiles == 0) return;  // the unpaired half-row when nb is odd: no work
  if (ntiles == 1) tile_qb[1] = tile_qb[0];
  const bool dense = a.dense != 0;

  TileList tl[2];
  bool bad = false;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qb = tile_qb[t];  // t is a compile-time index here (unrolled)
    if (t >= ntiles) {
      tl[t].cols = nullptr;
      tl[t].len = 0;
    } else if (dense) {
      tl[t].cols = nullptr;
      tl[t].len = qb + 1;
    } else {
      const int h = tile_h[t];
      const int32_t* rp = a.row_ptr + (size_t)h * (s.nb + 1);
      const int beg = __ldg(rp + qb);
      tl[t].len = __ldg(rp + qb + 1) - beg;
      tl[t].cols = a.cols + (size_t)h * s.cap + beg;
      bad |= tl[t].len <= 0 || tl[t].len > qb + 1 || beg < 0 || (long long)beg + tl[t].len > s.cap;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < NSK; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], ntiles);  // one release per tile
    }
    for (int i = 0; i < NSV; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], ntiles);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], 4);
    }
    mbar_init(&sm.o_done[0], 1);
    mbar_init(&sm.o_done[1], 1);
    for (int t = 0; t < 2; ++t)
      for (int g = 0; g < 4; ++g) mbar_init(&sm.turn[t][g], 1);
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
    // ------------------------------------------------------------------ TMA producer: Q, K
    if (lane == 0) {
      tma_prefetch_desc(&q_map);
      tma_prefetch_desc(&k_map);
      mbar_arrive_expect_tx(&sm.q_full, (F8 ? HALF_BYTES : TILE_BYTES) * ntiles);
      for (int t = 0; t < ntiles; ++t) {
        const int qh = t ? tile_h[1] : tile_h[0], qy = (t ? tile_qb[1] : tile_qb[0]) * kB;
        tma_load_3d(&q_map, &sm.q_full, sm.q[t], 0, qy, qh);
        if (!F8) tma_load_3d(&q_map, &sm.q_full, sm.q[t] + kB * 64, 64, qy, qh);
      }
      UnionWalk u(tl, dense, tile_qb);
      int kb, mask, nk = 0;
      for (int step = 0; u.next(kb, mask); ++step) {
        const int st = step % NSK;
        const uint32_t par = ((step / NSK) & 1) ^ 1;
        const int ky = kb * kB;
        trace_mark(a.trace, 0, 0, 1, step);
        if (!mbar_wait(&sm.k_empty[st], par, abort)) { fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT); break; }
        mbar_arrive_expect_tx(&sm.k_full[st], F8 ? HALF_BYTES : TILE_BYTES);
        tma_load_3d(&k_map, &sm.k_full[st], sm.k[st], 0, ky, kv);
        if (!F8) tma_load_3d(&k_map, &sm.k_full[st], sm.k[st] + kB * 64, 64, ky, kv);
        nk = step + 1;
      }
      if (u.bad) record_status(a.status, CRISP_ERR_DEVICE_CHECK);
      // Never leave with copies in flight (bounded waits on the last use of each slot).
      trace_mark(a.trace, 0, 0, 4, 0);
      mbar_wait(&sm.q_full, 0, nullptr);
      for (int i = max(0, nk - NSK); i < nk; ++i) mbar_wait(&sm.k_full[i % NSK], (i / NSK) & 1, nullptr);
      trace_mark(a.trace, 0, 0, 5, 0);
    }
    __syncwarp();
  } else if (warp == V_PRODUCER_WARP) {
    // ------------------------------------------------------------------ TMA producer: V
    // Its own thread, so a V slot that is released late never holds back the next K load.
    if (lane == 0) {
      tma_prefetch_desc(&v_map);
      UnionWalk u(tl, dense, tile_qb);
      int kb, mask, nv = 0;
      for (int step = 0; u.next(kb, mask); ++step) {
        const int st = step % NSV;
        const uint32_t par = ((step / NSV) & 1) ^ 1;
        const int ky = kb * kB;
        trace_mark(a.trace, 0, 5, 2, step);
        if (!mbar_wait(&sm.v_empty[st], par, abort)) { fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT); break; }
        mbar_arrive_expect_tx(&sm.v_full[st], TILE_BYTES);
        tma_load_3d(&v_map, &sm.v_full[st], sm.v[st], 0, ky, kv);
        tma_load_3d(&v_map, &sm.v_full[st], sm.v[st] + kB * 64, 64, ky, kv);
        nv = step + 1;
      }
      for (int i = max(0, nv - NSV); i < nv; ++i) mbar_wait(&sm.v_full[i % NSV], (i / NSV) & 1, nullptr);
      trace_mark(a.trace, 0, 5, 5, 0);
    }
    __syncwarp();
  } else if (warp >= MMA_WARP && warp - MMA_WARP < ntiles) {
    // ------------------------------------------------------------------ MMA issuer of tile t
    // Each tile has its own issuing thread, so a tile's PV and next QK go out as soon as its own
    // P is ready instead of waiting for the other tile's turn. K and V slots are released by
    // both issuers: with a commit after the tile's MMAs that read the slot, or with a plain
    // arrive for a block the tile skips (after the slot's fill completed, so an arrive never
    // counts towards an earlier use of the slot).
    const int t = warp - MMA_WARP;
    const int role = t ? 4 : 1;
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      const uint32_t bit = 1u << t;
      const uint32_t s_tmem = tmem + t * 128;
      const uint32_t o_tmem = tmem + 256 + t * 128;
      const uint32_t qa = smem_u32(sm.q[t]);
      bool ok = mbar_wait(&sm.q_full, 0, abort);
      if (!ok) fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
      UnionWalk u(tl, dense, tile_qb);
      int pv_n = 0;  // PV of this tile issued so far
      int prev_mask = 0, kb = 0, mask = 0, step = 0;
      while (ok) {
        const bool more = u.next(kb, mask);
        if (!more) mask = 0;
        const int st = step % NSK;
        const int prev_vs = (step + NSV - 1) % NSV;
        if (step > 0) {
          // V of the previous step: O_t += P_t V (P_t sits in the S_t columns), or skip it. V is
          // waited for first (it is normally in long before P), so the MMAs go out as soon as P is.
          trace_mark(a.trace, 0, role, 3, step);
          const bool use = (prev_mask & bit) != 0;
          if (!mbar_wait(&sm.v_full[prev_vs], ((step - 1) / NSV) & 1, abort) ||
              (use && !mbar_wait(&sm.p_full[t], pv_n & 1, abort))) {
            fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
            break;
          }
          if (use) {
            tc_fence_after();
            const uint32_t va = smem_u32(sm.v[prev_vs]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(o_tmem, s_tmem + kk * 8, desc_mnmajor_sw128(va + kk * 2048, HALF_BYTES), idesc_pv,
                      (pv_n > 0 || kk > 0) ? 1u : 0u);
            ++pv_n;
            umma_commit(&sm.v_empty[prev_vs]);
          } else {
            mbar_arrive(&sm.v_empty[prev_vs]);
          }
        }
        if (!more) break;
        // K of this step: S_t = Q_t K^T, or skip it
        trace_mark(a.trace, 0, role, 1, step);
        if (!mbar_wait(&sm.k_full[st], (step / NSK) & 1, abort)) {
          fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
          break;
        }
        if (mask & bit) {
          tc_fence_after();
          const uint32_t ka = smem_u32(sm.k[st]);
          if (F8) {
            // E4M3 rows of 128 bytes: four MMAs of K = 32
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss_f8(s_tmem, desc_kmajor_sw128(qa + kk * 32), desc_kmajor_sw128(ka + kk * 32),
                         idesc_e4m3_f32(128, 128), kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
              umma_ss(s_tmem, desc_kmajor_sw128(qa + off), desc_kmajor_sw128(ka + off), idesc_qk, kk > 0);
            }
          }
          umma_commit(&sm.s_full[t]);
          umma_commit(&sm.k_empty[st]);
        } else {
          mbar_arrive(&sm.k_empty[st]);
        }
        prev_mask = mask;
        ++step;
      }
      trace_mark(a.trace, 0, role, 6, step);
      // Never release TMEM under a running MMA: the epilogue and teardown wait for this.
      umma_commit(&sm.o_done[t]);
      mbar_wait(&sm.o_done[t], 0, nullptr);
      trace_mark(a.trace, 0, role, 7, step);
    }
    __syncwarp();
  } else if (warp < 4 * ntiles) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int my_qb = t ? tile_qb[1] : tile_qb[0];
    const int my_h = t ? tile_h[1] : tile_h[0];
    const int grp = warp & 3;
    const int r = grp * 32 + lane;
    const int role = 2 + t;                     // traced by the first warp of each tile
    const bool tracer = grp == 0 && lane == 0;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    const uint32_t s_tmem = tmem + t * 128 + lane_off;
    const uint32_t o_tmem = tmem + 256 + t * 128 + lane_off;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // Warp grp of tile 0 and warp grp of tile 1 share a sub-partition and its exp2 unit; they
    // take turns over the exponentials of each step of the union walk (tile 0 first), so the
    // two tiles stay half a cycle apart and one tile's MMAs run during the other's softmax.
    const bool turns = ntiles == 2;
    uint64_t* my_turn = &sm.turn[t][grp];
    uint64_t* next_turn = &sm.turn[t ^ 1][grp];
    UnionWalk u(tl, dense, tile_qb);
    int kb = 0, mask = 0, i = 0;
    for (int j = 0; u.next(kb, mask); ++j) {
      const bool mine = (mask >> t) & 1;
      const uint32_t turn_parity = (uint32_t)(j & 1) ^ (t == 0 ? 1u : 0u);
      if (!mine) {
        if (turns && !warp_wait(my_turn, turn_parity, abort)) {
          fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
          ok = false;
          break;
        }
        if (turns && lane == 0) mbar_arrive(next_turn);
        continue;
      }
      if (tracer) trace_mark(a.trace, 0, role, 1, i);
      if (!warp_wait(&sm.s_full[t], i & 1, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      // the logit scale of this block (E4M3 logits: times both blocks' dequantisation scales)
      const float sc = F8 ? a.scale_log2 * __ldg(a.qs + (size_t)my_h * s.nb + my_qb) * __ldg(a.ks + (size_t)kv * s.nb + kb)
                          : a.scale_log2;
      // Exponentials use the row reference m of the earlier blocks without looking for this
      // block's maximum: fp32 (and bf16) share fp32's exponent range, so exp2(x*sc - m) stays
      // exact as long as it does not overflow. The first block sets m from its maximum; a later
      // block whose exponentials sum beyond 2^64 (or overflow) is redone against its maximum,
      // with O and l rescaled. The result is the same softmax either way.
      uint32_t v[4][32];
      bool need_max = (i == 0), turn_ok = true;
      float rs = 0.f, alpha = 1.f;
      for (int attempt = 0; attempt < 2; ++attempt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_tmem + c * 32, v[c]);
        tmem_ld_wait();
        // the turn is taken once S is in registers
        if (attempt == 0 && turns && !warp_wait(my_turn, turn_parity, abort)) {
          turn_ok = false;
          break;
        }
        if (kb == my_qb) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (c * 32 + jj > r) v[c][jj] = __float_as_uint(-INFINITY);
        }
        if (need_max) {
          float mx8[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) mx8[jj] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) mx8[jj & 7] = fmaxf(mx8[jj & 7], __uint_as_float(v[c][jj]));
          const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * sc;
          const float m_new = fmaxf(m, mx);
          alpha = fast_exp2(m - m_new);  // 0 on the first block (m = -inf)
          m = m_new;
        }
        const float nm = -m;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const float e0 = fast_exp2(fmaf(__uint_as_float(v[c][2 * jj]), sc, nm));
            const float e1 = fast_exp2(fmaf(__uint_as_float(v[c][2 * jj + 1]), sc, nm));
            acc[jj & 3] += e0 + e1;
            v[c][jj] = pack_bf16(e0, e1);  // pair jj overwrites register jj, already read
          }
        rs = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        const bool redo = !need_max && !(rs <= 18446744073709551616.0f);  // 2^64, or inf / nan
        if (!__any_sync(0xffffffffu, redo)) break;
        need_max = true;
      }
      if (!turn_ok) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
        ok = false;
        break;
      }
      if (turns && lane == 0) mbar_arrive(next_turn);
      // After a redo the accumulator follows the new reference: O and l scale by alpha. The O
      // update is warp-collective; the PV of the previous step completed before S_t was
      // signalled. The first block's PV starts O afresh.
      if (i > 0 && need_max) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tmem + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) o[jj] = __float_as_uint(__uint_as_float(o[jj]) * alpha);
          tmem_st32(o_tmem + c * 32, o);
        }
      }
      l = l * alpha;
      // P: keys 32c..32c+31 -> packed columns 16c..16c+15 of S_t (S was read before)
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st16(s_tmem + c * 16, v[c]);
      l += rs;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[t]);
      if (tracer) trace_mark(a.trace, 0, role, 4, i);
      __syncwarp();
      ++i;
    }
    const int L = i;
    if (ok) {
      if (tracer) trace_mark(a.trace, 0, role, 5, L);
      if (!warp_wait(&sm.o_done[t], 0, abort)) {
        fail(sm, a.status, CRISP_ERR_DEVICE_TIMEOUT);
      } else {
        tc_fence_after();
        const float inv = 1.f / l;
        const size_t row = (size_t)my_h * s.ld + (size_t)my_qb * kB + r;
        const bool real = my_qb * kB + r < s.n;  // rows past n of a partial last block are not stored
        uint4* dst = reinterpret_cast<uint4*>(a.o + row * kD);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tmem + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (real)
              dst[c * 4 + j] = make_uint4(
                pack_bf16(__uint_as_float(o[8 * j + 0]) * inv, __uint_as_float(o[8 * j + 1]) * inv),
                pack_bf16(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv),
                pack_bf16(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv),
                pack_bf16(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv));
          }
        }
        if (a.lse != nullptr && real) a.lse[row] = (m + __log2f(l)) * kLn2;
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
  const bool f8 = a.qs != nullptr;
  auto kernel = f8 ? sparse_attn_kernel<true> : sparse_attn_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.s.h_q * ((a.s.nb + 1) / 2);
  kernel<<<grid, THREADS, smem, st>>>(q_map, k_map, v_map, a);
  return cudaGetLastError();
}

}  // namespace crisp
