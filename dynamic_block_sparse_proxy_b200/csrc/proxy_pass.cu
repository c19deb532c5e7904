// proxy_pass.cu — the proxy attention of CRISP reduced on the fly (CRISP paper §2: proxy
// attention A_hat = softmax(Q_hat K^T / sqrt(d)) over a representative query subset, here the
// last query block; §4: vertical = column means, slash = diagonal means, pooled into blocks).
//
// Work item: two q-heads of one GQA group (two "tiles": their last query blocks) against a chunk
// of kProxyChunk key blocks of the shared kv-head, so every K block is read once for both. The
// grid is persistent (one CTA per SM): CTA c takes a contiguous run of the items listed pair by
// pair, so a CTA's items mostly share their Q tiles, and the barrier rings run on from one item
// to the next.
//   warp 16     TMA producer: the two Q tiles whenever the pair changes (after the MMAs that read
//               the old ones), then the chunks' K blocks through a 3-stage ring;
//   warp 17     one thread issues S_t = Q_t K_blk^T (128x128x128, bf16 -> fp32) into a
//               double-buffered TMEM tile per head;
//   warps 0-15  softmax: per head 8 warps, two per TMEM lane quarter, each thread one proxy row
//               and one 64-column half of the S block (four exponentiating warps per
//               sub-partition keep the exp2 unit fed): read its columns from TMEM 32 at a time
//               (the next load in flight while the current columns are exponentiated), mask the
//               keys the causal limit cuts (key j visible to row r iff j <= n-B+r), and
//               accumulate exp2(x - m) against a lagging reference m of its own (set by its first
//               block of the chunk, moved only when a block's sum would leave [0, 2^64]) into two
//               sums per key block: keys at or below the row's diagonal offset (t <= r) and above
//               it (t > r). Each (chunk, half) is a segment with its own reference; the sums go
//               straight to global memory and the routing kernel weighs the segments;
//   warps 18-19 sum rows of each K block into the mean-pooled key K_bar of the PE path; the
//               items of one group share the 16 column chunks between them.
// A key at offset t of block kb seen by proxy row r lies on diagonal offset (N_b-1-kb)*B + (r-t),
// so the first sum belongs to slash block N_b-1-kb and the second to N_b-2-kb; their total is
// the block's vertical mass. When n is not a multiple of 128 (t_last keys in the last block) the
// split column is (t_last + r) mod 128, rows with t_last + r < 128 land one slash block lower, and
// each row also sums block N_b-2's part of the last-128-keys window for C_struct; that case runs in
// its own kernel instance. The per-row normalisation happens in the routing kernels.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

constexpr int NS = 3;
constexpr int SOFTMAX_WARPS = 16;
constexpr int PRODUCER_WARP = 16;
constexpr int MMA_WARP = 17;
constexpr int POOL_WARP = 18;   // and 19: two warps share the pooling
constexpr int THREADS = 640;
constexpr uint32_t TILE_BYTES = kB * kD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr float kScaleLog2 = 0.12751743074380045f;  // log2(e) / sqrt(128)

struct __align__(1024) ProxySmem {
  __nv_bfloat16 q[2][kB * kD];  // two 128-byte-swizzled halves [128 rows][64 cols] per tile
  __nv_bfloat16 k[NS][kB * kD];
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t k_full[NS];
  uint64_t k_empty[NS];
  uint64_t s_full[2][2];
  uint64_t s_free[2][2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail(ProxySmem& sm, int* status) {
  record_status(status, CRISP_ERR_DEVICE_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

// tcgen05.wait::ld that also names the destination registers of the load it waits for, so the
// compiler cannot move their first use above the wait.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
        "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
        "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
        "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// Item (pair, chunk) and what follows from it.
struct Item {
  int pair, chunk, kv, pig, h0, ntiles, kb0, nblk;
  __device__ __forceinline__ Item(const Shape& s, int pair_, int chunk_) {
    const int ppg = (s.G + 1) / 2;
    pair = pair_;
    chunk = chunk_;
    kv = pair / ppg;
    pig = pair % ppg;
    h0 = kv * s.G + 2 * pig;
    ntiles = (2 * pig + 1 < s.G) ? 2 : 1;
    kb0 = chunk * kProxyChunk;
    nblk = min(kProxyChunk, s.nb - kb0);
  }
};

// Which items a CTA runs: the items are the (head pair, chunk) pairs listed pair by pair; CTA c
// of P runs the contiguous share [c I / P, (c+1) I / P).
struct Sched {
  int I, P, n_chunks;
  __device__ __forceinline__ Sched(const Shape& s, int P_) {
    n_chunks = s.n_chunks;
    I = s.h_kv * ((s.G + 1) / 2) * n_chunks;
    P = P_;
  }
  __device__ __forceinline__ int count(int c) const {
    return (int)(((long long)(c + 1) * I) / P - ((long long)c * I) / P);
  }
  __device__ __forceinline__ void at(int c, int k, int& pair, int& chunk) const {
    const long long it = ((long long)c * I) / P + k;
    pair = (int)(it / n_chunks);
    chunk = (int)(it % n_chunks);
  }
};

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One block of one row and one 64-column half, the common case (n a multiple of 128, not the
// last block): S read 32 columns at a time (the next load in flight while these are
// exponentiated), and the sums below/above the row's diagonal column r (warp `grp` holds rows
// 32grp..32grp+31, so columns of 32-column chunk c < grp are all below, c > grp all above, and
// chunk grp splits at the lane).
__device__ __forceinline__ void block_sums_fast(uint32_t sbase, float nm, int grp, int lane, int half, float& lo,
                                                float& hi) {
  uint32_t v[2][32];
  lo = 0.f;
  hi = 0.f;
  tmem_ld32(sbase, v[0]);
  tmem_ld_wait_regs(v[0]);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t(&x)[32] = v[c];
    if (c == 0) tmem_ld32(sbase + 32, v[1]);
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const float e = fast_exp2(fmaf(__uint_as_float(x[q]), kScaleLog2, nm));
      x[q] = __float_as_uint(e);
      s4[q & 3] += e;
    }
    const float sc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    const int cc = 2 * half + c;  // chunk index within the 128 columns
    if (cc < grp) {
      lo += sc;
    } else if (cc > grp) {
      hi += sc;
    } else {
      float l2[2] = {0.f, 0.f}, h2[2] = {0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float e = __uint_as_float(x[q]);
        if (q <= lane) l2[q & 1] += e; else h2[q & 1] += e;
      }
      lo += l2[0] + l2[1];
      hi += h2[0] + h2[1];
    }
    if (c == 0) tmem_ld_wait_regs(v[1]);
  }
}

// Largest logit of the row in one 64-column half of this block (after the causal mask; col0 is
// the half's first column), scaled to log2 units.
__device__ __forceinline__ float block_max_scaled(uint32_t sbase, int col0, int lim, bool edge) {
  uint32_t v[2][32];
  float mx = -INFINITY;
  tmem_ld32(sbase, v[0]);
  tmem_ld32(sbase + 32, v[1]);
  tmem_ld_wait_regs(v[0]);
  tmem_ld_wait_regs(v[1]);
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
      float a = __uint_as_float(v[c][q]), b = __uint_as_float(v[c][q + 1]);
      if (edge) {
        if (col0 + c * 32 + q > lim) a = -INFINITY;
        if (col0 + c * 32 + q + 1 > lim) b = -INFINITY;
      }
      float m3;
      asm("max.f32 %0, %1, %2, %3;" : "=f"(m3) : "f"(mx), "f"(a), "f"(b));
      mx = m3;
    }
  return mx * kScaleLog2;
}

// RAGGED: n is not a multiple of 128 (separate instance, so the common case keeps the lane-aligned
// split with no extra work in its exponential loop).
template <bool RAGGED>
__global__ void __launch_bounds__(THREADS, 1)
    proxy_pass_kernel(const __grid_constant__ CUtensorMap q_map,
                      const __grid_constant__ CUtensorMap k_map, const SelectArgs a) {
  extern __shared__ uint8_t smem_raw[];
  ProxySmem& sm = *reinterpret_cast<ProxySmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const volatile int* abort = &sm.abort;

  const Shape& s = a.s;
  const int ppg = (s.G + 1) / 2;
  const Sched sched(s, (int)gridDim.x);
  const int cta = blockIdx.x;
  const int my_items = sched.count(cta);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 3);  // MMA commit + two pooling warps
    }
    for (int t = 0; t < 2; ++t)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[t][b], 1);
        mbar_init(&sm.s_free[t][b], 8);  // the tile's eight softmax warps
      }
    mbar_init(&sm.mma_done, 1);
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

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&q_map);
      tma_prefetch_desc(&k_map);
      int kc = 0, qn = 0, prev_pair = -1;
      bool ok = true;
      for (int it = 0; ok && it < my_items; ++it) {
        int ip, ic;
        sched.at(cta, it, ip, ic);
        const Item w(s, ip, ic);
        if (w.pair != prev_pair) {
          // the last 128 queries of each head, once the MMAs on the previous pair's tiles are done
          trace_mark(a.trace, 0, 0, 1, it);
          if (qn > 0 && !mbar_wait(&sm.q_empty, (qn - 1) & 1, abort)) {
            fail(sm, a.status);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES * w.ntiles);
          for (int t = 0; t < w.ntiles; ++t) {
            tma_load_3d(&q_map, &sm.q_full, sm.q[t], 0, s.n - kB, w.h0 + t);
            tma_load_3d(&q_map, &sm.q_full, sm.q[t] + kB * 64, 64, s.n - kB, w.h0 + t);
          }
          ++qn;
          prev_pair = w.pair;
        }
        for (int j = 0; j < w.nblk; ++j, ++kc) {
          const int st = kc % NS;
          trace_mark(a.trace, 0, 0, 2, kc);
          if (!mbar_wait(&sm.k_empty[st], ((kc / NS) & 1) ^ 1, abort)) {
            fail(sm, a.status);
            ok = false;
            break;
          }
          const int ky = (w.kb0 + j) * kB;  // rows past n of a partial last block arrive as zeros
          mbar_arrive_expect_tx(&sm.k_full[st], TILE_BYTES);
          tma_load_3d(&k_map, &sm.k_full[st], sm.k[st], 0, ky, w.kv);
          tma_load_3d(&k_map, &sm.k_full[st], sm.k[st] + kB * 64, 64, ky, w.kv);
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last load of each stage.
      trace_mark(a.trace, 0, 0, 3, kc);
      if (qn > 0) mbar_wait(&sm.q_full, (qn - 1) & 1, nullptr);
      for (int j = max(0, kc - NS); j < kc; ++j) mbar_wait(&sm.k_full[j % NS], (j / NS) & 1, nullptr);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      int kc = 0, qn = 0, prev_pair = -1;
      int tb[2] = {0, 0};  // blocks issued per tile so far (S buffer and phase)
      bool ok = true;
      for (int it = 0; ok && it < my_items; ++it) {
        int ip, ic;
        sched.at(cta, it, ip, ic);
        const Item w(s, ip, ic);
        if (w.pair != prev_pair) {
          if (qn > 0) umma_commit(&sm.q_empty);  // the old Q tiles are free once these MMAs finish
          trace_mark(a.trace, 0, 1, 1, it);
          if (!mbar_wait(&sm.q_full, qn & 1, abort)) {
            fail(sm, a.status);
            ok = false;
            break;
          }
          ++qn;
          prev_pair = w.pair;
        }
        for (int j = 0; ok && j < w.nblk; ++j, ++kc) {
          const int st = kc % NS;
          trace_mark(a.trace, 0, 1, 2, kc);
          if (!mbar_wait(&sm.k_full[st], (kc / NS) & 1, abort)) {
            fail(sm, a.status);
            ok = false;
            break;
          }
          for (int t = 0; t < w.ntiles; ++t) {
            trace_mark(a.trace, 0, 1, 3 + t, tb[t]);
            const int b = tb[t] & 1;
            if (!mbar_wait(&sm.s_free[t][b], ((tb[t] >> 1) & 1) ^ 1, abort)) {
              fail(sm, a.status);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t qa = smem_u32(sm.q[t]), ka = smem_u32(sm.k[st]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
              umma_ss(tmem + t * 256 + b * 128, desc_kmajor_sw128(qa + off), desc_kmajor_sw128(ka + off), idesc,
                      kk > 0);
            }
            umma_commit(&sm.s_full[t][b]);
            ++tb[t];
          }
          if (!ok) break;
          umma_commit(&sm.k_empty[st]);
        }
      }
      // Never release TMEM under a running MMA: wait (bounded) for all issued work.
      trace_mark(a.trace, 0, 1, 5, kc);
      umma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0, nullptr);
      trace_mark(a.trace, 0, 1, 6, kc);
    }
    __syncwarp();
  } else if (warp < SOFTMAX_WARPS) {
    // ------------------------------------------------------------------ softmax rows
    const int t = warp >> 3;           // tile (head of the pair)
    const int half = (warp >> 2) & 1;  // columns 64*half .. 64*half+63
    const int grp = warp & 3;          // TMEM lane quarter
    const int r = grp * 32 + lane;
    const int col0 = 64 * half;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    // With n = 128 (N_b - 1) + t_last, t_last in [1, 128]: row r sits at position n-128+r, a key
    // at column c of block kb has offset o = n-128+r - 128 kb - c, and the slash block of o is
    // N_b-2-kb + floor((t_last + r - c) / 128). Columns c <= (t_last + r) mod 128 ("lo") go to the
    // higher of the two slash blocks a (row, block) meets. When t_last = 128 that column is r.
    const int t_last = s.n - (s.nb - 1) * kB;
    constexpr bool ragged = RAGGED;
    const int sigma = (t_last + r) & (kB - 1);
    int tb = 0;  // blocks of this tile so far (S buffer and phase)
    bool ok = true;
    for (int it = 0; ok && it < my_items; ++it) {
      int ip, ic;
      sched.at(cta, it, ip, ic);
      const Item w(s, ip, ic);
      // (a group's odd last head: tile 1 has no head in its pair)
      if (t < w.ntiles) {
      const int h = w.h0 + t;
      float2* part = a.part + ((size_t)h * s.nb * 2 + half) * kB + r;  // block kb at [kb * 2 * kB]
      float m = -INFINITY;
      float tot = 0.f;
      float rec = 0.f;  // recency-window mass in block N_b-2 (columns >= t_last), ragged n only
      for (int j = 0; j < w.nblk; ++j, ++tb) {
        const int b = tb & 1;
        const bool tracer = grp == 0 && lane == 0;
        if (tracer) trace_mark(a.trace, 0, 2 + t + 2 * half, 1, tb);
        if (!warp_wait(&sm.s_full[t][b], (tb >> 1) & 1, abort)) {
          fail(sm, a.status);
          ok = false;
          break;
        }
        tc_fence_after();
        // Exponentials use the segment's reference m of its earlier blocks without this block's
        // maximum (fp32 keeps them exact until they overflow); the first block sets m from its
        // maximum, and a block whose sum would leave [0, 2^64] is redone against its maximum with
        // the earlier sums rescaled. S stays in TMEM until the block is done.
        const uint32_t sbase = tmem + t * 256 + b * 128 + col0 + lane_off;
        const int kb = w.kb0 + j;
        const int lim = s.n - kB + r - kb * kB;  // row r sees columns c <= lim of this block
        const bool edge = RAGGED ? kb >= s.nb - 2 : kb == s.nb - 1;  // blocks lim can cut
        const bool rec_blk = ragged && s.nb >= 3 && kb == s.nb - 2;
        // warp-uniform: the max pass reads TMEM with warp-collective loads, and a row whose half
        // of the chunk's first block lay wholly beyond its causal limit still has no reference
        // while the other rows of its warp have one
        bool need_max = __any_sync(0xffffffffu, m == -INFINITY);
        float lo = 0.f, hi = 0.f, rx = 0.f;
        for (int attempt = 0; attempt < 2; ++attempt) {
          if (need_max) {
            const float xm = block_max_scaled(sbase, col0, lim, edge);
            if (xm > m) {
              const float f = fast_exp2(m - xm);  // 0 while m = -inf
              if (m != -INFINITY) {
                for (int jj = 0; jj < j; ++jj) {  // rare: this thread's earlier sums of the chunk
                  float2 pv = part[(size_t)(w.kb0 + jj) * 2 * kB];
                  pv.x *= f;
                  pv.y *= f;
                  part[(size_t)(w.kb0 + jj) * 2 * kB] = pv;
                }
              }
              tot *= f;
              rec *= f;
              m = xm;
            }
          }
          const float nm = -m;
          if (!RAGGED && !edge) {
            block_sums_fast(sbase, nm, grp, lane, half, lo, hi);
          } else {
            // hardware exp2 only, every column tested against the causal limit and (n not a
            // multiple of 128) the split column, which is not aligned with the lanes
            lo = 0.f;
            hi = 0.f;
            rx = 0.f;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              uint32_t v[32];
              tmem_ld32(sbase + c * 32, v);
              tmem_ld_wait_regs(v);
#pragma unroll
              for (int q = 0; q < 32; ++q) {
                const int col = col0 + c * 32 + q;
                float e = fast_exp2(fmaf(__uint_as_float(v[q]), kScaleLog2, nm));
                if (edge && col > lim) e = 0.f;  // causal: row r sees keys up to its own position
                const bool low = RAGGED ? col <= sigma : col <= r;
                if (low) lo += e; else hi += e;
                if (rec_blk && col >= t_last) rx += e;
              }
            }
          }
          const bool redo = !need_max && !(lo + hi <= 18446744073709551616.0f);  // 2^64, or inf / nan
          if (!__any_sync(0xffffffffu, redo)) break;
          need_max = true;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[t][b]);
        part[(size_t)kb * 2 * kB] = make_float2(lo, hi);
        tot += lo + hi;
        if (rec_blk) rec = rx;
      }
      if (ok) {
        // the segment (chunk, half): its reference and total per row
        const size_t ci = (((size_t)h * s.n_chunks + w.chunk) * 2 + half) * kB + r;
        a.chunk_max[ci] = m;
        a.chunk_tot[ci] = tot;
        if (ragged && s.nb >= 3 && s.nb - 2 >= w.kb0 && s.nb - 2 < w.kb0 + w.nblk)
          a.rec_extra[((size_t)h * 2 + half) * kB + r] = rec;
      }
      }
    }
    __syncwarp();
  } else if (warp >= POOL_WARP) {
    // ------------------------------------------------------------------ K block mean (PE path)
    // Column chunk cc (8 bf16 of each row) belongs to the group's item cc % ppg (by the item's
    // pair index within its group), and within the item to pooling warp (its slot index) % 2.
    // Lane (slot, row group) sums every groups-th row of its chunk; shuffles combine the row
    // groups.
    const int pw = warp - POOL_WARP;
    int kc = 0;
    bool ok = true;
    for (int it = 0; ok && it < my_items; ++it) {
      int ip, ic;
      sched.at(cta, it, ip, ic);
      const Item w(s, ip, ic);
      const int ncc_item = (16 - w.pig + ppg - 1) / ppg;
      const int ncc = (ncc_item - pw + 1) / 2;
      int groups = 1;
      while (groups < 32 && groups * 2 * ncc <= 32) groups *= 2;
      const int slot = lane / groups;
      const int rg = lane % groups;
      const bool active = slot < ncc;
      const int cc = w.pig + (2 * slot + pw) * ppg;
      const int half = cc >> 3, ch = cc & 7;
      for (int j = 0; j < w.nblk; ++j, ++kc) {
        const int st = kc % NS;
        if (lane == 0 && pw == 0) trace_mark(a.trace, 0, 6, 1, kc);
        if (!warp_wait(&sm.k_full[st], (kc / NS) & 1, abort)) {
          fail(sm, a.status);
          ok = false;
          break;
        }
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        if (active) {
          // 128/groups rows per lane, eight independent 16-byte loads in flight
          const uint8_t* base = reinterpret_cast<const uint8_t*>(sm.k[st]) + half * HALF_BYTES;
          for (int row0 = rg; row0 < kB; row0 += 8 * groups) {
            uint4 u[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const int row = row0 + x * groups;
              u[x] = row < kB ? *reinterpret_cast<const uint4*>(base + sw128_offset(row, ch)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u[x]);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(p2[i]);
                acc[2 * i] += f.x;
                acc[2 * i + 1] += f.y;
              }
            }
          }
        }
        for (int o = 1; o < groups; o <<= 1)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
        if (active && rg == 0) {
          const size_t kb = (size_t)w.kb0 + j;
          float4* dst = reinterpret_cast<float4*>(a.kbar + ((size_t)w.kv * s.nb + kb) * kD + cc * 8);
          // a partial last block averages the rows it has (the rest arrived as zeros)
          const float inv = kb == (size_t)s.nb - 1 ? 1.f / (float)(s.n - (s.nb - 1) * kB) : 1.f / kB;
          float mv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mv[i] = acc[i] * inv;
          dst[0] = make_float4(mv[0], mv[1], mv[2], mv[3]);
          dst[1] = make_float4(mv[4], mv[5], mv[6], mv[7]);
          // the same means as three bf16 terms whose sum is exact (hi, mid, lo), for the
          // tensor-core pooled scores: [kv][term][N_b][128]
          uint32_t pk[3][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float r0 = mv[2 * i], r1 = mv[2 * i + 1];
#pragma unroll
            for (int tt = 0; tt < 3; ++tt) {
              const __nv_bfloat16 b0 = __float2bfloat16_rn(r0), b1 = __float2bfloat16_rn(r1);
              pk[tt][i] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
              r0 -= __bfloat162float(b0);
              r1 -= __bfloat162float(b1);
            }
          }
#pragma unroll
          for (int tt = 0; tt < 3; ++tt)
            *reinterpret_cast<uint4*>(a.kparts + (((size_t)w.kv * 3 + tt) * s.nb + kb) * kD + cc * 8) =
                make_uint4(pk[tt][0], pk[tt][1], pk[tt][2], pk[tt][3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.k_empty[st]);
      }
    }
    __syncwarp();
  }

  if (lane == 0 && (warp == PRODUCER_WARP || warp == MMA_WARP || warp == 0 || warp == 8 || warp == POOL_WARP))
    trace_mark(a.trace, 0, 7, 7, warp);
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int num_sms() {
  static int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 148;
    return v;
  }();
  return n;
}

cudaError_t launch_proxy_pass(const CUtensorMap& q_map, const CUtensorMap& k_map, const SelectArgs& a,
                              cudaStream_t st) {
  const size_t smem = sizeof(ProxySmem) + 1024;
  const bool ragged = a.s.n % kB != 0;
  auto kernel = ragged ? proxy_pass_kernel<true> : proxy_pass_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // Persistent: one CTA per SM.
  const int n_items = a.s.h_kv * ((a.s.G + 1) / 2) * a.s.n_chunks;
  kernel<<<min(n_items, num_sms()), THREADS, smem, st>>>(q_map, k_map, a);
  return cudaGetLastError();
}

}  // namespace crisp
