// proxy_pass.cu — the proxy attention of CRISP reduced on the fly (CRISP paper §2: proxy
// attention A_hat = softmax(Q_hat K^T / sqrt(d)) over a representative query subset, here the
// last query block; §4: vertical = column means, slash = diagonal means, pooled into blocks).
//
// One CTA handles two q-heads of one GQA group (two "tiles": their last query blocks) against a
// chunk of kProxyChunk key blocks of the shared kv-head, so every K block is read once for both.
//   warp 8      TMA producer: both Q tiles, then the chunk's K blocks through a 3-stage ring;
//   warp 9      one thread issues S_t = Q_t K_blk^T (128x128x128, bf16 -> fp32) into a
//               double-buffered TMEM tile per head;
//   warps 0-7   softmax, one warpgroup per head, one proxy row per thread: read the S row with
//               one TMEM round trip, mask the keys the causal limit cuts (key j visible to row r
//               iff j <= n-B+r), and accumulate exp2(x - m) against a lagging row reference m (set
//               by the chunk's first block, moved only when a block's sum would leave
//               [0, 2^64]) into two sums per key block: keys at or below the row's diagonal
//               offset (t <= r) and above it (t > r);
//   warps 10-11 sum rows of each K block into the mean-pooled key K_bar of the PE path; the
//               CTAs of one group share the 16 column chunks between them.
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
constexpr int THREADS = 384;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int POOL_WARP = 10;   // and 11: two warps share the pooling
constexpr uint32_t TILE_BYTES = kB * kD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr float kScaleLog2 = 0.12751743074380045f;  // log2(e) / sqrt(128)

struct __align__(1024) ProxySmem {
  __nv_bfloat16 q[2][kB * kD];  // two 128-byte-swizzled halves [128 rows][64 cols] per tile
  __nv_bfloat16 k[NS][kB * kD];
  float2 part[2][kProxyChunk][kB];  // per tile, block and row: (lower, upper) sums
  uint64_t q_full;
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
  const int pairs_per_group = (s.G + 1) / 2;
  const int n_pairs = s.h_kv * pairs_per_group;
  const int pair = blockIdx.x % n_pairs;
  const int chunk = blockIdx.x / n_pairs;
  const int kv = pair / pairs_per_group;
  const int pig = pair % pairs_per_group;  // pair index within its group
  const int h0 = kv * s.G + 2 * pig;
  const int ntiles = (2 * pig + 1 < s.G) ? 2 : 1;
  const int kb0 = chunk * kProxyChunk;
  const int nblk = min(kProxyChunk, s.nb - kb0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 3);  // MMA commit + two pooling warps
    }
    for (int t = 0; t < 2; ++t)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[t][b], 1);
        mbar_init(&sm.s_free[t][b], 4);
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
      mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES * ntiles);
      for (int t = 0; t < ntiles; ++t) {  // the last 128 queries of each head
        tma_load_3d(&q_map, &sm.q_full, sm.q[t], 0, s.n - kB, h0 + t);
        tma_load_3d(&q_map, &sm.q_full, sm.q[t] + kB * 64, 64, s.n - kB, h0 + t);
      }
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int st = j % NS;
        if (!mbar_wait(&sm.k_empty[st], ((j / NS) & 1) ^ 1, abort)) {
          fail(sm, a.status);
          break;
        }
        const int ky = (kb0 + j) * kB;  // rows past n of a partial last block arrive as zeros
        mbar_arrive_expect_tx(&sm.k_full[st], TILE_BYTES);
        tma_load_3d(&k_map, &sm.k_full[st], sm.k[st], 0, ky, kv);
        tma_load_3d(&k_map, &sm.k_full[st], sm.k[st] + kB * 64, 64, ky, kv);
        ++issued;
      }
      // Never leave with copies in flight: wait (bounded) for the last load of each stage.
      mbar_wait(&sm.q_full, 0, nullptr);
      for (int j = max(0, issued - NS); j < issued; ++j) mbar_wait(&sm.k_full[j % NS], (j / NS) & 1, nullptr);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      bool ok = mbar_wait(&sm.q_full, 0, abort);
      if (!ok) fail(sm, a.status);
      for (int j = 0; ok && j < nblk; ++j) {
        const int st = j % NS, b = j & 1;
        if (!mbar_wait(&sm.k_full[st], (j / NS) & 1, abort)) {
          fail(sm, a.status);
          break;
        }
        for (int t = 0; t < ntiles && ok; ++t) {
          if (!mbar_wait(&sm.s_free[t][b], ((j >> 1) & 1) ^ 1, abort)) {
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
        }
        if (!ok) break;
        umma_commit(&sm.k_empty[st]);
      }
      // Never release TMEM under a running MMA: wait (bounded) for all issued work.
      umma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0, nullptr);
    }
    __syncwarp();
  } else if (warp < 4 * ntiles) {
    // ------------------------------------------------------------------ softmax rows
    const int t = warp >> 2;
    const int grp = warp & 3;
    const int r = grp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    // With n = 128 (N_b - 1) + t_last, t_last in [1, 128]: row r sits at position n-128+r, a key
    // at column c of block kb has offset o = n-128+r - 128 kb - c, and the slash block of o is
    // N_b-2-kb + floor((t_last + r - c) / 128). Columns c <= (t_last + r) mod 128 ("lo") go to the
    // higher of the two slash blocks a (row, block) meets. When t_last = 128 that column is r.
    const int t_last = s.n - (s.nb - 1) * kB;
    constexpr bool ragged = RAGGED;
    const int sigma = (t_last + r) & (kB - 1);
    float m = -INFINITY;
    float rec = 0.f;  // recency-window mass in block N_b-2 (columns >= t_last), ragged n only
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      if (!warp_wait(&sm.s_full[t][b], (j >> 1) & 1, abort)) {
        fail(sm, a.status);
        ok = false;
        break;
      }
      tc_fence_after();
      // Exponentials use the row reference m of the chunk's earlier blocks without this block's
      // maximum (fp32 keeps them exact until they overflow); the first block sets m from its
      // maximum, and a block whose sum would leave [0, 2^64] is redone against its maximum with
      // the earlier partial sums rescaled. S stays in TMEM until the block is done.
      uint32_t v[4][32];
      const uint32_t sbase = tmem + t * 256 + b * 128 + lane_off;
      const int kb = kb0 + j;
      const int lim = s.n - kB + r - kb * kB;  // row r sees columns c <= lim of this block
      const bool edge = RAGGED ? kb >= s.nb - 2 : kb == s.nb - 1;  // blocks lim can cut
      const bool rec_blk = ragged && s.nb >= 3 && kb == s.nb - 2;
      bool need_max = (m == -INFINITY);
      float lo = 0.f, hi = 0.f, rx = 0.f;
      for (int attempt = 0; attempt < 2; ++attempt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(sbase + c * 32, v[c]);
        tmem_ld_wait();
        if (edge) {
          // causal: row r (position n-128+r) sees keys up to its own position only
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (c * 32 + q > lim) v[c][q] = __float_as_uint(-INFINITY);
        }
        if (need_max) {
          float mx8[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) mx8[q] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 32; ++q) mx8[q & 7] = fmaxf(mx8[q & 7], __uint_as_float(v[c][q]));
          const float xm = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * kScaleLog2;
          if (xm > m) {
            const float f = fast_exp2(m - xm);  // 0 while m = -inf
            for (int jj = 0; jj < j; ++jj) {
              float2 pv = sm.part[t][jj][r];
              pv.x *= f;
              pv.y *= f;
              sm.part[t][jj][r] = pv;
            }
            rec *= f;
            m = xm;
          }
        }
        const float nm = -m;
        // chunks below the warp's group hold keys t <= r, chunks above hold t > r; chunk grp
        // straddles the diagonal offset lane by lane
        lo = 0.f;
        hi = 0.f;
        rx = 0.f;
        if constexpr (RAGGED) {
          // the split column (t_last + r) mod 128 is not aligned with the warp's lanes
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int col = c * 32 + q;
              const float e = fast_exp2(fmaf(__uint_as_float(v[c][q]), kScaleLog2, nm));
              if (col <= sigma) lo += e; else hi += e;
              if (rec_blk && col >= t_last) rx += e;
            }
        } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float e = fast_exp2(fmaf(__uint_as_float(v[c][q]), kScaleLog2, nm));
            v[c][q] = __float_as_uint(e);
            s4[q & 3] += e;
          }
          const float sc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
          if (c < grp) {
            lo += sc;
          } else if (c > grp) {
            hi += sc;
          } else {
            float l2[2] = {0.f, 0.f}, h2[2] = {0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float e = __uint_as_float(v[c][q]);
              if (q <= lane) l2[q & 1] += e; else h2[q & 1] += e;
            }
            lo += l2[0] + l2[1];
            hi += h2[0] + h2[1];
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
      sm.part[t][j][r] = make_float2(lo, hi);
      if (rec_blk) rec = rx;
    }
    if (ok) {
      const int h = h0 + t;
      float tot = 0.f;
      for (int jj = 0; jj < nblk; ++jj) {
        const float2 pv = sm.part[t][jj][r];
        a.part[((size_t)h * s.nb + kb0 + jj) * kB + r] = pv;
        tot += pv.x + pv.y;
      }
      const size_t ci = ((size_t)h * s.n_chunks + chunk) * kB + r;
      a.chunk_max[ci] = m;
      a.chunk_tot[ci] = tot;
      if (ragged && s.nb >= 3 && s.nb - 2 >= kb0 && s.nb - 2 < kb0 + nblk) a.rec_extra[(size_t)h * kB + r] = rec;
    }
    __syncwarp();
  } else if (warp >= POOL_WARP) {
    // ------------------------------------------------------------------ K block mean (PE path)
    // Column chunk cc (8 bf16 of each row) belongs to the group's CTA cc % pairs_per_group, and
    // within the CTA to pooling warp (its slot index) % 2. Lane (slot, row group) sums every
    // groups-th row of its chunk; shuffles combine the row groups.
    const int pw = warp - POOL_WARP;
    const int ncc_cta = (16 - pig + pairs_per_group - 1) / pairs_per_group;
    const int ncc = (ncc_cta - pw + 1) / 2;
    int groups = 1;
    while (groups < 32 && groups * 2 * ncc <= 32) groups *= 2;
    const int slot = lane / groups;
    const int rg = lane % groups;
    const bool active = slot < ncc;
    const int cc = pig + (2 * slot + pw) * pairs_per_group;
    const int half = cc >> 3, ch = cc & 7;
    for (int j = 0; j < nblk; ++j) {
      const int st = j % NS;
      if (!warp_wait(&sm.k_full[st], (j / NS) & 1, abort)) {
        fail(sm, a.status);
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
        float4* dst = reinterpret_cast<float4*>(a.kbar + ((size_t)kv * s.nb + kb0 + j) * kD + cc * 8);
        // a partial last block averages the rows it has (the rest arrived as zeros)
        const float inv = kb0 + j == s.nb - 1 ? 1.f / (float)(s.n - (s.nb - 1) * kB) : 1.f / kB;
        dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.k_empty[st]);
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

cudaError_t launch_proxy_pass(const CUtensorMap& q_map, const CUtensorMap& k_map, const SelectArgs& a,
                              cudaStream_t st) {
  const size_t smem = sizeof(ProxySmem) + 1024;
  const bool ragged = a.s.n % kB != 0;
  auto kernel = ragged ? proxy_pass_kernel<true> : proxy_pass_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_pairs = a.s.h_kv * ((a.s.G + 1) / 2);
  dim3 grid(n_pairs * a.s.n_chunks);
  kernel<<<grid, THREADS, smem, st>>>(q_map, k_map, a);
  return cudaGetLastError();
}

}  // namespace crisp
