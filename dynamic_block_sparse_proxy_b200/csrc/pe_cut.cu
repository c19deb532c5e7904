// pe_cut.cu — the Pooled-Estimation path of CRISP (paper §2 and §4: pooled query and key
// blocks, softmax, then the flattened gamma cumulative cut; the rcap.io summary's per-head
// pseudocode: gamma_cumsum(pool(Q), pool(K), gamma)).
//
// For every head routed to PE:
//   qbar_kernel     Q_bar[qb] = mean of the block's query rows (fp32; 128, or fewer in a partial
//                   last block), read once from HBM, stored as three bf16 terms whose sum is the
//                   fp32 value exactly (hi, mid, lo);
//   scores_kernel   logits Q_bar[qb] . K_bar[kb] / sqrt(d) for kb <= qb, one 128x128 tile per
//                   CTA on the tensor cores: the six products hi.hi + hi.mid + mid.hi + hi.lo +
//                   mid.mid + lo.hi of the split operands accumulate in fp32 in TMEM (the terms
//                   left out are below 2^-24 of the product), so the tile carries fp32 accuracy;
//   rowsoft_kernel  P[qb, kb] = softmax over kb <= qb, in place, one warp per row held in
//                   registers, plus the first radix histogram; the last CTA of a head picks the
//                   level-1 bin;
//   cut_hist_kernel levels 2 and 3 of the radix select (11 + 10 + 10 bits of the positive fp32
//                   pattern, count and fixed-point mass per bin); the last CTA of a head picks the
//                   bin. The result is the value T where the mass of the sorted prefix first
//                   reaches gamma*N_b: every entry > T is kept; entries equal to T are kept in
//                   (qb, kb) order until the target is met, which reproduces the sort order
//                   (P desc, qb asc, kb asc) of the global cut.
// gamma >= 1 keeps every causal block.
#include "crisp_internal.h"
#include "sm100.cuh"

#include <algorithm>

namespace crisp {
namespace {

__device__ __forceinline__ bool is_pe(const SelectArgs& a, int h) { return a.route[h] == 0; }

// x == hi + mid + lo exactly (fp32 has 24 significant bits, each bf16 term takes 8 of them).
__device__ __forceinline__ void split3(float x, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r1);
  lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
}

// -------------------------------------------------------------------------------- Q_bar
__global__ void __launch_bounds__(128) qbar_kernel(const SelectArgs a) {
  const int qb = blockIdx.x, h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const Shape& s = a.s;
  const int t = threadIdx.x, c16 = t & 15, rg = t >> 4;
  const __nv_bfloat16* base = a.q + ((size_t)h * s.ld + (size_t)qb * kB) * kD + c16 * 8;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const int rows = min(kB, s.n - qb * kB);  // a partial last block has fewer rows
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int row = rg + 8 * i;
    const uint4 u = row < rows ? __ldg(reinterpret_cast<const uint4*>(base + (size_t)row * kD)) : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p2[j]);
      acc[2 * j] += f.x;
      acc[2 * j + 1] += f.y;
    }
  }
  __shared__ float red[8][kD];
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rg][c16 * 8 + i] = acc[i];
  __syncthreads();
  float v = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) v += red[i][t];
  v *= 1.f / (float)rows;
  __nv_bfloat16 p0, p1, p2;
  split3(v, p0, p1, p2);
  __nv_bfloat16* dst = a.qparts + ((size_t)h * 3 * s.nb + qb) * kD + t;  // [h][part][nb][128]
  dst[0] = p0;
  dst[(size_t)s.nb * kD] = p1;
  dst[(size_t)2 * s.nb * kD] = p2;
}

// -------------------------------------------------------------------------------- logits
// One CTA per (PE head, 128x128 tile of the block-causal pooled matrix). The head dimension runs
// in two 64-column halves; per half the three terms of the Q_bar tile and of the K_bar tile
// arrive by TMA (6 x 16 KB, 128-byte swizzle) and one thread issues the 6 products x 4 UMMAs
// (M = N = 128, K = 16) into one fp32 TMEM accumulator. The four warps then read their 32 rows,
// scale by 1/sqrt(d), stage them in shared memory and store the causal part row by row.
constexpr int SC_THREADS = 128;
constexpr uint32_t PART_BYTES = kB * 64 * 2;  // 128 rows x 64 bf16
constexpr int STAGE_LD = kB + 1;              // padded staging row (floats)

struct __align__(1024) ScoreSmem {
  __nv_bfloat16 a[3][kB * 64];
  __nv_bfloat16 b[3][kB * 64];
  uint64_t full;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(float) * kB * STAGE_LD <= 6 * PART_BYTES, "staging fits in the operand buffers");

__global__ void __launch_bounds__(SC_THREADS) scores_kernel(const __grid_constant__ CUtensorMap qp_map,
                                                            const __grid_constant__ CUtensorMap kp_map,
                                                            const SelectArgs a) {
  const int h = blockIdx.y;
  if (!is_pe(a, h)) return;
  extern __shared__ uint8_t smem_raw[];
  ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Shape& s = a.s;
  // tile t of the lower triangle, row-major: (i, j) with j <= i
  const int t = blockIdx.x;
  int i = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
  while ((i + 1) * (i + 2) / 2 <= t) ++i;
  while (i * (i + 1) / 2 > t) --i;
  const int j = t - i * (i + 1) / 2;
  const int kv = h / s.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // products (A term, B term): smallest first, so the large ones are added last
  constexpr int PA[6] = {1, 0, 2, 0, 1, 0};
  constexpr int PB[6] = {1, 2, 0, 1, 0, 0};
  bool ok = true;
  for (int half = 0; half < 2 && ok; ++half) {
    if (threadIdx.x == 0) {
      if (half == 0) {
        tma_prefetch_desc(&qp_map);
        tma_prefetch_desc(&kp_map);
      }
      mbar_arrive_expect_tx(&sm.full, 6 * PART_BYTES);
      for (int p = 0; p < 3; ++p) {
        tma_load_3d(&qp_map, &sm.full, sm.a[p], 64 * half, i * kB, h * 3 + p);
        tma_load_3d(&kp_map, &sm.full, sm.b[p], 64 * half, j * kB, kv * 3 + p);
      }
      if (!mbar_wait(&sm.full, half & 1, nullptr)) {
        record_status(a.status, CRISP_ERR_DEVICE_TIMEOUT);
        sm.abort = 1;
      } else {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
        for (int pr = 0; pr < 6; ++pr)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(tmem, desc_kmajor_sw128(smem_u32(sm.a[PA[pr]]) + kk * 32),
                    desc_kmajor_sw128(smem_u32(sm.b[PB[pr]]) + kk * 32), idesc,
                    (half > 0 || pr > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sm.mma_done);
    }
    // every thread waits for the MMAs of this half (the buffers are reused, then TMEM is read);
    // a wait that runs out raises the CTA-wide abort flag, read by all after the barrier
    if (!mbar_wait(&sm.mma_done, half & 1, nullptr)) {
      record_status(a.status, CRISP_ERR_DEVICE_TIMEOUT);
      *reinterpret_cast<volatile int*>(&sm.abort) = 1;
    }
    __syncthreads();
    ok = *reinterpret_cast<volatile int*>(&sm.abort) == 0;
  }

  if (ok) {
    tc_fence_after();
    float* stage = reinterpret_cast<float*>(&sm.a[0][0]);
    const int r = warp * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    const float inv_sqrt_d = 0.08838834764831845f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld32(taddr + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 32; ++q) stage[r * STAGE_LD + c * 32 + q] = __uint_as_float(v[q]) * inv_sqrt_d;
    }
    __syncwarp();
    // the warp's rows, one at a time: lanes store consecutive key blocks
    float* P = a.pbuf + (size_t)h * s.cap;
    for (int rr = 0; rr < 32; ++rr) {
      const int row = warp * 32 + rr;
      const int qb = i * kB + row;
      if (qb >= s.nb) break;
      float* dst = P + (size_t)qb * (qb + 1) / 2;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int col = u * 32 + lane;
        const int kb = j * kB + col;
        if (kb <= qb) dst[kb] = stage[row * STAGE_LD + col];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------------ histograms, select
// Histogram masses are fixed point (2^-40 units, rounded to nearest, ties to even): integer
// atomics are exact and order-independent, and N_b * 2^40 stays far below 2^64. The product
// p * 2^40 of an fp32 p is exact in fp64, so one conversion rounds it as the definition asks.
__device__ __forceinline__ unsigned long long to_fixed(float p) {
  return __double2ull_rn((double)p * kMassUnit);  // exact product, rounded to nearest even
}

// Level-1 histogram of one row step (all lanes call it): only the mass of a bin decides the
// level-1 choice (the chosen bin's mass is positive, so it holds entries), so level 1 keeps no
// counts. Lanes with the same bin form a group (match.any); each group sums its fixed-point masses
// as three 16-bit parts (redux.sync, one instruction per part for every group at once) and its
// lowest lane adds them to three 32-bit shared arrays: no 64-bit shared atomics, and no two lanes
// of a warp hit the same word. A CTA's part sums stay below 2^32 (at most 8192 entries of < 2^16).
// Only bins [kL1Lo, kL1Lo + kL1Bins) can receive mass: an entry with a non-zero fixed-point mass has
// p >= 2^-41 (biased exponent >= 86, bin >= 86 * 8), and p <= 1 up to rounding (bin <= 127 * 8).
constexpr uint32_t kL1Lo = 86u * 8u;
constexpr uint32_t kL1Bins = 336;
__device__ __forceinline__ void warp_mass_add(uint32_t (*smass3)[kL1Bins], bool valid, float p) {
  const unsigned long long fx = valid ? to_fixed(p) : 0ull;
  const uint32_t bin = (__float_as_uint(p) >> 20) - kL1Lo;
  const uint32_t key = (fx != 0ull && bin < kL1Bins) ? bin : 0xffffffffu;
  const unsigned grp = __match_any_sync(0xffffffffu, key);
  const uint32_t s0 = __reduce_add_sync(grp, (uint32_t)(fx & 0xffffu));
  const uint32_t s1 = __reduce_add_sync(grp, (uint32_t)((fx >> 16) & 0xffffu));
  const uint32_t s2 = __reduce_add_sync(grp, (uint32_t)(fx >> 32));
  if (key != 0xffffffffu && (threadIdx.x & 31) == __ffs(grp) - 1) {
    atomicAdd(&smass3[0][key], s0);
    atomicAdd(&smass3[1][key], s1);
    atomicAdd(&smass3[2][key], s2);
  }
}

// Adds a CTA's shared histogram (nbins bins of counts and masses) to the head's global one, then
// reports whether this CTA is the last of the head's `ctas` to finish (that CTA then sees every
// CTA's updates).
__device__ bool flush_and_check_last(const SelectArgs& a, int h, const uint32_t* scnt,
                                     const unsigned long long* smass, int nbins, int ctas) {
  uint32_t* gcnt = a.hist_cnt + (size_t)h * kHistBins;
  unsigned long long* gmass = a.hist_mass + (size_t)h * kHistBins;
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) {
    if (scnt[i]) {
      atomicAdd(gcnt + i, scnt[i]);
      atomicAdd(gmass + i, smass[i]);
    }
  }
  __threadfence();
  __syncthreads();
  __shared__ int last;
  if (threadIdx.x == 0) last = atomicAdd(a.cut_done + h, 1u) == (unsigned)(ctas - 1);
  __syncthreads();
  if (last) __threadfence();  // acquire: the other CTAs' histogram updates are visible
  return last != 0;
}

// Run by the last CTA of a head at each level: walk the bins from the largest values down and
// find the bin where the cumulative mass (plus the mass already above the prefix) first reaches
// the target, narrow the prefix to it, and clear the histogram and the CTA counter for the next
// level. Masses are summed exactly in fixed point; the target is rounded up to the same grid.
// Level 1 also initialises the cut state. Needs blockDim.x == 256.
constexpr int SEL_THREADS = 256;
__device__ void select_bin(const SelectArgs& a, int h, int level) {
  const Shape& s = a.s;
  CutState* cs = a.cut + h;
  const int nbins = level == 1 ? kHistBins : 1024;
  const int per = nbins / SEL_THREADS;  // 8 or 4 consecutive bins per thread
  // written by other CTAs' atomics: read through L2
  uint32_t* gcnt = a.hist_cnt + (size_t)h * kHistBins;
  unsigned long long* gmass = a.hist_mass + (size_t)h * kHistBins;
  __shared__ unsigned long long tsum[SEL_THREADS];
  __shared__ int found;
  __shared__ unsigned long long found_hi;
  __shared__ uint32_t found_cnt;
  __shared__ CutState st;
  if (threadIdx.x == 0) {
    if (level == 1) {
      st.target = (double)a.gamma * (double)s.nb;
      st.mass_above = 0.0;
      st.prefix = 0;
      st.keep_all = a.gamma >= 1.0f ? 1u : 0u;
      st.thr_bits = 0;
      st.t_eq = 0;
      st.count_eq = 0;
    } else {
      st = *cs;
    }
    found = -1;
  }
  __syncthreads();
  if (!st.keep_all) {
    const int tid = threadIdx.x, b0 = tid * per;
    unsigned long long mb[8];
    uint32_t cb[8];
    unsigned long long m = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < per) {
        mb[k] = __ldcg(gmass + b0 + k);
        cb[k] = __ldcg(gcnt + b0 + k);
        m += mb[k];
      }
    }
    tsum[tid] = m;
    __syncthreads();
    // suffix sums over threads: after the loop tsum[t] = mass of bins >= t*per
    for (int off = 1; off < SEL_THREADS; off <<= 1) {
      const unsigned long long y = tid + off < SEL_THREADS ? tsum[tid + off] : 0ull;
      __syncthreads();
      tsum[tid] += y;
      __syncthreads();
    }
    const unsigned long long above = __double2ull_rn(st.mass_above * kMassUnit);
    const unsigned long long target = __double2ull_ru(st.target * kMassUnit);
    // the wanted bin b is the largest with above + suffix[b] >= target; the bins above b alone
    // stay below the target (one bin at most satisfies both)
    const unsigned long long suf0 = tid + 1 < SEL_THREADS ? tsum[tid + 1] : 0ull;  // bins >= b0 + per
    unsigned long long suf = suf0;
#pragma unroll
    for (int k = 7; k >= 0; --k) {
      if (k < per) {
        const unsigned long long hi = suf;
        suf += mb[k];
        // (both hold only if the bin's mass is positive: it holds entries)
        if (above + suf >= target && above + hi < target) atomicMax(&found, b0 + k);
      }
    }
    __syncthreads();
    // the owner of the chosen bin reports its count and the mass of the bins above it
    if (found >= 0 && found / per == tid) {
      unsigned long long hi = suf0;
#pragma unroll
      for (int k = 7; k >= 0; --k)
        if (k < per && b0 + k > found) hi += mb[k];
      found_hi = hi;
      found_cnt = cb[found - b0];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const int b = found;
      if (b < 0) {
        st.keep_all = 1;  // target not reachable: keep everything
      } else {
        st.mass_above = (double)(above + found_hi) / kMassUnit;
        st.prefix = (st.prefix << (level == 1 ? 0 : 10)) | (uint32_t)b;
        if (level == 3) {
          const uint32_t bits = st.prefix;
          const double val = (double)__uint_as_float(bits);
          const double rem = st.target - st.mass_above;
          uint32_t t = val > 0.0 ? (uint32_t)ceil(rem / val) : found_cnt;
          if (t < 1) t = 1;
          if (t > found_cnt) t = found_cnt;
          st.thr_bits = bits;
          st.t_eq = t;
          st.count_eq = found_cnt;
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *cs = st;
    a.cut_done[h] = 0;
  }
  for (int k = threadIdx.x; k < kHistBins; k += SEL_THREADS) {
    gcnt[k] = 0;
    gmass[k] = 0ull;
  }
}

// One warp per pooled row (8 rows per CTA): P[qb, kb] = softmax over kb <= qb, in place, and
// the level-1 mass histogram (bits 30..20 of the positive fp32 pattern). A row of up to 1024 entries
// stays in registers (32 per lane, all loads in flight at once); longer rows take three passes
// over memory. Exponentials use the exp2 unit on log2(e)-scaled logits.
constexpr int ROWS_PER_CTA = 8;
__global__ void __launch_bounds__(ROWS_PER_CTA * 32, 4) rowsoft_kernel(const SelectArgs a) {
  const int h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const Shape& s = a.s;
  __shared__ uint32_t smass3[3][kL1Bins];  // 16-bit parts of the fixed-point bin masses
  for (int i = threadIdx.x; i < (int)kL1Bins; i += blockDim.x) smass3[0][i] = smass3[1][i] = smass3[2][i] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int qb = blockIdx.x * ROWS_PER_CTA + w;
  constexpr float kLog2e = 1.4426950408889634f;
  if (qb < s.nb) {
    float* row = a.pbuf + (size_t)h * s.cap + (size_t)qb * (qb + 1) / 2;
    const int L = qb + 1;
    if (L <= 1024) {
      float x[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int i = u * 32 + lane;
        x[u] = (u * 32 < L && i < L) ? row[i] : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int u = 0; u < 32; ++u) mx = fmaxf(mx, x[u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float nm = -mx * kLog2e;
      float z = 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        if (u * 32 < L) {
          x[u] = (u * 32 + lane < L) ? fast_exp2(fmaf(x[u], kLog2e, nm)) : 0.f;
          z += x[u];
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      const float inv = 1.f / z;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int i = u * 32 + lane;
        if (u * 32 < L && i < L) row[i] = x[u] * inv;
      }
      // the histogram from the values just stored (this thread's own stores), in a rolled loop
#pragma unroll 2
      for (int base = 0; base < L; base += 32) {
        const int i = base + lane;
        const float p = i < L ? row[i] : 0.f;
        warp_mass_add(smass3, i < L, p);
      }
    } else {
      float mx = -INFINITY;
      for (int base = 0; base < L; base += 256) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = base + 32 * u + lane;
          x[u] = i < L ? row[i] : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) mx = fmaxf(mx, x[u]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float nm = -mx * kLog2e;
      float z = 0.f;
      for (int base = 0; base < L; base += 256) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = base + 32 * u + lane;
          x[u] = i < L ? row[i] : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float e = fast_exp2(fmaf(x[u], kLog2e, nm));
          z += e;
          const int i = base + 32 * u + lane;
          if (i < L) row[i] = e;  // unnormalised for now
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      const float inv = 1.f / z;
      __syncwarp();
      for (int base = 0; base < L; base += 256) {
        float e[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = base + 32 * u + lane;
          e[u] = i < L ? row[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = base + 32 * u + lane;
          const float p = e[u] * inv;
          if (i < L) row[i] = p;
          warp_mass_add(smass3, i < L, p);
        }
      }
    }
  }
  __syncthreads();
  // the CTA's bin masses (the parts recombined), then its share of the global histogram
  for (int i = threadIdx.x; i < (int)kL1Bins; i += blockDim.x) {
    const unsigned long long m = (unsigned long long)smass3[0][i] + ((unsigned long long)smass3[1][i] << 16) +
                                 ((unsigned long long)smass3[2][i] << 32);
    if (m) atomicAdd(a.hist_mass + (size_t)h * kHistBins + kL1Lo + i, m);
  }
  if (flush_and_check_last(a, h, nullptr, nullptr, 0, gridDim.x)) select_bin(a, h, 1);
}

// --------------------------------------------------------------------- histogram, levels 2-3
// level 2: entries whose bits[30:20] match the prefix, bin = bits[19:10]
// level 3: entries whose bits[30:10] match the prefix, bin = bits[9:0]
// Matching values are spread over many bins: plain per-lane shared atomics. Each CTA takes a
// contiguous range of the head's entries, sized so that one or two steps of HIST_UNROLL loads per
// thread cover it (the whole level is then about one round trip to memory).
constexpr int HIST_UNROLL = 8;
__global__ void __launch_bounds__(SEL_THREADS) cut_hist_kernel(const SelectArgs a, int level) {
  const int h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const CutState cs = a.cut[h];
  if (cs.keep_all) return;  // every CTA of the head sees the same state, and none selects
  const Shape& s = a.s;
  __shared__ uint32_t scnt[1024];
  __shared__ unsigned long long smass[1024];
  for (int i = threadIdx.x; i < 1024; i += SEL_THREADS) {
    scnt[i] = 0;
    smass[i] = 0ull;
  }
  __syncthreads();
  const float* P = a.pbuf + (size_t)h * s.cap;
  const int shift = level == 2 ? 20 : 10;
  const int bshift = level == 2 ? 10 : 0;
  // a contiguous range per CTA, HIST_UNROLL loads in flight per thread per step
  const long long per = (s.cap + gridDim.x - 1) / gridDim.x;
  const long long e0 = (long long)blockIdx.x * per, e1 = min((long long)s.cap, e0 + per);
  for (long long i0 = e0; i0 < e1; i0 += HIST_UNROLL * SEL_THREADS) {
    float v[HIST_UNROLL];
#pragma unroll
    for (int u = 0; u < HIST_UNROLL; ++u) {
      const long long i = i0 + u * SEL_THREADS + threadIdx.x;
      v[u] = i < e1 ? __ldg(P + i) : -1.f;  // -1 matches no prefix
    }
#pragma unroll
    for (int u = 0; u < HIST_UNROLL; ++u) {
      const uint32_t bits = __float_as_uint(v[u]);
      if ((bits >> shift) == cs.prefix) {
        const uint32_t bin = (bits >> bshift) & 1023u;
        atomicAdd(&scnt[bin], 1u);
        atomicAdd(&smass[bin], to_fixed(v[u]));
      }
    }
  }
  __syncthreads();
  if (flush_and_check_last(a, h, scnt, smass, 1024, gridDim.x)) select_bin(a, h, level);
}

}  // namespace

cudaError_t launch_pe(const SelectArgs& a, const CUtensorMap& qp_map, const CUtensorMap& kp_map, cudaStream_t st) {
  const Shape& s = a.s;
  qbar_kernel<<<dim3(s.nb, s.h_q), 128, 0, st>>>(a);
  const int T = (s.nb + kB - 1) / kB;
  const size_t smem = sizeof(ScoreSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  scores_kernel<<<dim3(T * (T + 1) / 2, s.h_q), SC_THREADS, smem, st>>>(qp_map, kp_map, a);
  rowsoft_kernel<<<dim3((s.nb + ROWS_PER_CTA - 1) / ROWS_PER_CTA, s.h_q), ROWS_PER_CTA * 32, 0, st>>>(a);
  // about 4K entries per CTA (two steps of 8 loads per thread), at most 1024 CTAs per head
  const int hist_ctas = (int)std::max<long long>(1, std::min<long long>(1024, (s.cap + 4095) / 4096));
  cut_hist_kernel<<<dim3(hist_ctas, s.h_q), SEL_THREADS, 0, st>>>(a, 2);
  cut_hist_kernel<<<dim3(hist_ctas, s.h_q), SEL_THREADS, 0, st>>>(a, 3);
  return cudaGetLastError();
}

}  // namespace crisp
