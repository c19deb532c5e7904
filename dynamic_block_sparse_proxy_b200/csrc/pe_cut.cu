// pe_cut.cu — the Pooled-Estimation path of CRISP (paper §2 and §4: pooled query and key
// blocks, softmax, then the flattened gamma cumulative cut; the rcap.io summary's per-head
// pseudocode: gamma_cumsum(pool(Q), pool(K), gamma)).
//
// For every head routed to PE:
//   qbar_kernel     Q_bar[qb] = mean of the block's query rows (fp32; 128, or fewer in a partial
//                   last block), read once from HBM;
//   scores_kernel   logits Q_bar[qb] . K_bar[kb] / sqrt(d) for kb <= qb (128x128 fp32 tiles);
//   rowsoft_kernel  P[qb, kb] = softmax over kb <= qb, in place, plus the first radix histogram;
//   cut_select / cut_hist: an exact radix select (11 + 10 + 10 bits of the positive fp32
//                   pattern, count and fixed-point mass per bin) of the value T where the mass of the
//                   sorted prefix first reaches gamma*N_b. Every entry > T is kept; entries equal
//                   to T are kept in (qb, kb) order until the target is met, which reproduces
//                   the sort order (P desc, qb asc, kb asc) of the global cut.
// gamma >= 1 keeps every causal block.
#include "crisp_internal.h"
#include "sm100.cuh"

#include <algorithm>

namespace crisp {
namespace {

__device__ __forceinline__ bool is_pe(const SelectArgs& a, int h) { return a.route[h] == 0; }

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
  a.qbar[((size_t)h * s.nb + qb) * kD + t] = v * (1.f / (float)rows);
}

// -------------------------------------------------------------------------------- logits
// 128x128 tile of Q_bar K_bar^T per CTA (256 threads, 8x8 outputs each: rows ty*4+{0..3, 64..67},
// columns tx*4+{0..3, 64..67}), fp32, the d dimension staged through shared memory 32 at a time.
constexpr int TS = 128;
constexpr int TK = 32;
__global__ void __launch_bounds__(256) scores_kernel(const SelectArgs a) {
  const int tk = blockIdx.x, tq = blockIdx.y, h = blockIdx.z;
  if (tk > tq || !is_pe(a, h)) return;
  const Shape& s = a.s;
  const int kv = h / s.G;
  __shared__ __align__(16) float qs[TK][TS + 4];
  __shared__ __align__(16) float ks[TK][TS + 4];
  const int q0 = tq * TS, k0 = tk * TS;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int d0 = 0; d0 < kD; d0 += TK) {
    // stage [128 rows][32 dims] of Q_bar and K_bar, transposed to [dim][row]
    for (int e = tid; e < TS * TK / 4; e += 256) {
      const int row = e / (TK / 4), c4 = (e % (TK / 4)) * 4;
      float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), kv4 = qv;
      if (q0 + row < s.nb) qv = *reinterpret_cast<const float4*>(a.qbar + ((size_t)h * s.nb + q0 + row) * kD + d0 + c4);
      if (k0 + row < s.nb) kv4 = *reinterpret_cast<const float4*>(a.kbar + ((size_t)kv * s.nb + k0 + row) * kD + d0 + c4);
      qs[c4 + 0][row] = qv.x; qs[c4 + 1][row] = qv.y; qs[c4 + 2][row] = qv.z; qs[c4 + 3][row] = qv.w;
      ks[c4 + 0][row] = kv4.x; ks[c4 + 1][row] = kv4.y; ks[c4 + 2][row] = kv4.z; ks[c4 + 3][row] = kv4.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < TK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&qs[kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&qs[kk][ty * 4 + 64]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ks[kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ks[kk][tx * 4 + 64]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float inv_sqrt_d = 0.08838834764831845f;
  float* P = a.pbuf + (size_t)h * s.cap;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int qb = q0 + ty * 4 + (i & 3) + (i >> 2) * 64;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int kb = k0 + tx * 4 + (j & 3) + (j >> 2) * 64;
      if (qb < s.nb && kb <= qb) P[(size_t)qb * (qb + 1) / 2 + kb] = acc[i][j] * inv_sqrt_d;
    }
  }
}

// ----------------------------------------------------------------- row softmax + histogram 1
// Histogram masses are fixed point (2^-40 units, rounded): integer atomics are exact and
// order-independent, and N_b * 2^40 stays far below 2^64.
__device__ __forceinline__ unsigned long long to_fixed(float p) {
  return __double2ull_rn((double)p * kMassUnit);
}

// Warp-aggregated update for rows whose values mostly share a bin: lanes with the same bin are
// summed first, one shared atomic per distinct bin. All lanes must call it.
__device__ __forceinline__ void warp_hist_add(uint32_t* scnt, unsigned long long* smass, bool valid, uint32_t bin,
                                              unsigned long long fx) {
  const int lane = threadIdx.x & 31;
  unsigned todo = __ballot_sync(0xffffffffu, valid);
  while (todo) {
    const int leader = __ffs(todo) - 1;
    const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
    const bool mine = ((todo >> lane) & 1u) && bin == lb;
    const unsigned grp = __ballot_sync(0xffffffffu, mine);
    unsigned long long v = mine ? fx : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == leader) {
      atomicAdd(&scnt[lb], (uint32_t)__popc(grp));
      atomicAdd(&smass[lb], v);
    }
    todo &= ~grp;
  }
}

__device__ __forceinline__ void flush_hist(uint32_t* scnt, unsigned long long* smass, int nbins, uint32_t* gcnt,
                                           unsigned long long* gmass) {
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) {
    if (scnt[i]) {
      atomicAdd(gcnt + i, scnt[i]);
      atomicAdd(gmass + i, smass[i]);
    }
  }
}

// One warp per pooled row (8 rows per CTA): P[qb, kb] = softmax over kb <= qb, in place, and
// the level-1 histogram (bits 30..20 of the positive fp32 pattern). Each lane keeps eight
// independent loads in flight; exponentials use the exp2 unit on log2(e)-scaled logits.
constexpr int ROWS_PER_CTA = 8;
__global__ void __launch_bounds__(ROWS_PER_CTA * 32) rowsoft_kernel(const SelectArgs a) {
  const int h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const Shape& s = a.s;
  __shared__ uint32_t scnt[kHistBins];
  __shared__ unsigned long long smass[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
    scnt[i] = 0;
    smass[i] = 0ull;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int qb = blockIdx.x * ROWS_PER_CTA + w;
  if (qb < s.nb) {
    float* row = a.pbuf + (size_t)h * s.cap + (size_t)qb * (qb + 1) / 2;
    const int L = qb + 1;
    constexpr float kLog2e = 1.4426950408889634f;
    // pass 1: maximum (8 independent loads in flight per lane)
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
    // pass 2: normaliser, exponentials staged in shared memory (ROW_STAGE at a time)
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
    // pass 3: normalise and histogram
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
        const bool valid = i < L;
        const float p = e[u] * inv;
        if (valid) row[i] = p;
        warp_hist_add(scnt, smass, valid, __float_as_uint(p) >> 20, to_fixed(p));
      }
    }
  }
  __syncthreads();
  flush_hist(scnt, smass, kHistBins, a.hist_cnt + (size_t)h * kHistBins, a.hist_mass + (size_t)h * kHistBins);
}

// --------------------------------------------------------------------- histogram, levels 2-3
// level 2: entries whose bits[30:20] match the prefix, bin = bits[19:10]
// level 3: entries whose bits[30:10] match the prefix, bin = bits[9:0]
// Matching values are spread over many bins: plain per-lane shared atomics.
__global__ void __launch_bounds__(256) cut_hist_kernel(const SelectArgs a, int level) {
  const int h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const CutState cs = a.cut[h];
  if (cs.keep_all) return;
  const Shape& s = a.s;
  __shared__ uint32_t scnt[1024];
  __shared__ unsigned long long smass[1024];
  for (int i = threadIdx.x; i < 1024; i += 256) {
    scnt[i] = 0;
    smass[i] = 0ull;
  }
  __syncthreads();
  const float4* P4 = reinterpret_cast<const float4*>(a.pbuf + (size_t)h * s.cap);
  const float* P = a.pbuf + (size_t)h * s.cap;
  const int shift = level == 2 ? 20 : 10;
  const int bshift = level == 2 ? 10 : 0;
  // the head's row-major array is 4-float aligned only when h*cap is; walk scalars otherwise
  const bool vec = ((s.cap & 3) == 0);
  const long long n4 = vec ? s.cap / 4 : 0;
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n4; i += (long long)gridDim.x * 256) {
    const float4 v = P4[i];
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t bits = __float_as_uint(vv[j]);
      if ((bits >> shift) == cs.prefix) {
        const uint32_t bin = (bits >> bshift) & 1023u;
        atomicAdd(&scnt[bin], 1u);
        atomicAdd(&smass[bin], to_fixed(vv[j]));
      }
    }
  }
  for (long long i = n4 * 4 + (long long)blockIdx.x * 256 + threadIdx.x; i < s.cap; i += (long long)gridDim.x * 256) {
    const uint32_t bits = __float_as_uint(P[i]);
    if ((bits >> shift) == cs.prefix) {
      const uint32_t bin = (bits >> bshift) & 1023u;
      atomicAdd(&scnt[bin], 1u);
      atomicAdd(&smass[bin], to_fixed(P[i]));
    }
  }
  __syncthreads();
  flush_hist(scnt, smass, 1024, a.hist_cnt + (size_t)h * kHistBins, a.hist_mass + (size_t)h * kHistBins);
}

// ------------------------------------------------------------------------- bin selection
// One CTA per head: walk the bins from the largest values down and find the bin where the
// cumulative mass (plus the mass already above the prefix) first reaches the target.
// Masses are summed exactly in fixed point; the target is rounded up to the same grid.
__global__ void __launch_bounds__(1024) cut_select_kernel(const SelectArgs a, int level) {
  const int h = blockIdx.x;
  const Shape& s = a.s;
  CutState* cs = a.cut + h;
  const int nbins = level == 1 ? kHistBins : 1024;
  uint32_t* gcnt = a.hist_cnt + (size_t)h * kHistBins;
  unsigned long long* gmass = a.hist_mass + (size_t)h * kHistBins;
  if (!is_pe(a, h)) return;
  if (level == 1 && threadIdx.x == 0) {
    cs->target = (double)a.gamma * (double)s.nb;
    cs->mass_above = 0.0;
    cs->prefix = 0;
    cs->keep_all = a.gamma >= 1.0f ? 1u : 0u;
  }
  __syncthreads();
  __shared__ unsigned long long suffix[kHistBins];
  __shared__ int found;
  if (!cs->keep_all) {
    for (int i = threadIdx.x; i < nbins; i += 1024) suffix[i] = gmass[i];
    __syncthreads();
    for (int off = 1; off < nbins; off <<= 1) {
      unsigned long long v[2];
      for (int k = 0; k < 2; ++k) {
        const int i = threadIdx.x + k * 1024;
        v[k] = (i < nbins && i + off < nbins) ? suffix[i + off] : 0ull;
      }
      __syncthreads();
      for (int k = 0; k < 2; ++k) {
        const int i = threadIdx.x + k * 1024;
        if (i < nbins) suffix[i] += v[k];
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) found = -1;
    __syncthreads();
    // suffix[i] = mass of bins >= i; the wanted bin b is the largest i with
    // above + suffix[i] >= target, i.e. the bins above b alone stay below the target.
    const unsigned long long above = __double2ull_rn(cs->mass_above * kMassUnit);
    const unsigned long long target = __double2ull_ru(cs->target * kMassUnit);
    for (int i = threadIdx.x; i < nbins; i += 1024) {
      const unsigned long long hi = (i + 1 < nbins) ? suffix[i + 1] : 0ull;
      if (above + suffix[i] >= target && above + hi < target && gcnt[i] > 0) atomicMax(&found, i);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const int b = found;
      if (b < 0) {
        cs->keep_all = 1;  // target not reachable: keep everything
      } else {
        const unsigned long long hi = (b + 1 < nbins) ? suffix[b + 1] : 0ull;
        cs->mass_above = (double)(above + hi) / kMassUnit;
        cs->prefix = (cs->prefix << (level == 1 ? 0 : 10)) | (uint32_t)b;
        if (level == 3) {
          const uint32_t bits = cs->prefix;
          const double val = (double)__uint_as_float(bits);
          const double rem = cs->target - cs->mass_above;
          uint32_t t = val > 0.0 ? (uint32_t)ceil(rem / val) : gcnt[b];
          if (t < 1) t = 1;
          if (t > gcnt[b]) t = gcnt[b];
          cs->thr_bits = bits;
          cs->t_eq = t;
          cs->count_eq = gcnt[b];
        }
      }
    }
  }
  __syncthreads();
  // clear the histogram for the next level
  for (int i = threadIdx.x; i < kHistBins; i += 1024) {
    gcnt[i] = 0;
    gmass[i] = 0ull;
  }
}

}  // namespace

cudaError_t launch_pe(const SelectArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  qbar_kernel<<<dim3(s.nb, s.h_q), 128, 0, st>>>(a);
  const int nt = (s.nb + TS - 1) / TS;
  scores_kernel<<<dim3(nt, nt, s.h_q), 256, 0, st>>>(a);
  rowsoft_kernel<<<dim3((s.nb + ROWS_PER_CTA - 1) / ROWS_PER_CTA, s.h_q), ROWS_PER_CTA * 32, 0, st>>>(a);
  cut_select_kernel<<<s.h_q, 1024, 0, st>>>(a, 1);
  const int hist_ctas = (int)std::min<long long>(512, (s.cap + 4095) / 4096);
  cut_hist_kernel<<<dim3(hist_ctas, s.h_q), 256, 0, st>>>(a, 2);
  cut_select_kernel<<<s.h_q, 1024, 0, st>>>(a, 2);
  cut_hist_kernel<<<dim3(hist_ctas, s.h_q), 256, 0, st>>>(a, 3);
  cut_select_kernel<<<s.h_q, 1024, 0, st>>>(a, 3);
  return cudaGetLastError();
}

}  // namespace crisp
