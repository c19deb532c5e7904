// pe_cut.cu — the Pooled-Estimation path of CRISP (paper §2 and §4: pooled query and key
// blocks, softmax, then the flattened gamma cumulative cut; the rcap.io summary's per-head
// pseudocode: gamma_cumsum(pool(Q), pool(K), gamma)).
//
// For every head routed to PE:
//   qbar_kernel     Q_bar[qb] = mean of the block's 128 query rows (fp32), read once from HBM;
//   scores_kernel   logits Q_bar[qb] . K_bar[kb] / sqrt(d) for kb <= qb (64x64 fp32 tiles);
//   rowsoft_kernel  P[qb, kb] = softmax over kb <= qb, in place, plus the first radix histogram;
//   cut_select / cut_hist: an exact radix select (11 + 10 + 10 bits of the positive fp32
//                   pattern, count and fp64 mass per bin) of the value T where the mass of the
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
  const __nv_bfloat16* base = a.q + ((size_t)h * s.n + (size_t)qb * kB) * kD + c16 * 8;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int row = rg + 8 * i;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(base + (size_t)row * kD));
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
  a.qbar[((size_t)h * s.nb + qb) * kD + t] = v * (1.f / kB);
}

// -------------------------------------------------------------------------------- logits
constexpr int TS = 64;
__global__ void __launch_bounds__(256) scores_kernel(const SelectArgs a) {
  const int tk = blockIdx.x, tq = blockIdx.y, h = blockIdx.z;
  if (tk > tq || !is_pe(a, h)) return;
  const Shape& s = a.s;
  const int kv = h / s.G;
  extern __shared__ float fsm[];
  float* qs = fsm;               // [TS][kD+1]
  float* ks = fsm + TS * (kD + 1);
  const int q0 = tq * TS, k0 = tk * TS;
  for (int i = threadIdx.x; i < TS * kD; i += 256) {
    const int r = i / kD, c = i % kD;
    qs[r * (kD + 1) + c] = (q0 + r < s.nb) ? a.qbar[((size_t)h * s.nb + q0 + r) * kD + c] : 0.f;
    ks[r * (kD + 1) + c] = (k0 + r < s.nb) ? a.kbar[((size_t)kv * s.nb + k0 + r) * kD + c] : 0.f;
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float acc[4][4] = {};
  for (int c = 0; c < kD; ++c) {
    float qv[4], kv4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qv[i] = qs[(ty + 16 * i) * (kD + 1) + c];
      kv4[i] = ks[(tx + 16 * i) * (kD + 1) + c];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv4[j], acc[i][j]);
  }
  const float inv_sqrt_d = 0.08838834764831845f;
  float* P = a.pbuf + (size_t)h * s.cap;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qb = q0 + ty + 16 * i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int kb = k0 + tx + 16 * j;
      if (qb < s.nb && kb <= qb) P[(size_t)qb * (qb + 1) / 2 + kb] = acc[i][j] * inv_sqrt_d;
    }
  }
}

// ----------------------------------------------------------------- row softmax + histogram 1
// Warp-aggregated histogram update: lanes with the same bin are summed first, so a row whose
// values share one bin costs one shared atomic per warp instead of 32. All lanes must call it.
__device__ __forceinline__ void warp_hist_add(uint32_t* scnt, double* smass, bool valid, uint32_t bin,
                                              float p) {
  const int lane = threadIdx.x & 31;
  unsigned todo = __ballot_sync(0xffffffffu, valid);
  while (todo) {
    const int leader = __ffs(todo) - 1;
    const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
    const bool mine = ((todo >> lane) & 1u) && bin == lb;
    const unsigned grp = __ballot_sync(0xffffffffu, mine);
    double v = mine ? (double)p : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == leader) {
      atomicAdd(&scnt[lb], (uint32_t)__popc(grp));
      atomicAdd(&smass[lb], v);
    }
    todo &= ~grp;
  }
}

__device__ __forceinline__ void flush_hist(uint32_t* scnt, double* smass, int nbins, uint32_t* gcnt,
                                           double* gmass) {
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) {
    if (scnt[i]) {
      atomicAdd(gcnt + i, scnt[i]);
      atomicAdd(gmass + i, smass[i]);
    }
  }
}

__global__ void __launch_bounds__(256) rowsoft_kernel(const SelectArgs a) {
  const int qb = blockIdx.x, h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const Shape& s = a.s;
  __shared__ uint32_t scnt[kHistBins];
  __shared__ double smass[kHistBins];
  __shared__ float red[8];
  for (int i = threadIdx.x; i < kHistBins; i += 256) {
    scnt[i] = 0;
    smass[i] = 0.0;
  }
  __syncthreads();
  float* row = a.pbuf + (size_t)h * s.cap + (size_t)qb * (qb + 1) / 2;
  const int L = qb + 1, tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  float mx = -INFINITY;
  for (int i = tid; i < L; i += 256) mx = fmaxf(mx, row[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (l == 0) red[w] = mx;
  __syncthreads();
  mx = red[0];
  for (int i = 1; i < 8; ++i) mx = fmaxf(mx, red[i]);
  __syncthreads();
  float z = 0.f;
  for (int i = tid; i < L; i += 256) z += expf(row[i] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (l == 0) red[w] = z;
  __syncthreads();
  z = 0.f;
  for (int i = 0; i < 8; ++i) z += red[i];
  const float inv = 1.f / z;
  for (int base = 0; base < L; base += 256) {
    const int i = base + tid;
    const bool valid = i < L;
    float p = 0.f;
    if (valid) {
      p = expf(row[i] - mx) * inv;
      row[i] = p;
    }
    warp_hist_add(scnt, smass, valid, __float_as_uint(p) >> 20, p);
  }
  __syncthreads();
  flush_hist(scnt, smass, kHistBins, a.hist_cnt + (size_t)h * kHistBins, a.hist_mass + (size_t)h * kHistBins);
}

// --------------------------------------------------------------------- histogram, levels 2-3
// level 2: entries whose bits[30:20] match the prefix, bin = bits[19:10]
// level 3: entries whose bits[30:10] match the prefix, bin = bits[9:0]
__global__ void __launch_bounds__(256) cut_hist_kernel(const SelectArgs a, int level) {
  const int h = blockIdx.y;
  if (!is_pe(a, h)) return;
  const CutState cs = a.cut[h];
  if (cs.keep_all) return;
  const Shape& s = a.s;
  __shared__ uint32_t scnt[1024];
  __shared__ double smass[1024];
  for (int i = threadIdx.x; i < 1024; i += 256) {
    scnt[i] = 0;
    smass[i] = 0.0;
  }
  __syncthreads();
  const float* P = a.pbuf + (size_t)h * s.cap;
  const int shift = level == 2 ? 20 : 10;
  const int bshift = level == 2 ? 10 : 0;
  const long long per_cta = (s.cap + gridDim.x - 1) / gridDim.x;
  const long long beg = (long long)blockIdx.x * per_cta;
  const long long end = min(s.cap, beg + per_cta);
  for (long long b0 = beg; b0 < end; b0 += 256) {
    const long long i = b0 + threadIdx.x;
    const uint32_t bits = i < end ? __float_as_uint(P[i]) : 0xffffffffu;
    const bool valid = i < end && (bits >> shift) == cs.prefix;
    warp_hist_add(scnt, smass, valid, (bits >> bshift) & 1023u, __uint_as_float(bits));
  }
  __syncthreads();
  flush_hist(scnt, smass, 1024, a.hist_cnt + (size_t)h * kHistBins, a.hist_mass + (size_t)h * kHistBins);
}

// ------------------------------------------------------------------------- bin selection
// One CTA per head: walk the bins from the largest values down and find the bin where the
// cumulative mass (plus the mass already above the prefix) first reaches the target.
__global__ void __launch_bounds__(1024) cut_select_kernel(const SelectArgs a, int level) {
  const int h = blockIdx.x;
  const Shape& s = a.s;
  CutState* cs = a.cut + h;
  const int nbins = level == 1 ? kHistBins : 1024;
  uint32_t* gcnt = a.hist_cnt + (size_t)h * kHistBins;
  double* gmass = a.hist_mass + (size_t)h * kHistBins;
  if (!is_pe(a, h)) return;
  if (level == 1 && threadIdx.x == 0) {
    cs->target = (double)a.gamma * (double)s.nb;
    cs->mass_above = 0.0;
    cs->prefix = 0;
    cs->keep_all = a.gamma >= 1.0f ? 1u : 0u;
  }
  __syncthreads();
  __shared__ double suffix[kHistBins];
  __shared__ int found;
  if (!cs->keep_all) {
    // suffix sums of the mass from the top bin down (Hillis-Steele over <= 2048 entries)
    for (int i = threadIdx.x; i < nbins; i += 1024) suffix[i] = gmass[i];
    __syncthreads();
    for (int off = 1; off < nbins; off <<= 1) {
      double v[2];
      for (int k = 0; k < 2; ++k) {
        const int i = threadIdx.x + k * 1024;
        v[k] = (i < nbins && i + off < nbins) ? suffix[i + off] : 0.0;
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
    // mass_above + suffix[i] >= target, i.e. bins above b stay below the target.
    const double need = cs->target - cs->mass_above;
    for (int i = threadIdx.x; i < nbins; i += 1024) {
      const double above = (i + 1 < nbins) ? suffix[i + 1] : 0.0;
      if (suffix[i] >= need && above < need && gcnt[i] > 0) atomicMax(&found, i);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const int b = found;
      if (b < 0) {
        cs->keep_all = 1;  // target not reachable in fp arithmetic: keep everything
      } else {
        cs->mass_above += (b + 1 < nbins) ? suffix[b + 1] : 0.0;
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
    gmass[i] = 0.0;
  }
}

}  // namespace

cudaError_t launch_pe(const SelectArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  cudaError_t e;
  qbar_kernel<<<dim3(s.nb, s.h_q), 128, 0, st>>>(a);
  const int nt = (s.nb + TS - 1) / TS;
  const size_t ssm = (size_t)2 * TS * (kD + 1) * sizeof(float);
  e = cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm);
  if (e != cudaSuccess) return e;
  scores_kernel<<<dim3(nt, nt, s.h_q), 256, ssm, st>>>(a);
  rowsoft_kernel<<<dim3(s.nb, s.h_q), 256, 0, st>>>(a);
  cut_select_kernel<<<s.h_q, 1024, 0, st>>>(a, 1);
  const int hist_ctas = (int)std::min<long long>(1024, (s.cap + 8191) / 8192);
  cut_hist_kernel<<<dim3(hist_ctas, s.h_q), 256, 0, st>>>(a, 2);
  cut_select_kernel<<<s.h_q, 1024, 0, st>>>(a, 2);
  cut_hist_kernel<<<dim3(hist_ctas, s.h_q), 256, 0, st>>>(a, 3);
  cut_select_kernel<<<s.h_q, 1024, 0, st>>>(a, 3);
  return cudaGetLastError();
}

}  // namespace crisp
