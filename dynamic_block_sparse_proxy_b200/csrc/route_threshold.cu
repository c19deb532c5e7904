// route_threshold.cu — per-head routing and the Vertical-Slash noise-floor rule.
//
// Inputs are the proxy pass's per-(row, key block) split sums, each relative to its chunk's
// reference row maximum. Three kernels (row statistics, block masses over many CTAs, and one
// CTA per q-head for the decisions):
//   1. per proxy row r: global max M_r and normaliser Z_r over all chunks, and the weight
//      w = exp2(m_chunk - M_r) / (Z_r * B) that turns a chunk's sums into column-mean mass;
//   2. p_v[kb] = sum_r w*(lo+hi) (vertical block mass), and the slash block masses
//      p_s[N_b-1-kb] += sum_r w*lo, p_s[N_b-2-kb] += sum_r w*hi (CRISP §4, both directions);
//   3. C_struct = p_v[0] + p_v[N_b-1], the mass on the first and last 128 keys (CRISP §3.2);
//      route = Vertical-Slash iff C_struct >= tau_proxy;
//   4. per direction the noise floor mu = (mass of blocks 1..N_b-2) / (N_b-2). The block masses
//      add up to one, so this is max(1 - p[0] - p[N_b-1], 0) / (N_b-2) of CRISP §4 summed
//      without the cancellation that subtracting a near-one sink mass from 1 would cause;
//   5. keep block j in [1, N_b-2] iff p[j] > alpha*mu (strict), then top up to min_blocks with
//      the largest remaining blocks (ties to the lower index).
// Reductions run in fp64.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

constexpr int THREADS = 512;
constexpr int NWARP = THREADS / 32;

__device__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
  for (int i = 0; i < NWARP; ++i) t += red[i];
  return t;
}

// Block-wide argmax of (value, -index) over candidates; returns the index or -1.
__device__ int block_argmax(double v, int idx, double* redv, int* redi) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (oi >= 0 && (idx < 0 || ov > v || (ov == v && oi < idx))) {
      v = ov;
      idx = oi;
    }
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) {
    redv[w] = v;
    redi[w] = idx;
  }
  __syncthreads();
  double bv = 0.0;
  int bi = -1;
  for (int i = 0; i < NWARP; ++i) {
    if (redi[i] >= 0 && (bi < 0 || redv[i] > bv || (redv[i] == bv && redi[i] < bi))) {
      bv = redv[i];
      bi = redi[i];
    }
  }
  return bi;
}

// 1. Per proxy row r of head h: global reference max M_r over the chunks, normaliser Z_r, and
//    the weight w = exp2(m_chunk - M_r) / (Z_r * B) that turns a chunk's sums into column-mean mass.
//    One warp per row, its lanes across the chunks.
constexpr int STAT_ROWS = 8;
__global__ void __launch_bounds__(STAT_ROWS * 32) row_stats_kernel(const SelectArgs a) {
  const Shape& s = a.s;
  const int h = blockIdx.y, r = blockIdx.x * STAT_ROWS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const float* mc = a.chunk_max + (size_t)h * s.n_chunks * kB;
  const float* tc = a.chunk_tot + (size_t)h * s.n_chunks * kB;
  float M = -INFINITY;
  for (int c = lane; c < s.n_chunks; c += 32) M = fmaxf(M, mc[c * kB + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  double Z = 0.0;
  for (int c = lane; c < s.n_chunks; c += 32) Z += (double)exp2f(mc[c * kB + r] - M) * (double)tc[c * kB + r];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
  float* w = a.row_w + (size_t)h * s.n_chunks * kB;
  const double inv = 1.0 / (Z * kB);
  for (int c = lane; c < s.n_chunks; c += 32) w[c * kB + r] = (float)((double)exp2f(mc[c * kB + r] - M) * inv);
}

// 2. Block masses, one warp per key block: p_v[kb] = sum_r w*(lo+hi); the lower-offset halves
//    belong to slash block N_b-1-kb and the upper ones to N_b-2-kb (CRISP §4, both directions).
constexpr int MASS_WARPS = 16;
__global__ void __launch_bounds__(MASS_WARPS * 32) block_mass_kernel(const SelectArgs a) {
  const Shape& s = a.s;
  const int h = blockIdx.y, nb = s.nb;
  const int kb = blockIdx.x * MASS_WARPS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (kb >= nb) return;
  const float2* p = a.part + ((size_t)h * nb + kb) * kB;
  const float* wc = a.row_w + ((size_t)h * s.n_chunks + kb / kProxyChunk) * kB;
  double lo = 0.0, hi = 0.0;
#pragma unroll
  for (int i = 0; i < kB / 32; ++i) {
    const int r = lane + 32 * i;
    const float2 v = p[r];
    const double ww = wc[r];
    lo += (double)v.x * ww;
    hi += (double)v.y * ww;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo += __shfl_xor_sync(0xffffffffu, lo, o);
    hi += __shfl_xor_sync(0xffffffffu, hi, o);
  }
  if (lane == 0) {
    a.pv[(size_t)h * nb + kb] = lo + hi;
    a.ps_lo[(size_t)h * nb + nb - 1 - kb] = lo;
    a.ps_hi[(size_t)h * nb + (nb - 2 - kb >= 0 ? nb - 2 - kb : nb - 1)] = nb - 2 - kb >= 0 ? hi : 0.0;
  }
}

// 3. Per head: C_struct, route, noise floors, keep flags (+ top-up).
__global__ void __launch_bounds__(THREADS) route_threshold_kernel(const SelectArgs a) {
  extern __shared__ double dsm[];
  const Shape& s = a.s;
  const int nb = s.nb, h = blockIdx.x, tid = threadIdx.x;
  double* pv = dsm;       // [nb]
  double* ps = dsm + nb;  // [nb]
  __shared__ double red[NWARP];
  __shared__ double redv[NWARP];
  __shared__ int redi[NWARP];
  for (int i = tid; i < nb; i += THREADS) {
    pv[i] = a.pv[(size_t)h * nb + i];
    ps[i] = a.ps_lo[(size_t)h * nb + i] + (i == nb - 1 ? 0.0 : a.ps_hi[(size_t)h * nb + i]);
  }
  __syncthreads();

  // C_struct and route
  const double C = nb >= 2 ? pv[0] + pv[nb - 1] : pv[0];
  const int vs = C >= (double)a.tau ? 1 : 0;

  // noise floors
  double mu_v = 0.0, mu_s = 0.0;
  if (nb >= 3) {
    double rv = 0.0, rs = 0.0;
    for (int j = 1 + tid; j <= nb - 2; j += THREADS) {
      rv += pv[j];
      rs += ps[j];
    }
    rv = block_sum(rv, red);
    rs = block_sum(rs, red);
    mu_v = rv / (nb - 2);
    mu_s = rs / (nb - 2);
  }

  // keep flags (+ top-up)
  uint8_t* kv_out = a.keep_v + (size_t)h * nb;
  uint8_t* ks_out = a.keep_s + (size_t)h * nb;
  const double alpha = (double)a.alpha;
  int nv = 0, ns = 0;
  for (int j = tid; j < nb; j += THREADS) {
    const bool inner = nb >= 3 && j >= 1 && j <= nb - 2;
    const uint8_t fv = inner && pv[j] > alpha * mu_v;
    const uint8_t fs = inner && ps[j] > alpha * mu_s;
    kv_out[j] = fv;
    ks_out[j] = fs;
    nv += fv;
    ns += fs;
  }
  nv = (int)block_sum((double)nv, red);
  ns = (int)block_sum((double)ns, red);
  if (vs && nb >= 3 && a.min_blocks > 0) {
    __syncthreads();
    for (int dir = 0; dir < 2; ++dir) {
      uint8_t* flags = dir == 0 ? kv_out : ks_out;
      const double* p = dir == 0 ? pv : ps;
      int have = dir == 0 ? nv : ns;
      const int want = min(a.min_blocks, nb - 2);
      while (have < want) {
        double bv = 0.0;
        int bi = -1;
        for (int j = 1 + tid; j <= nb - 2; j += THREADS) {
          if (!flags[j] && (bi < 0 || p[j] > bv)) {  // ascending j: ties keep the lower index
            bv = p[j];
            bi = j;
          }
        }
        const int pick = block_argmax(bv, bi, redv, redi);
        if (pick < 0) break;
        if (tid == 0) flags[pick] = 1;
        __syncthreads();
        ++have;
      }
    }
  }

  if (tid == 0) {
    a.route[h] = vs;
    a.c_struct[h] = (float)C;
  }
  if (a.debug != nullptr) {
    float* dbg = a.debug + (size_t)h * (2 * nb + 4);
    for (int j = tid; j < nb; j += THREADS) {
      dbg[j] = (float)pv[j];
      dbg[nb + j] = (float)ps[j];
    }
    if (tid == 0) {
      dbg[2 * nb] = (float)mu_v;
      dbg[2 * nb + 1] = (float)mu_s;
      dbg[2 * nb + 2] = (float)C;
    }
  }
}

}  // namespace

cudaError_t launch_route_threshold(const SelectArgs& a, cudaStream_t st) {
  row_stats_kernel<<<dim3(kB / STAT_ROWS, a.s.h_q), STAT_ROWS * 32, 0, st>>>(a);
  block_mass_kernel<<<dim3((a.s.nb + MASS_WARPS - 1) / MASS_WARPS, a.s.h_q), MASS_WARPS * 32, 0, st>>>(a);
  const size_t smem = (size_t)2 * a.s.nb * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(route_threshold_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  route_threshold_kernel<<<a.s.h_q, THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace crisp
