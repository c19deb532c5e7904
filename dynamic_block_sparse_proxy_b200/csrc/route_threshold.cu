// route_threshold.cu — per-head routing and the Vertical-Slash noise-floor rule.
//
// Inputs are the proxy pass's per-(row, key block) split sums, each relative to its chunk's
// reference row maximum. Row statistics (one CTA per head), then block masses over many CTAs per
// head, the head's last CTA taking the decisions:
//   1. per proxy row r: global max M_r and normaliser Z_r over all chunks, and the weight
//      w = exp2(m_chunk - M_r) / (Z_r * B) that turns a chunk's sums into column-mean mass;
//   2. p_v[kb] = sum_r w*(lo+hi) (vertical block mass), and the slash block masses
//      p_s[N_b-1-kb] += sum_r w*lo, p_s[N_b-2-kb] += sum_r w*hi (CRISP §4, both directions);
//   3. C_struct = p_v[0] + p_v[N_b-1], the mass on the first and last 128 keys (CRISP §3.2);
//      route = Vertical-Slash iff C_struct >= tau_proxy (or, with the FlexPrefill router the
//      CRISP paper compares against, iff JSD(a_bar, a_hat) >= tau_jsd);
//   4. per direction the noise floor mu = (mass of blocks 1..N_b-2) / (N_b-2). The block masses
//      add up to one, so this is max(1 - p[0] - p[N_b-1], 0) / (N_b-2) of CRISP §4 summed
//      without the cancellation that subtracting a near-one sink mass from 1 would cause;
//   5. keep block j in [1, N_b-2] iff p[j] > alpha*mu (strict), then top up to min_blocks with
//      the largest remaining blocks (ties to the lower index). Variants: mu as the median of
//      p[1..N_b-2]; or FlexPrefill's per-direction cut, the shortest (p desc, index asc) prefix
//      reaching gamma of the direction's mass.
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

// Block-wide maximum and sum of doubles (all threads receive the result).
__device__ double block_max(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double t = -INFINITY;
  for (int i = 0; i < NWARP; ++i) t = fmax(t, red[i]);
  return t;
}

// FlexPrefill's routing statistic (route_rule 1): JSD between a_bar, the softmax over all key
// blocks of the last query block's mean query against the key-block means (1/sqrt(d) scale),
// and a_hat, the proxy's per-query mean pooled to blocks (p_v, normalised to sum 1). Natural
// logarithm, 0 log 0 = 0. `abar` is scratch for N_b doubles; `qpart` stages the query mean.
__device__ double jsd_statistic(const SelectArgs& a, int h, const double* pv, double* abar, float* qm,
                                float (*qpart)[kD], double* red) {
  const Shape& s = a.s;
  const int nb = s.nb, tid = threadIdx.x, kv = h / s.G;
  // mean of the last 128 query rows; thread t sums column t%128 over rows t/128, t/128+4, ...
  {
    const int col = tid & (kD - 1), rg = tid >> 7;
    const __nv_bfloat16* qrow = a.q + ((size_t)h * s.ld + (size_t)(s.n - kB)) * kD + col;
    float acc = 0.f;
    for (int r = rg; r < kB; r += THREADS / kD) acc += __bfloat162float(qrow[(size_t)r * kD]);
    qpart[rg][col] = acc;
    __syncthreads();
    if (tid < kD) {
      float t = 0.f;
      for (int g = 0; g < THREADS / kD; ++g) t += qpart[g][tid];
      qm[tid] = t * (1.f / kB);
    }
    __syncthreads();
  }
  // logits and softmax over the key blocks
  const double inv_sqrt_d = 0.08838834764831845;
  double mx = -INFINITY;
  for (int kb = tid; kb < nb; kb += THREADS) {
    const float4* kr = reinterpret_cast<const float4*>(a.kbar + ((size_t)kv * nb + kb) * kD);
    double dot = 0.0;
#pragma unroll 4
    for (int i = 0; i < kD / 4; ++i) {
      const float4 kk = kr[i];
      dot += (double)qm[4 * i] * kk.x + (double)qm[4 * i + 1] * kk.y + (double)qm[4 * i + 2] * kk.z +
             (double)qm[4 * i + 3] * kk.w;
    }
    abar[kb] = dot * inv_sqrt_d;
    mx = fmax(mx, abar[kb]);
  }
  mx = block_max(mx, red);
  double z = 0.0, spv = 0.0;
  for (int kb = tid; kb < nb; kb += THREADS) {
    abar[kb] = exp(abar[kb] - mx);
    z += abar[kb];
    spv += pv[kb];
  }
  z = block_sum(z, red);
  spv = block_sum(spv, red);
  double t = 0.0;
  for (int kb = tid; kb < nb; kb += THREADS) {
    const double p = abar[kb] / z, q = pv[kb] / spv, m = 0.5 * (p + q);
    if (p > 0.0) t += p * log(p / m);
    if (q > 0.0) t += q * log(q / m);
  }
  return 0.5 * block_sum(t, red);
}

// Sorts the indices 0..P2-1 in sidx so that (p desc, index asc) order holds for the indices
// `member` accepts; all others go last. P2 is a power of two >= the number of indices.
template <typename Member>
__device__ void sort_desc(const double* p, int* sidx, int P2, Member member) {
  for (int i = threadIdx.x; i < P2; i += THREADS) sidx[i] = i;
  __syncthreads();
  auto before = [&](int x, int y) {  // x strictly before y
    const bool mx = member(x), my = member(y);
    if (mx != my) return mx;
    if (!mx) return x < y;
    return p[x] > p[y] || (p[x] == p[y] && x < y);
  };
  for (int k = 2; k <= P2; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P2; i += THREADS) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const int x = sidx[i], y = sidx[ixj];
          const bool asc = (i & k) == 0;  // this pair's sequence runs in the final order
          if (asc ? before(y, x) : before(x, y)) {
            sidx[i] = y;
            sidx[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
}

// FlexPrefill's per-direction cut (vs_rule 1): the shortest prefix of the blocks sorted
// (p desc, index asc) whose sum reaches gamma * sum(p); sets flags on its blocks in
// [1, N_b-2] and returns the value of the last block kept.
__device__ double gamma_direction(const double* p, int* sidx, int nb, int P2, double gamma, uint8_t* flags,
                                  double* red, int* pos_min) {
  sort_desc(p, sidx, P2, [nb](int x) { return x < nb; });
  double tot = 0.0;
  for (int i = threadIdx.x; i < nb; i += THREADS) tot += p[i];
  tot = block_sum(tot, red);
  const double target = gamma * tot;
  // per-thread contiguous segment of the sorted order, then a block exclusive scan of segments
  const int seg = (nb + THREADS - 1) / THREADS;
  const int b0 = threadIdx.x * seg, b1 = min(nb, b0 + seg);
  double local = 0.0;
  for (int i = b0; i < b1; ++i) local += p[sidx[i]];
  // exclusive scan over threads (warp shuffles, then warp totals)
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  double incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) red[w] = incl;
  if (threadIdx.x == 0) *pos_min = nb;
  __syncthreads();
  double base = incl - local;
  for (int i = 0; i < w; ++i) base += red[i];
  double c = base;
  for (int i = b0; i < b1; ++i) {
    c += p[sidx[i]];
    if (c >= target) {
      atomicMin(pos_min, i);
      break;
    }
  }
  __syncthreads();
  const int count = min(*pos_min + 1, nb);
  for (int i = threadIdx.x; i < nb; i += THREADS) {
    const int j = sidx[i];
    if (j >= 1 && j <= nb - 2) flags[j] = i < count ? 1 : 0;
  }
  const double cut = p[sidx[count - 1]];
  __syncthreads();
  return cut;
}

// The median of p[1..N_b-2] (mean of the two middle values for an even count).
__device__ double median_inner(const double* p, int* sidx, int nb, int P2) {
  sort_desc(p, sidx, P2, [nb](int x) { return x >= 1 && x <= nb - 2; });
  const int m = nb - 2;
  const double lo = p[sidx[(m - 1) / 2]], hi = p[sidx[m / 2]];
  const double med = 0.5 * (lo + hi);
  __syncthreads();
  return med;
}

// 3. Per head: C_struct (or the JSD), route, noise floors, keep flags (+ top-up). Run by the
//    last CTA of the head's block-mass kernel (every CTA of the head has written its masses).
__device__ void route_head(const SelectArgs& a, int h) {
  extern __shared__ double dsm[];
  const Shape& s = a.s;
  const int nb = s.nb, tid = threadIdx.x;
  double* pv = dsm;        // [nb]
  double* ps = dsm + nb;   // [nb]
  double* aux = dsm + 2 * nb;                  // [nb] doubles: a_bar, then sort indices
  int* sidx = reinterpret_cast<int*>(aux);     // [P2] ints (P2 <= 2 nb)
  __shared__ double red[NWARP];
  __shared__ double redv[NWARP];
  __shared__ int redi[NWARP];
  __shared__ float qm[kD];
  __shared__ float qpart[THREADS / kD][kD];
  __shared__ int pos_min;
  // written by the head's other CTAs: read through L2
  for (int i = tid; i < nb; i += THREADS) {
    pv[i] = __ldcg(a.pv + (size_t)h * nb + i);
    ps[i] = __ldcg(a.ps_lo + (size_t)h * nb + i) + __ldcg(a.ps_hi + (size_t)h * nb + i) +
            __ldcg(a.ps_x + (size_t)h * nb + i);
  }
  __syncthreads();

  // C_struct: mass on the first 128 keys and the last 128 keys. When n is a multiple of 128 these
  // are blocks 0 and N_b-1; otherwise the last 128 keys also cover block N_b-2's columns from
  // t_last on (collected per proxy row by the proxy pass). With N_b = 2 the windows overlap and
  // their union is every key.
  double C = nb >= 2 ? pv[0] + pv[nb - 1] : pv[0];
  const int t_last = s.n - (nb - 1) * kB;
  if (t_last != kB && nb >= 3) {
    // both 64-column halves of block N_b-2, each with its segment's weight
    double x = 0.0;
    for (int i = tid; i < 2 * kB; i += THREADS) {
      const int half = i / kB, r = i % kB;
      const float* wr = a.row_w + (((size_t)h * s.n_chunks + (nb - 2) / kProxyChunk) * 2 + half) * kB;
      x += (double)a.rec_extra[((size_t)h * 2 + half) * kB + r] * (double)__ldcg(wr + r);
    }
    C += block_sum(x, red);
  }
  double jsd = 0.0;
  int vs;
  if (a.route_rule == 1) {
    jsd = jsd_statistic(a, h, pv, aux, qm, qpart, red);
    vs = jsd >= (double)a.tau_jsd ? 1 : 0;
  } else {
    vs = C >= (double)a.tau ? 1 : 0;
  }
  __syncthreads();

  // keep flags per direction
  uint8_t* kv_out = a.keep_v + (size_t)h * nb;
  uint8_t* ks_out = a.keep_s + (size_t)h * nb;
  const double alpha = (double)a.alpha;
  int P2 = 1;
  while (P2 < nb) P2 <<= 1;
  double mu_out[2] = {0.0, 0.0};
  int nkeep[2] = {0, 0};
  for (int dir = 0; dir < 2; ++dir) {
    const double* p = dir == 0 ? pv : ps;
    uint8_t* flags = dir == 0 ? kv_out : ks_out;
    for (int j = tid; j < nb; j += THREADS) flags[j] = 0;
    __syncthreads();
    if (nb >= 3) {
      if (a.vs_rule == 1) {
        if (vs) mu_out[dir] = gamma_direction(p, sidx, nb, P2, (double)a.gamma, flags, red, &pos_min);
      } else {
        double mu;
        if (a.floor_rule == 1) {
          mu = median_inner(p, sidx, nb, P2);
        } else {
          // mean residual mass of blocks 1..N_b-2: their sum, without subtracting from 1
          double r = 0.0;
          for (int j = 1 + tid; j <= nb - 2; j += THREADS) r += p[j];
          mu = block_sum(r, red) / (nb - 2);
        }
        mu_out[dir] = mu;
        for (int j = 1 + tid; j <= nb - 2; j += THREADS) flags[j] = p[j] > alpha * mu ? 1 : 0;
      }
    }
    __syncthreads();
    int cnt = 0;
    for (int j = tid; j < nb; j += THREADS) cnt += flags[j];
    nkeep[dir] = (int)block_sum((double)cnt, red);
  }

  // top-up to min_blocks (both rules)
  if (vs && nb >= 3 && a.min_blocks > 0) {
    __syncthreads();
    for (int dir = 0; dir < 2; ++dir) {
      uint8_t* flags = dir == 0 ? kv_out : ks_out;
      const double* p = dir == 0 ? pv : ps;
      int have = nkeep[dir];
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
    float* dbg = a.debug + (size_t)h * (2 * nb + 5);
    for (int j = tid; j < nb; j += THREADS) {
      dbg[j] = (float)pv[j];
      dbg[nb + j] = (float)ps[j];
    }
    if (tid == 0) {
      dbg[2 * nb] = (float)mu_out[0];
      dbg[2 * nb + 1] = (float)mu_out[1];
      dbg[2 * nb + 2] = (float)C;
      dbg[2 * nb + 4] = (float)jsd;
    }
  }
}

// 1-2. One CTA per run of MASS_BLOCKS key blocks of a head:
//   (a) per proxy row r: the global reference max M_r over the segments (the proxy pass keeps
//       one reference per chunk and 64-column half), the normaliser Z_r, and for the CTA's
//       segments the weight w = exp2(m_seg - M_r) / (Z_r * B) that turns a segment's sums into
//       column-mean mass (four threads per row, fp64 sums);
//   (b) block masses, one warp per key block: p_v[kb] = sum_r sum_half w*(lo+hi). A row r whose split
//       column is (t_last + r) mod 128 (t_last = n - 128 (N_b-1), 128 when n is a multiple of
//       128) meets slash blocks N_b-1-kb (lo) and N_b-2-kb (hi) when t_last + r >= 128, else
//       N_b-2-kb (lo) and N_b-3-kb (hi) (CRISP §4, both directions). Every slot of ps_lo, ps_hi
//       and ps_x is written once: by the key block that maps there, or with 0 by the block whose
//       target lies below 0;
//   (c) the head's last CTA to finish routes the head (route_head).
// 1. Per proxy row r: the global reference max M_r over the segments (the proxy pass keeps one
//    reference per chunk and 64-column half), the normaliser Z_r (fp64), and for every segment
//    the weight w = exp2(m_seg - M_r) / (Z_r * B) that turns the segment's sums into column-mean
//    mass. One CTA per (32 rows, head); thread (part, row) takes segments part, part+16, ..., all
//    of its loads in flight before the first use.
constexpr int STAT_ROWS = 32;
constexpr int STAT_PARTS = THREADS / STAT_ROWS;  // 16
constexpr int STAT_UNROLL = 8;
__global__ void __launch_bounds__(THREADS) row_stats_kernel(const SelectArgs a) {
  const Shape& s = a.s;
  const int h = blockIdx.y, tid = threadIdx.x;
  const int r = blockIdx.x * STAT_ROWS + (tid % STAT_ROWS), part = tid / STAT_ROWS;
  const int nseg = 2 * s.n_chunks;
  const float* mc = a.chunk_max + (size_t)h * nseg * kB + r;
  const float* tc = a.chunk_tot + (size_t)h * nseg * kB + r;
  __shared__ float smax[STAT_PARTS][STAT_ROWS];
  __shared__ double ssum[STAT_PARTS][STAT_ROWS];
  float M = -INFINITY;
  for (int g0 = part; g0 < nseg; g0 += STAT_PARTS * STAT_UNROLL) {
    float x[STAT_UNROLL];
#pragma unroll
    for (int u = 0; u < STAT_UNROLL; ++u) {
      const int g = g0 + STAT_PARTS * u;
      x[u] = g < nseg ? mc[(size_t)g * kB] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < STAT_UNROLL; ++u) M = fmaxf(M, x[u]);
  }
  smax[part][tid % STAT_ROWS] = M;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < STAT_PARTS; ++i) M = fmaxf(M, smax[i][tid % STAT_ROWS]);
  double Z = 0.0;
  for (int g0 = part; g0 < nseg; g0 += STAT_PARTS * STAT_UNROLL) {
    float x[STAT_UNROLL], y[STAT_UNROLL];
#pragma unroll
    for (int u = 0; u < STAT_UNROLL; ++u) {
      const int g = g0 + STAT_PARTS * u;
      x[u] = g < nseg ? mc[(size_t)g * kB] : -INFINITY;
      y[u] = g < nseg ? tc[(size_t)g * kB] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < STAT_UNROLL; ++u)
      if (g0 + STAT_PARTS * u < nseg) Z += (double)exp2f(x[u] - M) * (double)y[u];
  }
  ssum[part][tid % STAT_ROWS] = Z;
  __syncthreads();
  Z = 0.0;
#pragma unroll
  for (int i = 0; i < STAT_PARTS; ++i) Z += ssum[i][tid % STAT_ROWS];
  const double inv = 1.0 / (Z * kB);
  float* wr = a.row_w + (size_t)h * nseg * kB + r;
  for (int g = part; g < nseg; g += STAT_PARTS) wr[(size_t)g * kB] = (float)((double)exp2f(mc[(size_t)g * kB] - M) * inv);
}

// 2-3. One CTA per run of MASS_BLOCKS key blocks of a head:
//   (a) block masses, one warp per key block: p_v[kb] = sum_r sum_half w*(lo+hi). A row r whose
//       split column is (t_last + r) mod 128 (t_last = n - 128 (N_b-1), 128 when n is a multiple
//       of 128) meets slash blocks N_b-1-kb (lo) and N_b-2-kb (hi) when t_last + r >= 128, else
//       N_b-2-kb (lo) and N_b-3-kb (hi) (CRISP §4, both directions). Every slot of ps_lo, ps_hi
//       and ps_x is written once: by the key block that maps there, or with 0 by the block whose
//       target lies below 0;
//   (b) the head's last CTA to finish routes the head (route_head).
constexpr int MASS_BLOCKS = 64;                     // key blocks per CTA
constexpr int MASS_CHUNKS = MASS_BLOCKS / kProxyChunk;
__global__ void __launch_bounds__(THREADS) mass_route_kernel(const SelectArgs a) {
  const Shape& s = a.s;
  const int h = blockIdx.y, nb = s.nb, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kb0 = blockIdx.x * MASS_BLOCKS;
  const int c0 = kb0 / kProxyChunk, c1 = min(s.n_chunks, c0 + MASS_CHUNKS);
  const int nseg = 2 * s.n_chunks;
  __shared__ float w_s[2 * MASS_CHUNKS][kB];
  for (int i = tid; i < 2 * (c1 - c0) * kB; i += THREADS)
    w_s[i / kB][i % kB] = a.row_w[((size_t)h * nseg + 2 * c0) * kB + i];
  __syncthreads();
  const int t_last = s.n - (nb - 1) * kB;
  for (int kb = kb0 + warp; kb < min(nb, kb0 + MASS_BLOCKS); kb += NWARP) {
    const float2* v = a.part + (size_t)(h * nb + kb) * 2 * kB + lane;  // [half][128], this lane's rows
    const float* wc = w_s[2 * (kb / kProxyChunk - c0)];         // [half][128]
    double loA = 0.0, hiA = 0.0, loB = 0.0, hiB = 0.0;
    float2 vv[2 * kB / 32];
#pragma unroll
    for (int i = 0; i < 2 * kB / 32; ++i) vv[i] = v[32 * i];
#pragma unroll
    for (int i = 0; i < 2 * kB / 32; ++i) {
      const int r = (lane + 32 * i) & (kB - 1);
      const double ww = wc[lane + 32 * i];
      if (t_last + r >= kB) {
        loA += (double)vv[i].x * ww;
        hiA += (double)vv[i].y * ww;
      } else {
        loB += (double)vv[i].x * ww;
        hiB += (double)vv[i].y * ww;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      loA += __shfl_xor_sync(0xffffffffu, loA, o);
      hiA += __shfl_xor_sync(0xffffffffu, hiA, o);
      loB += __shfl_xor_sync(0xffffffffu, loB, o);
      hiB += __shfl_xor_sync(0xffffffffu, hiB, o);
    }
    if (lane == 0) {
      const size_t base = (size_t)h * nb;
      a.pv[base + kb] = (loA + hiA) + (loB + hiB);
      a.ps_lo[base + nb - 1 - kb] = loA;
      if (nb - 2 - kb >= 0) a.ps_hi[base + nb - 2 - kb] = hiA + loB;
      else a.ps_hi[base + nb - 1] = 0.0;  // kb = N_b-1: the slot no block maps to
      if (nb - 3 - kb >= 0) a.ps_x[base + nb - 3 - kb] = hiB;
      else a.ps_x[base + (nb - 3 - kb == -1 ? nb - 2 : nb - 1)] = 0.0;  // kb = N_b-2, N_b-1
    }
  }
  // the head's last CTA routes it (counter back to zero for the radix levels that reuse it)
  __threadfence();
  __syncthreads();
  __shared__ int last;
  if (tid == 0) last = atomicAdd(a.cut_done + h, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (tid == 0) a.cut_done[h] = 0;
  route_head(a, h);
}

}  // namespace

cudaError_t launch_route_threshold(const SelectArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)3 * a.s.nb * sizeof(double);  // p_v, p_s, and a_bar / sort indices
  cudaError_t e = cudaFuncSetAttribute(mass_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  row_stats_kernel<<<dim3(kB / STAT_ROWS, a.s.h_q), THREADS, 0, st>>>(a);
  mass_route_kernel<<<dim3((a.s.nb + MASS_BLOCKS - 1) / MASS_BLOCKS, a.s.h_q), THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace crisp
