// merge.cu — per-query-block key-block lists (CSR) from the routing decisions.
//
// Vertical-Slash head, query block qb (CRISP §4: both directions thresholded separately and
// unioned; the first and last blocks always retained): key block kb <= qb is selected iff
//   kb == 0, or kb is a kept vertical block (or the last block), or a kept slash offset block m
//   (or the anchor offsets 0 and N_b-1) satisfies m == qb-kb or m == qb-kb-1.
// A query in block qb and a key at token offset o in [mB, mB+B) meet in key block qb-m or
// qb-m-1, so selecting both covers every token of a kept diagonal band.
// Pooled-Estimation head: (qb, kb) is selected iff its pooled score lies above the cut value T,
// or equals T and is among the first t_eq such entries in (qb, kb) order, or kb is one of the
// anchors {0, qb-1, qb}. With N_b <= 2 every causal block is selected.
//
// Three kernels:
//   merge_mask   one warp per row: the row's selection bitmask (32 key blocks per word), its
//                count, and, when more than one entry of the head equals the cut value, the
//                row's tied entries (all, and those that are not anchors);
//   merge_scan   one CTA per head: the CSR offsets from the counts (tied entries taken in
//                (qb, kb) order up to the quota);
//   merge_write  one warp per row: the column indices, expanded from the bitmask one word per
//                warp step.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

struct RowCtx {
  int qb;
  const float* P;
  uint32_t thr;
  uint32_t keep_all;
};

// PE: where an entry stands relative to the cut value: 0 below, 1 above, 2 equal. Anchors do not
// change this: the cut is taken over every entry, and the anchors are added on top.
__device__ __forceinline__ int pe_flag_of(const RowCtx& c, float p) {
  if (c.keep_all) return 1;
  const uint32_t bits = __float_as_uint(p);
  if (bits > c.thr) return 1;
  return bits == c.thr ? 2 : 0;
}

__device__ __forceinline__ bool pe_anchor(const RowCtx& c, int kb) {
  return kb == 0 || kb == c.qb || kb == c.qb - 1;
}

__device__ __forceinline__ RowCtx make_ctx(const SelectArgs& a, int h, int qb) {
  RowCtx c;
  const Shape& s = a.s;
  c.qb = qb;
  c.P = a.pbuf + (size_t)h * s.cap + (size_t)qb * (qb + 1) / 2;
  const CutState cs = a.cut[h];
  c.thr = cs.thr_bits;
  c.keep_all = (s.nb <= 2 || a.route[h] != 0) ? 1u : cs.keep_all;
  return c;
}

// Tied entries need ranking only when the head has more than one of them (a single tie is
// always kept: the quota t_eq is at least 1).
__device__ __forceinline__ bool head_ranks_ties(const SelectArgs& a, int h) {
  return a.route[h] == 0 && a.s.nb > 2 && !a.cut[h].keep_all && a.cut[h].count_eq > 1;
}

constexpr int ROWS = 8;  // rows (warps) per merge_mask CTA

// A Vertical-Slash head's selection as bitmasks (staged in shared memory, 32 key blocks per
// word): V holds the kept vertical blocks and the anchors 0 and N_b-1; R holds the kept slash
// offset blocks and the anchor offsets 0 and N_b-1, reversed (bit x of R is offset N_b-1-x).
// Row qb then selects kb iff V[kb], or offset qb-kb or qb-kb-1 is kept, i.e. R[kb + N_b-1-qb] or
// R[kb + N_b-qb]: a row's word is V's word or two funnel-shifted words of R.
__device__ void stage_vs_masks(const SelectArgs& a, int h, uint32_t* V, uint32_t* R, int words) {
  const int nb = a.s.nb, lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const uint8_t* gv = a.keep_v + (size_t)h * nb;
  const uint8_t* gs = a.keep_s + (size_t)h * nb;
  for (int w = warp; w < words; w += nwarp) {
    const int j = w * 32 + lane;
    const bool v = j < nb && (gv[j] != 0 || j == 0 || j == nb - 1);
    const int m = nb - 1 - j;  // bit j of R is offset m
    const bool r = j < nb && (gs[m] != 0 || m == 0 || m == nb - 1);
    const uint32_t vw = __ballot_sync(0xffffffffu, v), rw = __ballot_sync(0xffffffffu, r);
    if (lane == 0) {
      V[w] = vw;
      R[w] = rw;
    }
  }
  if (threadIdx.x < 2) R[words + threadIdx.x] = 0u;  // the shifted reads run up to two words past
  __syncthreads();
}

// 32 bits of R from bit position p on.
__device__ __forceinline__ uint32_t bits_at(const uint32_t* R, int p) {
  const int w = p >> 5, sh = p & 31;
  const uint32_t lo = R[w] >> sh;
  return sh ? (lo | (R[w + 1] << (32 - sh))) : lo;
}

// One warp per row: the row's selection bitmask (words of 32 key blocks), its count, and, when
// the head ranks ties, its tied entries (all, and those that are not anchors). Vertical-Slash
// rows take one word per lane from the staged masks; Pooled-Estimation rows compare their pooled
// scores with the cut value, loaded eight words ahead.
__global__ void __launch_bounds__(ROWS * 32) merge_mask_kernel(const SelectArgs a) {
  const int h = blockIdx.y;
  const int nb = a.s.nb, lane = threadIdx.x & 31;
  const int words = (nb + 31) / 32;
  __shared__ uint32_t V[kMaxSelectBlocks / 32], R[kMaxSelectBlocks / 32 + 2];
  const bool vshead = a.route[h] != 0 || nb <= 2;
  if (vshead) stage_vs_masks(a, h, V, R, words);
  const int qb = blockIdx.x * ROWS + (threadIdx.x >> 5);
  if (qb >= nb) return;
  uint32_t* mrow = a.selmask + ((size_t)h * nb + qb) * sel_mask_words(nb);
  const int nw = qb / 32 + 1;  // words holding blocks 0..qb
  int cnt = 0, eqc = 0, eqna = 0;
  if (vshead) {
    for (int w = lane; w < nw; w += 32) {
      uint32_t word;
      if (nb <= 2) {
        word = 0xffffffffu;
      } else {
        const int p = w * 32 + nb - 1 - qb;
        word = V[w] | bits_at(R, p) | bits_at(R, p + 1);
      }
      if (w == nw - 1) {
        const int keep = (qb & 31) + 1;  // blocks <= qb in the last word
        word &= keep == 32 ? 0xffffffffu : ((1u << keep) - 1u);
      }
      mrow[w] = word;
      cnt += __popc(word);
    }
  } else {
    const RowCtx c = make_ctx(a, h, qb);
    const bool rank = head_ranks_ties(a, h);
    for (int w0 = 0; w0 < nw; w0 += 8) {
      float pv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int kb = (w0 + u) * 32 + lane;
        pv[u] = kb <= qb ? __ldg(c.P + kb) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int w = w0 + u;
        if (w >= nw) break;
        const int kb = w * 32 + lane;
        bool sel = false, eq = false;
        if (kb <= qb) {
          const int f = pe_flag_of(c, pv[u]);
          const bool anchor = pe_anchor(c, kb);
          sel = f == 1 || anchor || (f == 2 && !rank);
          eq = rank && f == 2;
          eqna += (eq && !anchor) ? 1 : 0;
        }
        const uint32_t word = __ballot_sync(0xffffffffu, sel);
        eqc += __popc(__ballot_sync(0xffffffffu, eq));
        if (lane == (w & 31)) mrow[w] = word;
        if (lane == 0) cnt += __popc(word);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    eqna += __shfl_xor_sync(0xffffffffu, eqna, o);
  }
  if (lane == 0) {
    const size_t i = (size_t)h * nb + qb;
    a.cnt[i] = cnt;
    a.eqcnt[i] = eqc;
    a.eqbase[i] = eqna;
  }
}

// Tied entries of row qb (PE, head with ranked ties) in kb order: calls f(kb, anchor) for each.
template <typename F>
__device__ __forceinline__ void for_each_tie(const RowCtx& c, F f) {
  const int lane = threadIdx.x & 31;
  for (int base = 0; base <= c.qb; base += 32) {
    const int kb = base + lane;
    const bool eq = kb <= c.qb && pe_flag_of(c, __ldg(c.P + kb)) == 2;
    unsigned b = __ballot_sync(0xffffffffu, eq);
    while (b) {
      const int j = __ffs(b) - 1;
      f(base + j, pe_anchor(c, base + j));
      b &= b - 1;
    }
  }
}

// Non-anchor tied entries of row qb among global tie ranks [rank0, t_eq) — the ones the quota
// adds to the row. Warp-collective; every lane returns the count.
__device__ int quota_ties(const RowCtx& c, long long rank0, long long t_eq) {
  int add = 0;
  long long r = rank0;
  for_each_tie(c, [&](int, bool anchor) {
    if (r < t_eq && !anchor) ++add;
    ++r;
  });
  return add;
}

constexpr int SCAN_THREADS = 1024;

// Block-wide exclusive scan of one value per thread (returns the thread's prefix; *total gets
// the sum of all threads).
__device__ long long block_exclusive_scan(long long v, long long* warp_tot, long long* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    long long t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive
  }
  __syncthreads();
  *total = warp_tot[SCAN_THREADS / 32 - 1];
  return (w > 0 ? warp_tot[w - 1] : 0) + x - v;
}

// One CTA per head: CSR offsets row_ptr[0..N_b] from the row counts. When the head ranks ties,
// the tied entries are taken in (qb, kb) order up to the quota t_eq: a row whose ties all fall
// inside the quota adds its non-anchor ties, the row where the quota ends adds those of its ties
// that fall inside (recounted from its scores), later rows none; the tie rank of each row's first
// tied entry is left in cnt[] for the write pass.
__global__ void __launch_bounds__(SCAN_THREADS) merge_scan_kernel(const SelectArgs a) {
  const int h = blockIdx.x, nb = a.s.nb, tid = threadIdx.x;
  int* cnt = a.cnt + (size_t)h * nb;
  const int* eqc = a.eqcnt + (size_t)h * nb;
  const int* eqna = a.eqbase + (size_t)h * nb;
  const bool rank = head_ranks_ties(a, h);
  const long long t_eq = rank ? (long long)a.cut[h].t_eq : 0;
  __shared__ long long warp_tot[32];
  __shared__ int s_brow;
  __shared__ long long s_brank;
  __shared__ int s_badd;
  int32_t* rp = a.row_ptr + (size_t)h * (nb + 1);
  if (tid == 0) s_brow = -1;
  // pass 1 (ranked ties only): tie ranks, and the boundary row
  if (rank) {
    long long carry = 0;
    for (int base = 0; base < nb; base += SCAN_THREADS) {
      const int r = base + tid;
      const long long e = r < nb ? eqc[r] : 0;
      long long tot;
      const long long rank_r = carry + block_exclusive_scan(e, warp_tot, &tot);
      if (r < nb) {
        if (rank_r < t_eq && rank_r + e > t_eq) {
          s_brow = r;
          s_brank = rank_r;
        }
      }
      carry += tot;
      // the ranks wait in row_ptr until pass 2 replaces each with the row's offset
      if (r < nb) rp[r] = (int32_t)rank_r;
    }
    __syncthreads();
    if (s_brow >= 0 && (tid >> 5) == 0) {
      const RowCtx c = make_ctx(a, h, s_brow);
      const int add = quota_ties(c, s_brank, t_eq);
      if ((tid & 31) == 0) s_badd = add;
    }
    __syncthreads();
  }
  // pass 2: final counts and offsets
  long long carry = 0;
  for (int base = 0; base < nb; base += SCAN_THREADS) {
    const int r = base + tid;
    long long fin = 0, rank_r = 0;
    if (r < nb) {
      fin = cnt[r];
      if (rank) {
        rank_r = rp[r];
        const long long e = eqc[r];
        if (rank_r + e <= t_eq) fin += eqna[r];
        else if (r == s_brow) fin += s_badd;
      }
    }
    long long tot;
    const long long start = carry + block_exclusive_scan(fin, warp_tot, &tot);
    if (r < nb) {
      if (rank) cnt[r] = (int)rank_r;  // tie rank for the write pass
      rp[r] = (int32_t)start;
    }
    carry += tot;
  }
  if (tid == 0) {
    rp[nb] = (int32_t)carry;
    if (a.debug != nullptr) a.debug[(size_t)h * (2 * nb + 5) + 2 * nb + 3] = (float)carry;
  }
}

// One warp per row: the column indices, expanded from the row's bitmask one word per step (lane
// j writes block 32w+j if its bit is set, so the stores of a word are contiguous). Rows of a head
// that ranks ties add the tied entries whose rank falls inside the quota first.
__global__ void __launch_bounds__(ROWS * 32) merge_write_kernel(const SelectArgs a) {
  const int qb = blockIdx.x * ROWS + (threadIdx.x >> 5), h = blockIdx.y;
  const int nb = a.s.nb, lane = threadIdx.x & 31;
  if (qb >= nb) return;
  const uint32_t* m = a.selmask + ((size_t)h * nb + qb) * sel_mask_words(nb);
  int32_t* out = a.cols + (size_t)h * a.s.cap + a.row_ptr[(size_t)h * (nb + 1) + qb];
  const bool rank = head_ranks_ties(a, h);
  const long long t_eq = rank ? (long long)a.cut[h].t_eq : 0;
  long long r = rank ? a.cnt[(size_t)h * nb + qb] : 0;  // tie rank of the row's first tie
  const bool ties_here = rank && a.eqcnt[(size_t)h * nb + qb] > 0 && r < t_eq;
  const RowCtx c = make_ctx(a, h, qb);
  const unsigned below = (1u << lane) - 1u;
  const int nw = qb / 32 + 1;  // words that hold blocks 0..qb
  int pos = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int cw = min(32, nw - w0);
    uint32_t mine = lane < cw ? m[w0 + lane] : 0u;  // one load per lane, then shared
    if (ties_here) {
      for (int wi = 0; wi < cw; ++wi) {
        const int kb = (w0 + wi) * 32 + lane;
        const bool eq = kb <= qb && pe_flag_of(c, __ldg(c.P + kb)) == 2;
        const unsigned eb = __ballot_sync(0xffffffffu, eq);
        const uint32_t take = __ballot_sync(0xffffffffu, eq && r + __popc(eb & below) < t_eq);
        if (lane == wi) mine |= take;
        r += __popc(eb);
      }
    }
#pragma unroll 4
    for (int i = 0; i < cw; ++i) {
      const uint32_t bits = __shfl_sync(0xffffffffu, mine, i);
      if ((bits >> lane) & 1u) out[pos + __popc(bits & below)] = (w0 + i) * 32 + lane;
      pos += __popc(bits);
    }
  }
}

}  // namespace

cudaError_t launch_merge(const SelectArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const dim3 rows((s.nb + ROWS - 1) / ROWS, s.h_q);
  merge_mask_kernel<<<rows, ROWS * 32, 0, st>>>(a);
  merge_scan_kernel<<<s.h_q, SCAN_THREADS, 0, st>>>(a);
  merge_write_kernel<<<rows, ROWS * 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace crisp
