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
// Passes: ties with the cut value per row and their exclusive scan (global tie ranks), the exact
// count per row and its exclusive scan (row_ptr), then compaction.
#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

struct RowCtx {
  int vs, nb, qb;
  const uint8_t* kv;
  const uint8_t* ks;
  const float* P;
  uint32_t thr;
  uint32_t keep_all;
};

// kv/ks point at the head's keep flags (staged in shared memory); every test is branch-free.
__device__ __forceinline__ bool vs_sel(const RowCtx& c, int kb) {
  const int m0 = c.qb - kb;  // offset block m with qb-m == kb
  const int m1 = m0 - 1;     // offset block m with qb-m-1 == kb
  const bool fixed = c.nb <= 2 || kb == 0 || kb == c.nb - 1 || m0 == 0 || m0 == c.nb - 1 || m1 == 0;
  const bool v = c.kv[kb] != 0;
  const bool s0 = c.ks[m0] != 0;
  const bool s1 = m1 >= 0 && c.ks[m1 >= 0 ? m1 : 0] != 0;
  return fixed | v | s0 | s1;
}

// PE: where an entry stands relative to the cut value: 0 below, 1 above, 2 equal. Anchors do not
// change this: the cut is taken over every entry, and the anchors are added on top.
__device__ __forceinline__ int pe_cut_flag(const RowCtx& c, int kb) {
  if (c.keep_all) return 1;
  const uint32_t bits = __float_as_uint(c.P[kb]);
  if (bits > c.thr) return 1;
  return bits == c.thr ? 2 : 0;
}

__device__ __forceinline__ bool pe_anchor(const RowCtx& c, int kb) {
  return kb == 0 || kb == c.qb || kb == c.qb - 1;
}

__device__ __forceinline__ RowCtx make_ctx(const SelectArgs& a, int h, int qb) {
  RowCtx c;
  const Shape& s = a.s;
  c.vs = a.route[h];
  c.nb = s.nb;
  c.qb = qb;
  c.kv = a.keep_v + (size_t)h * s.nb;
  c.ks = a.keep_s + (size_t)h * s.nb;
  c.P = a.pbuf + (size_t)h * s.cap + (size_t)qb * (qb + 1) / 2;
  const CutState cs = a.cut[h];
  c.thr = cs.thr_bits;
  c.keep_all = (s.nb <= 2 || c.vs) ? 1u : cs.keep_all;
  return c;
}

__device__ __forceinline__ long long tie_quota(const SelectArgs& a, int h) {
  const CutState cs = a.cut[h];
  return (a.route[h] || a.s.nb <= 2 || cs.keep_all) ? 0 : (long long)cs.t_eq;
}

// One warp per row, ROWS rows per CTA. Walks row qb of head h in key-block order, 32 blocks per
// step, and calls emit(kb, position) for every selected block; returns the row's count. Entries
// tied with the cut value are ranked over the whole head in (qb, kb) order, starting from
// eqbase[qb]; the first t_eq of them are kept.
constexpr int ROWS = 8;
// The head's keep flags staged in shared memory (all rows of a CTA share one head).
constexpr int kMaxStagedBlocks = 8192;
__device__ __forceinline__ void stage_flags(const SelectArgs& a, int h, uint8_t* skv, uint8_t* sks) {
  const int nb = a.s.nb;
  if (nb > kMaxStagedBlocks) return;
  const uint8_t* gv = a.keep_v + (size_t)h * nb;
  const uint8_t* gs = a.keep_s + (size_t)h * nb;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    skv[i] = gv[i];
    sks[i] = gs[i];
  }
  __syncthreads();
}

template <typename Emit>
__device__ __forceinline__ int walk_row(const SelectArgs& a, int h, int qb, long long erank, const uint8_t* skv,
                                        const uint8_t* sks, Emit emit, uint32_t* mrow = nullptr) {
  RowCtx c = make_ctx(a, h, qb);
  if (a.s.nb <= kMaxStagedBlocks) {
    c.kv = skv;
    c.ks = sks;
  }
  const bool vsrow = c.vs || a.s.nb <= 2;
  const long long t_eq = tie_quota(a, h);
  // With at most one entry equal to the cut value it is always kept (t_eq >= 1): no ranking.
  const bool rank_ties = !vsrow && a.cut[h].count_eq > 1;
  const int lane = threadIdx.x & 31;
  const unsigned below = (1u << lane) - 1u;
  int count = 0;
  for (int base = 0; base <= qb; base += 128) {
    // four 32-entry sub-chunks; the pooled scores of a PE row are loaded together
    int flag[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int kb = base + 32 * u + lane;
      flag[u] = (kb <= qb && !vsrow) ? pe_cut_flag(c, kb) : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int kb = base + 32 * u + lane;
      bool sel = false, eqf = false;
      if (kb <= qb) {
        if (vsrow) {
          sel = vs_sel(c, kb);
        } else {
          sel = flag[u] == 1 || pe_anchor(c, kb) || (flag[u] == 2 && !rank_ties);
          eqf = rank_ties && flag[u] == 2;
        }
      }
      if (rank_ties) {
        const unsigned eb = __ballot_sync(0xffffffffu, eqf);
        if (eqf && erank + __popc(eb & below) < t_eq) sel = true;
        erank += __popc(eb);
      }
      const unsigned sb = __ballot_sync(0xffffffffu, sel);
      if (sel) emit(kb, count + __popc(sb & below));
      if (mrow != nullptr && lane == 0) mrow[base / 32 + u] = sb;  // blocks base+32u .. +31
      count += __popc(sb);
    }
  }
  return count;
}

// Pass 1: entries of each PE row that tie with the cut value (only heads with >1 such entry).
__global__ void __launch_bounds__(ROWS * 32) merge_ties_kernel(const SelectArgs a) {
  const int qb = blockIdx.x * ROWS + (threadIdx.x >> 5), h = blockIdx.y;
  if (qb >= a.s.nb) return;
  if (a.cut[h].count_eq <= 1) {
    if ((threadIdx.x & 31) == 0) a.eqcnt[(size_t)h * a.s.nb + qb] = 0;
    return;
  }
  const RowCtx c = make_ctx(a, h, qb);
  int ne = 0;
  if (!(c.vs || a.s.nb <= 2))
    for (int kb = threadIdx.x & 31; kb <= qb; kb += 32) ne += pe_cut_flag(c, kb) == 2;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ne += __shfl_xor_sync(0xffffffffu, ne, o);
  if ((threadIdx.x & 31) == 0) a.eqcnt[(size_t)h * a.s.nb + qb] = ne;
}

// Pass 2: exact number of selected blocks per row.
__global__ void __launch_bounds__(ROWS * 32) merge_count_kernel(const SelectArgs a) {
  const int qb = blockIdx.x * ROWS + (threadIdx.x >> 5), h = blockIdx.y;
  __shared__ uint8_t skv[kMaxStagedBlocks], sks[kMaxStagedBlocks];
  stage_flags(a, h, skv, sks);
  if (qb >= a.s.nb) return;
  const long long erank = a.eqbase[(size_t)h * (a.s.nb + 1) + qb];
  uint32_t* mrow = a.selmask + ((size_t)h * a.s.nb + qb) * sel_mask_words(a.s.nb);
  const int n = walk_row(a, h, qb, erank, skv, sks, [](int, int) {}, mrow);
  if ((threadIdx.x & 31) == 0) a.cnt[(size_t)h * a.s.nb + qb] = n;
}

// Pass 3: compaction into the CSR column array, from the bitmask the count pass left: one warp per
// row takes one word at a time, lane j writing block 32w+j if its bit is set, so the stores of a
// word are contiguous.
__global__ void __launch_bounds__(ROWS * 32) merge_write_kernel(const SelectArgs a) {
  const int qb = blockIdx.x * ROWS + (threadIdx.x >> 5), h = blockIdx.y;
  const int nb = a.s.nb, lane = threadIdx.x & 31;
  if (qb >= nb) return;
  const uint32_t* m = a.selmask + ((size_t)h * nb + qb) * sel_mask_words(nb);
  int32_t* out = a.cols + (size_t)h * a.s.cap + a.row_ptr[(size_t)h * (nb + 1) + qb];
  const unsigned below = (1u << lane) - 1u;
  const int nw = qb / 32 + 1;  // words that hold blocks 0..qb
  int pos = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const uint32_t mine = w0 + lane < nw ? m[w0 + lane] : 0u;  // one load per lane, then shared
    const int cnt = min(32, nw - w0);
    for (int i = 0; i < cnt; ++i) {
      const uint32_t bits = __shfl_sync(0xffffffffu, mine, i);
      if ((bits >> lane) & 1u) out[pos + __popc(bits & below)] = (w0 + i) * 32 + lane;
      pos += __popc(bits);
    }
  }
}

// One CTA per head: exclusive scan of in[h][0..nb) into out[h][0..nb] (out[nb] = total).
__global__ void __launch_bounds__(1024) scan_rows_kernel(const int* in, int* out, int nb, float* debug_total) {
  const int h = blockIdx.x;
  const int* src = in + (size_t)h * nb;
  int* dst = out + (size_t)h * (nb + 1);
  __shared__ int wsum[32];
  __shared__ long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int base = 0; base < nb; base += 1024) {
    const int i = base + threadIdx.x;
    const int v = i < nb ? src[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      wsum[lane] = t;
    }
    __syncthreads();
    const long long before = carry + (w > 0 ? wsum[w - 1] : 0) + x - v;
    if (i < nb) dst[i] = (int)before;
    __syncthreads();
    if (threadIdx.x == 0) carry += wsum[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    dst[nb] = (int)carry;
    if (debug_total != nullptr) debug_total[(size_t)h * (2 * nb + 5) + 2 * nb + 3] = (float)carry;
  }
}

}  // namespace

cudaError_t launch_merge(const SelectArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const dim3 rows((s.nb + ROWS - 1) / ROWS, s.h_q);
  merge_ties_kernel<<<rows, ROWS * 32, 0, st>>>(a);
  scan_rows_kernel<<<s.h_q, 1024, 0, st>>>(a.eqcnt, a.eqbase, s.nb, nullptr);
  merge_count_kernel<<<rows, ROWS * 32, 0, st>>>(a);
  scan_rows_kernel<<<s.h_q, 1024, 0, st>>>(a.cnt, a.row_ptr, s.nb, a.debug);
  merge_write_kernel<<<rows, ROWS * 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace crisp
