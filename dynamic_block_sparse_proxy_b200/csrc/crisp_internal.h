// crisp_internal.h — shapes, workspace layout and kernel launch declarations shared by the
// host entry points and the kernels of libcrisp.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "crisp.h"

namespace crisp {

constexpr int kB = 128;        // block size (queries and keys)
constexpr int kD = 128;        // head dimension
constexpr int kProxyChunk = 16;  // key blocks per proxy CTA
constexpr int kHistBins = 2048;        // radix-select bins of the first pass (11, 10, 10 bits)
constexpr int kMaxSelectBlocks = 8192;  // selection keeps per-head block arrays in shared memory
constexpr double kMassUnit = 1099511627776.0;  // 2^40: fixed-point scale of histogram masses

struct Shape {
  int h_q, h_kv, n, nb, G, n_chunks;
  int ld;  // rows between consecutive heads in Q, K, V, O and LSE (n, or the packed batch length)
  long long cap;  // per-head capacity of the column array: nb*(nb+1)/2
};

// State of the Pooled-Estimation cut of one head (device memory, inside the workspace).
struct CutState {
  double target;       // gamma * N_b
  double mass_above;   // mass of entries above the current bucket prefix
  uint32_t prefix;     // bit prefix fixed so far
  uint32_t keep_all;   // 1: gamma >= 1 or the target is not reachable -> keep every entry
  uint32_t thr_bits;   // final threshold value (fp32 bit pattern)
  uint32_t t_eq;       // entries equal to the threshold to keep, in (qb, kb) order
  uint32_t count_eq;   // entries equal to the threshold
  uint32_t pad;
};

struct Workspace {
  size_t status, trace, part, chunk_max, chunk_tot, row_w, pv, ps_lo, ps_hi, ps_x, rec_extra, kbar, kparts, qparts,
      pbuf, hist_cnt, hist_mass, cut, cut_done, keep_v, keep_s, cnt,
      eqcnt, eqbase, selmask, idx_route, idx_c, idx_row_ptr, idx_cols, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// 32-bit words of one row's selection bitmask: blocks are decided 128 at a time, 32 per word.
inline __host__ __device__ int sel_mask_words(int nb) { return 4 * ((nb + 127) / 128); }

inline Workspace workspace_layout(const Shape& s) {
  Workspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t hq = s.h_q, nb = s.nb, ch = s.n_chunks;
  w.status = take(256);
  w.trace = take((size_t)256 * 2 * 8 * 8);
  // the proxy pass keeps one reference per (chunk, 64-column half) "segment" and proxy row
  w.part = take(hq * nb * 2 * kB * 8);
  w.chunk_max = take(hq * ch * 2 * kB * 4);
  w.chunk_tot = take(hq * ch * 2 * kB * 4);
  w.row_w = take(hq * ch * 2 * kB * 4);
  w.pv = take(hq * nb * 8);
  w.ps_lo = take(hq * nb * 8);
  w.ps_hi = take(hq * nb * 8);
  w.ps_x = take(hq * nb * 8);
  w.rec_extra = take(hq * 2 * kB * 4);
  w.kbar = take((size_t)s.h_kv * nb * kD * 4);
  w.kparts = take((size_t)s.h_kv * 3 * nb * kD * 2);
  w.qparts = take(hq * 3 * nb * kD * 2);
  w.pbuf = take(hq * (size_t)s.cap * 4);
  // hist_cnt .. cut_done are contiguous: one memset clears them at the start of a selection
  w.hist_cnt = take(hq * kHistBins * 4);
  w.hist_mass = take(hq * kHistBins * 8);
  w.cut = take(hq * sizeof(CutState));
  w.cut_done = take(hq * 4);
  w.keep_v = take(hq * nb);
  w.keep_s = take(hq * nb);
  w.cnt = take(hq * nb * 4);
  w.eqcnt = take(hq * nb * 4);
  w.eqbase = take(hq * (nb + 1) * 4);
  w.selmask = take(hq * nb * (size_t)sel_mask_words((int)nb) * 4);
  w.idx_route = take(hq * 4);
  w.idx_c = take(hq * 4);
  w.idx_row_ptr = take(hq * (nb + 1) * 4);
  w.idx_cols = take(hq * (size_t)s.cap * 4);
  w.total = off;
  return w;
}

// Kernel parameter block for the selection kernels.
struct SelectArgs {
  Shape s;
  float tau, alpha, gamma;
  int min_blocks;
  int route_rule;  // 0: C_struct >= tau; 1: JSD(a_bar, a_hat) >= tau_jsd
  float tau_jsd;
  int vs_rule;     // 0: noise-floor keep rule; 1: per-direction gamma cut
  int floor_rule;  // 0: mean floor; 1: median floor
  int* status;
  unsigned long long* trace;
  float2* part;        // [h_q][N_b][half][128]: per key block, half and proxy row (lower, upper) sums
  float* chunk_max;    // [h_q][chunk][half][128]: the segment's reference (log2 units)
  float* chunk_tot;    // ... and its total against that reference
  float* row_w;        // ... and the weight that turns its sums into column-mean mass
  double* pv;      // vertical block masses
  double* ps_lo;   // slash block masses from the keys at or below each row's diagonal offset
  double* ps_hi;   // ... and from the keys above it
  double* ps_x;    // ... and (n not a multiple of 128) the next offset block down
  float* rec_extra;  // [h_q][half][128]: recency-window mass inside block N_b-2 (n not a multiple of 128)
  float* kbar;                  // K_bar fp32 [h_kv][N_b][128]
  __nv_bfloat16* kparts;        // K_bar as three bf16 terms [h_kv][3][N_b][128] (sum exact)
  __nv_bfloat16* qparts;        // Q_bar of PE heads, likewise [h_q][3][N_b][128]
  float* pbuf;
  uint32_t* hist_cnt;
  unsigned long long* hist_mass;  // fixed point, 2^-40 units
  CutState* cut;
  uint32_t* cut_done;           // per head: CTAs of the current radix level that finished
  uint8_t* keep_v;
  uint8_t* keep_s;
  int* cnt;
  int* eqcnt;
  int* eqbase;
  uint32_t* selmask;  // per (head, query block): bit kb set iff key block kb is selected
  const __nv_bfloat16* q;
  int32_t* route;
  float* c_struct;
  int32_t* row_ptr;
  int32_t* cols;
  float* debug;
};

struct AttnArgs {
  Shape s;
  int dense;             // 1: every block <= qb, index ignored
  const int32_t* row_ptr;
  const int32_t* cols;
  const int32_t* route;  // per q-head class used to pair heads in a CTA; may be null
  __nv_bfloat16* o;
  float* lse;
  int* status;
  unsigned long long* trace;
  float scale_log2;      // log2(e)/sqrt(d)
  // FP8 logits (q_map and k_map then view E4M3 copies of Q and K): per (head, 128-row block)
  // dequantisation scales [h_q][N_b] and [h_kv][N_b]; null for the bf16 kernel
  const float* qs;
  const float* ks;
};

// Launchers (return cudaGetLastError()).
cudaError_t launch_proxy_pass(const CUtensorMap& q_map, const CUtensorMap& k_map, const SelectArgs& a,
                              cudaStream_t st);
cudaError_t launch_route_threshold(const SelectArgs& a, cudaStream_t st);
cudaError_t launch_pe(const SelectArgs& a, const CUtensorMap& qp_map, const CUtensorMap& kp_map, cudaStream_t st);
cudaError_t launch_merge(const SelectArgs& a, cudaStream_t st);
cudaError_t launch_sparse_attn(const CUtensorMap& q_map, const CUtensorMap& k_map,
                               const CUtensorMap& v_map, const AttnArgs& a, cudaStream_t st);
cudaError_t launch_timeout_selftest(int* status, unsigned long long limit_ns, cudaStream_t st);
// E4M3 copy [heads][n][128] of x (heads `ld` rows apart) and its per-block scales [heads][N_b].
cudaError_t launch_fp8_quant(const __nv_bfloat16* x, int heads, int n, int ld, uint8_t* out, float* scales,
                             cudaStream_t st);

// SMs of the current device (queried once).
int num_sms();

// Host-side helpers shared by the entry points (crisp_api.cu).
int check_shape(int h_q, int h_kv, int n, int d, Shape* s);
int check_params(const crisp_params* p);
int make_map3(CUtensorMap* m, const void* base, uint64_t n, uint64_t heads, uint64_t ld);
// The selection launch sequence on the workspace at `ws` (at least workspace_layout(s).total
// bytes, 256-byte aligned). `status`, when not null, replaces the workspace's status word.
int run_select(const void* q, const void* k, const Shape& s, const crisp_params* p, const crisp_index& out,
               void* ws, int* status, cudaStream_t st);

}  // namespace crisp
