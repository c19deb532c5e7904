// crisp_api.cu — the C ABI of libcrisp: argument validation, workspace layout, TMA descriptor
// encoding and the launch sequence of each entry point. Nothing here allocates device memory;
// every buffer comes from the caller.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstring>

#include "crisp_internal.h"
#include "sm100.cuh"

namespace crisp {
namespace {

// NVTX push/pop range over a scope: the kernels launched inside it carry the range's name in a
// profiler (ncu --nvtx --nvtx-include "crisp_select/" selects the selection kernels). With no
// profiler attached a push or pop is a call through a no-op pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // Resolved once through the runtime (no link-time dependency on libcuda).
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

}  // namespace

// 3D bf16 view [heads][n][128] (heads `ld` rows apart) with 64x128x1 boxes: a head's rows past n
// read as zeros, so a partial last block never sees the next head's (or sequence's) rows.
int make_map3(CUtensorMap* m, const void* base, uint64_t n, uint64_t heads, uint64_t ld) {
  auto fn = encode_fn();
  if (fn == nullptr) return CRISP_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)n, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kD * 2 * ld};
  cuuint32_t box[3] = {64, (cuuint32_t)kB, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CRISP_OK : CRISP_ERR_CUDA;
}

namespace {
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

// Any n >= 1 (a partial last block when n is not a multiple of 128); selection adds n >= 128.
int check_shape(int h_q, int h_kv, int n, int d, Shape* s) {
  if (h_q <= 0 || h_kv <= 0 || n <= 0 || d <= 0) return CRISP_ERR_INVALID_ARG;
  if (d != kD || h_q % h_kv != 0) return CRISP_ERR_UNSUPPORTED;
  const long long nb = (n + kB - 1) / kB;
  const long long cap = nb * (nb + 1) / 2;
  if (cap > 0x7fffffffLL || (long long)h_q * n > 0x7fffffffLL || (long long)h_kv * n > 0x7fffffffLL)
    return CRISP_ERR_OVERFLOW;
  s->h_q = h_q;
  s->h_kv = h_kv;
  s->n = n;
  s->ld = n;
  s->nb = (int)nb;
  s->G = h_q / h_kv;
  s->n_chunks = (int)((nb + kProxyChunk - 1) / kProxyChunk);
  s->cap = cap;
  return CRISP_OK;
}

int check_params(const crisp_params* p) {
  if (p == nullptr) return CRISP_ERR_INVALID_ARG;
  if (p->block != kB || p->anchors != kB) return CRISP_ERR_UNSUPPORTED;
  if (!std::isfinite(p->tau_proxy) || !std::isfinite(p->alpha) || !std::isfinite(p->gamma))
    return CRISP_ERR_INVALID_ARG;
  if (p->alpha < 0.f || p->gamma <= 0.f || p->min_blocks < 0) return CRISP_ERR_INVALID_ARG;
  if ((p->route_rule != 0 && p->route_rule != 1) || (p->vs_rule != 0 && p->vs_rule != 1) ||
      (p->floor_rule != 0 && p->floor_rule != 1) || !std::isfinite(p->tau_jsd) || p->tau_jsd < 0.f)
    return CRISP_ERR_INVALID_ARG;
  return CRISP_OK;
}

namespace {
int check_index(const crisp_index* idx, bool need_select_fields) {
  if (idx == nullptr || idx->row_ptr == nullptr || idx->cols == nullptr) return CRISP_ERR_INVALID_ARG;
  if (need_select_fields && (idx->route == nullptr || idx->c_struct == nullptr)) return CRISP_ERR_INVALID_ARG;
  if (!aligned(idx->row_ptr, 4) || !aligned(idx->cols, 4)) return CRISP_ERR_INVALID_ARG;
  return CRISP_OK;
}

int check_ws(void* ws, size_t ws_bytes, const Shape& s) {
  if (ws == nullptr || !aligned(ws, 256)) return CRISP_ERR_INVALID_ARG;
  if (ws_bytes < workspace_layout(s).total) return CRISP_ERR_WORKSPACE;
  return CRISP_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace

int run_select(const void* q, const void* k, const Shape& s, const crisp_params* p, const crisp_index& out,
               void* ws, int* status, cudaStream_t st) {
  NvtxRange range("crisp_select");
  const Workspace w = workspace_layout(s);
  SelectArgs a{};
  a.s = s;
  a.tau = p->tau_proxy;
  a.alpha = p->alpha;
  a.gamma = p->gamma;
  a.min_blocks = p->min_blocks;
  a.route_rule = p->route_rule;
  a.tau_jsd = p->tau_jsd;
  a.vs_rule = p->vs_rule;
  a.floor_rule = p->floor_rule;
  a.status = status != nullptr ? status : at<int>(ws, w.status);
  a.trace = at<unsigned long long>(ws, w.trace);
  a.part = at<float2>(ws, w.part);
  a.chunk_max = at<float>(ws, w.chunk_max);
  a.chunk_tot = at<float>(ws, w.chunk_tot);
  a.row_w = at<float>(ws, w.row_w);
  a.pv = at<double>(ws, w.pv);
  a.ps_lo = at<double>(ws, w.ps_lo);
  a.ps_hi = at<double>(ws, w.ps_hi);
  a.ps_x = at<double>(ws, w.ps_x);
  a.rec_extra = at<float>(ws, w.rec_extra);
  a.kbar = at<float>(ws, w.kbar);
  a.kparts = at<__nv_bfloat16>(ws, w.kparts);
  a.qparts = at<__nv_bfloat16>(ws, w.qparts);
  a.pbuf = at<float>(ws, w.pbuf);
  a.hist_cnt = at<uint32_t>(ws, w.hist_cnt);
  a.hist_mass = at<unsigned long long>(ws, w.hist_mass);
  a.cut = at<CutState>(ws, w.cut);
  a.cut_done = at<uint32_t>(ws, w.cut_done);
  a.keep_v = at<uint8_t>(ws, w.keep_v);
  a.keep_s = at<uint8_t>(ws, w.keep_s);
  a.cnt = at<int>(ws, w.cnt);
  a.eqcnt = at<int>(ws, w.eqcnt);
  a.eqbase = at<int>(ws, w.eqbase);
  a.selmask = at<uint32_t>(ws, w.selmask);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.route = out.route;
  a.c_struct = out.c_struct;
  a.row_ptr = out.row_ptr;
  a.cols = out.cols;
  a.debug = out.debug;

  // Q and K as the inputs lay them out; the pooled-block terms as [heads x 3][N_b][128].
  CUtensorMap qm, km, qpm, kpm;
  int rc = make_map3(&qm, q, (uint64_t)s.n, (uint64_t)s.h_q, (uint64_t)s.ld);
  if (rc == CRISP_OK) rc = make_map3(&km, k, (uint64_t)s.n, (uint64_t)s.h_kv, (uint64_t)s.ld);
  if (rc == CRISP_OK) rc = make_map3(&qpm, a.qparts, (uint64_t)s.nb, (uint64_t)s.h_q * 3, (uint64_t)s.nb);
  if (rc == CRISP_OK) rc = make_map3(&kpm, a.kparts, (uint64_t)s.nb, (uint64_t)s.h_kv * 3, (uint64_t)s.nb);
  if (rc != CRISP_OK) return rc;

  // The radix histograms accumulate with atomics and the cut levels count finished CTAs: start
  // from zero (the arrays are contiguous).
  if (cudaMemsetAsync(at<uint8_t>(ws, w.hist_cnt), 0, w.cut_done + (size_t)s.h_q * 4 - w.hist_cnt, st) != cudaSuccess)
    return CRISP_ERR_CUDA;
  {
    NvtxRange stage("proxy_pass");
    if (launch_proxy_pass(qm, km, a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  }
  {
    NvtxRange stage("route_threshold");
    if (launch_route_threshold(a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  }
  {
    NvtxRange stage("pooled_estimation");
    if (launch_pe(a, qpm, kpm, st) != cudaSuccess) return CRISP_ERR_CUDA;
  }
  {
    NvtxRange stage("merge");
    if (launch_merge(a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  }
  return CRISP_OK;
}

namespace {

int run_attention(const void* q, const void* k, const void* v, const Shape& s, const int32_t* row_ptr,
                  const int32_t* cols, const int32_t* route, int dense, void* o, float* lse, void* ws,
                  cudaStream_t st) {
  const Workspace w = workspace_layout(s);
  AttnArgs a{};
  a.s = s;
  a.dense = dense;
  a.row_ptr = row_ptr;
  a.cols = cols;
  a.route = route;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = at<int>(ws, w.status);
  a.trace = at<unsigned long long>(ws, w.trace);
  a.scale_log2 = 0.12751743074380045f;  // log2(e) / sqrt(128)
  CUtensorMap qm, km, vm;
  int rc = make_map3(&qm, q, (uint64_t)s.n, (uint64_t)s.h_q, (uint64_t)s.ld);
  if (rc == CRISP_OK) rc = make_map3(&km, k, (uint64_t)s.n, (uint64_t)s.h_kv, (uint64_t)s.ld);
  if (rc == CRISP_OK) rc = make_map3(&vm, v, (uint64_t)s.n, (uint64_t)s.h_kv, (uint64_t)s.ld);
  if (rc != CRISP_OK) return rc;
  NvtxRange range(dense ? "crisp_dense_attention" : "crisp_attention");
  return launch_sparse_attn(qm, km, vm, a, st) == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}

bool tensors_ok(const void* q, const void* k, const void* v) {
  return q != nullptr && k != nullptr && (v == nullptr || aligned(v, 16)) && aligned(q, 16) && aligned(k, 16);
}

// Device-side timeout self-test: waits on a barrier that nothing signals.
__global__ void timeout_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, nullptr, limit_ns)) record_status(status, CRISP_ERR_DEVICE_TIMEOUT);
  }
}

}  // namespace

cudaError_t launch_timeout_selftest(int* status, unsigned long long limit_ns, cudaStream_t st) {
  timeout_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace crisp

using namespace crisp;

extern "C" {

size_t crisp_workspace_size(int h_q, int h_kv, int n, int d, const crisp_params* params) {
  Shape s;
  if (check_shape(h_q, h_kv, n, d, &s) != CRISP_OK) return 0;
  if (params != nullptr && n < kB) return 0;
  if (params != nullptr && check_params(params) != CRISP_OK) return 0;
  return workspace_layout(s).total;
}

int crisp_select(const void* q, const void* k, int h_q, int h_kv, int n, int d, const crisp_params* params,
                 const crisp_index* out, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  int rc = check_shape(h_q, h_kv, n, d, &s);
  if (rc == CRISP_OK) rc = check_params(params);
  if (rc == CRISP_OK && (s.nb > kMaxSelectBlocks || n < kB)) rc = CRISP_ERR_UNSUPPORTED;
  if (rc == CRISP_OK && !tensors_ok(q, k, nullptr)) rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK) rc = check_index(out, true);
  if (rc == CRISP_OK) rc = check_ws(ws, ws_bytes, s);
  if (rc != CRISP_OK) return rc;
  return run_select(q, k, s, params, *out, ws, nullptr, static_cast<cudaStream_t>(stream));
}

int crisp_sparse_prefill(const void* q, const void* k, const void* v, int h_q, int h_kv, int n, int d,
                         const crisp_index* idx, void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  int rc = check_shape(h_q, h_kv, n, d, &s);
  if (rc == CRISP_OK && (!tensors_ok(q, k, v) || v == nullptr || o == nullptr || !aligned(o, 16)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK) rc = check_index(idx, false);
  if (rc == CRISP_OK) rc = check_ws(ws, ws_bytes, s);
  if (rc != CRISP_OK) return rc;
  return run_attention(q, k, v, s, idx->row_ptr, idx->cols, idx->route, 0, o, lse, ws,
                       static_cast<cudaStream_t>(stream));
}

int crisp_prefill(const void* q, const void* k, const void* v, int h_q, int h_kv, int n, int d,
                  const crisp_params* params, void* o, float* lse, const crisp_index* idx_out, void* ws,
                  size_t ws_bytes, void* stream) {
  Shape s;
  int rc = check_shape(h_q, h_kv, n, d, &s);
  if (rc == CRISP_OK) rc = check_params(params);
  if (rc == CRISP_OK && (s.nb > kMaxSelectBlocks || n < kB)) rc = CRISP_ERR_UNSUPPORTED;
  if (rc == CRISP_OK && (!tensors_ok(q, k, v) || v == nullptr || o == nullptr || !aligned(o, 16)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK && idx_out != nullptr) rc = check_index(idx_out, true);
  if (rc == CRISP_OK) rc = check_ws(ws, ws_bytes, s);
  if (rc != CRISP_OK) return rc;
  crisp_index idx;
  if (idx_out != nullptr) {
    idx = *idx_out;
  } else {
    const Workspace w = workspace_layout(s);
    idx.route = at<int32_t>(ws, w.idx_route);
    idx.c_struct = at<float>(ws, w.idx_c);
    idx.row_ptr = at<int32_t>(ws, w.idx_row_ptr);
    idx.cols = at<int32_t>(ws, w.idx_cols);
    idx.debug = nullptr;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = run_select(q, k, s, params, idx, ws, nullptr, st);
  if (rc != CRISP_OK) return rc;
  return run_attention(q, k, v, s, idx.row_ptr, idx.cols, idx.route, 0, o, lse, ws, st);
}

int crisp_prefill_varlen(const void* q, const void* k, const void* v, int h_q, int h_kv, int total,
                         const int32_t* cu_seqlens, int n_seqs, int d, const crisp_params* params, void* o,
                         float* lse, void* ws, size_t ws_bytes, void* stream) {
  // every check comes before the first launch
  Shape whole;
  int rc = check_shape(h_q, h_kv, total, d, &whole);
  if (rc == CRISP_OK) rc = check_params(params);
  if (rc == CRISP_OK && (!tensors_ok(q, k, v) || v == nullptr || o == nullptr || !aligned(o, 16)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK && (cu_seqlens == nullptr || n_seqs <= 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != total))
    rc = CRISP_ERR_INVALID_ARG;
  int longest = 0;
  for (int i = 0; rc == CRISP_OK && i < n_seqs; ++i) {
    const int len = cu_seqlens[i + 1] - cu_seqlens[i];
    if (len < 0) rc = CRISP_ERR_INVALID_ARG;
    else if (len > 0 && len < kB) rc = CRISP_ERR_UNSUPPORTED;  // selection takes the last 128 queries
    longest = len > longest ? len : longest;
  }
  Shape big;
  if (rc == CRISP_OK) rc = longest > 0 ? check_shape(h_q, h_kv, longest, d, &big) : CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK && big.nb > kMaxSelectBlocks) rc = CRISP_ERR_UNSUPPORTED;
  if (rc == CRISP_OK) rc = check_ws(ws, ws_bytes, big);
  if (rc != CRISP_OK) return rc;
  // One sequence after another on the stream, each on the same workspace (its index included);
  // a sequence's tensors start at its first token and keep the batch's per-head stride.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < n_seqs; ++i) {
    const int beg = cu_seqlens[i], len = cu_seqlens[i + 1] - beg;
    if (len == 0) continue;
    Shape s;
    check_shape(h_q, h_kv, len, d, &s);
    s.ld = total;
    const Workspace w = workspace_layout(s);
    crisp_index idx;
    idx.route = at<int32_t>(ws, w.idx_route);
    idx.c_struct = at<float>(ws, w.idx_c);
    idx.row_ptr = at<int32_t>(ws, w.idx_row_ptr);
    idx.cols = at<int32_t>(ws, w.idx_cols);
    idx.debug = nullptr;
    const size_t off = (size_t)beg * kD;
    const auto* qs = static_cast<const __nv_bfloat16*>(q) + off;
    const auto* ks = static_cast<const __nv_bfloat16*>(k) + off;
    const auto* vs = static_cast<const __nv_bfloat16*>(v) + off;
    auto* os = static_cast<__nv_bfloat16*>(o) + off;
    rc = run_select(qs, ks, s, params, idx, ws, nullptr, st);
    if (rc == CRISP_OK) rc = run_attention(qs, ks, vs, s, idx.row_ptr, idx.cols, idx.route, 0, os,
                                           lse != nullptr ? lse + beg : nullptr, ws, st);
    if (rc != CRISP_OK) return rc;
  }
  return CRISP_OK;
}

namespace {

struct Fp8Layout {
  size_t q8, k8, qs, ks, total;
};

Fp8Layout fp8_layout(const Shape& s) {
  Fp8Layout f{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  f.q8 = take((size_t)s.h_q * s.n * kD);
  f.k8 = take((size_t)s.h_kv * s.n * kD);
  f.qs = take((size_t)s.h_q * s.nb * 4);
  f.ks = take((size_t)s.h_kv * s.nb * 4);
  f.total = off;
  return f;
}

// 3D uint8 view [heads][n][128] of E4M3 codes with 128x128x1 boxes (one 128-byte swizzle span per
// row): rows past n read as zeros.
int make_map3_u8(CUtensorMap* m, const void* base, uint64_t n, uint64_t heads) {
  auto fn = encode_fn();
  if (fn == nullptr) return CRISP_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)n, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)kD, (cuuint64_t)kD * n};
  cuuint32_t box[3] = {(cuuint32_t)kD, (cuuint32_t)kB, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CRISP_OK : CRISP_ERR_CUDA;
}

}  // namespace

size_t crisp_fp8qk_buffer_size(int h_q, int h_kv, int n, int d) {
  Shape s;
  if (check_shape(h_q, h_kv, n, d, &s) != CRISP_OK) return 0;
  return fp8_layout(s).total;
}

int crisp_sparse_prefill_fp8qk(const void* q, const void* k, const void* v, int h_q, int h_kv, int n, int d,
                               const crisp_index* idx, void* o, float* lse, void* ws, size_t ws_bytes,
                               void* fp8_buf, size_t fp8_bytes, void* stream) {
  Shape s;
  int rc = check_shape(h_q, h_kv, n, d, &s);
  if (rc == CRISP_OK && (!tensors_ok(q, k, v) || v == nullptr || o == nullptr || !aligned(o, 16)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK) rc = check_index(idx, false);
  if (rc == CRISP_OK) rc = check_ws(ws, ws_bytes, s);
  if (rc == CRISP_OK && (fp8_buf == nullptr || !aligned(fp8_buf, 256))) rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK && fp8_bytes < fp8_layout(s).total) rc = CRISP_ERR_WORKSPACE;
  if (rc != CRISP_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Fp8Layout f = fp8_layout(s);
  uint8_t* q8 = at<uint8_t>(fp8_buf, f.q8);
  uint8_t* k8 = at<uint8_t>(fp8_buf, f.k8);
  float* qs = at<float>(fp8_buf, f.qs);
  float* ks = at<float>(fp8_buf, f.ks);
  {
    NvtxRange range("crisp_fp8_quantise");
    if (launch_fp8_quant(static_cast<const __nv_bfloat16*>(q), s.h_q, s.n, s.ld, q8, qs, st) != cudaSuccess ||
        launch_fp8_quant(static_cast<const __nv_bfloat16*>(k), s.h_kv, s.n, s.ld, k8, ks, st) != cudaSuccess)
      return CRISP_ERR_CUDA;
  }
  const Workspace w = workspace_layout(s);
  AttnArgs a{};
  a.s = s;
  a.dense = 0;
  a.row_ptr = idx->row_ptr;
  a.cols = idx->cols;
  a.route = idx->route;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = at<int>(ws, w.status);
  a.trace = at<unsigned long long>(ws, w.trace);
  a.scale_log2 = 0.12751743074380045f;  // log2(e) / sqrt(128)
  a.qs = qs;
  a.ks = ks;
  CUtensorMap qm, km, vm;
  rc = make_map3_u8(&qm, q8, (uint64_t)s.n, (uint64_t)s.h_q);
  if (rc == CRISP_OK) rc = make_map3_u8(&km, k8, (uint64_t)s.n, (uint64_t)s.h_kv);
  if (rc == CRISP_OK) rc = make_map3(&vm, v, (uint64_t)s.n, (uint64_t)s.h_kv, (uint64_t)s.ld);
  if (rc != CRISP_OK) return rc;
  NvtxRange range("crisp_attention_fp8qk");
  return launch_sparse_attn(qm, km, vm, a, st) == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}

int crisp_dense_prefill(const void* q, const void* k, const void* v, int h_q, int h_kv, int n, int d, void* o,
                        float* lse, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  int rc = check_shape(h_q, h_kv, n, d, &s);
  if (rc == CRISP_OK && (!tensors_ok(q, k, v) || v == nullptr || o == nullptr || !aligned(o, 16)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK) rc = check_ws(ws, ws_bytes, s);
  if (rc != CRISP_OK) return rc;
  return run_attention(q, k, v, s, nullptr, nullptr, nullptr, 1, o, lse, ws, static_cast<cudaStream_t>(stream));
}

int crisp_get_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return CRISP_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CRISP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return CRISP_ERR_CUDA;
  if (v != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return CRISP_ERR_CUDA;
  return v;
}

const char* crisp_status_string(int status) {
  switch (status) {
    case CRISP_OK: return "CRISP_OK";
    case CRISP_ERR_INVALID_ARG: return "CRISP_ERR_INVALID_ARG";
    case CRISP_ERR_UNSUPPORTED: return "CRISP_ERR_UNSUPPORTED";
    case CRISP_ERR_WORKSPACE: return "CRISP_ERR_WORKSPACE";
    case CRISP_ERR_CUDA: return "CRISP_ERR_CUDA";
    case CRISP_ERR_DEVICE_TIMEOUT: return "CRISP_ERR_DEVICE_TIMEOUT";
    case CRISP_ERR_OVERFLOW: return "CRISP_ERR_OVERFLOW";
    case CRISP_ERR_DEVICE_CHECK: return "CRISP_ERR_DEVICE_CHECK";
    default: return "CRISP_ERR_UNKNOWN";
  }
}

int crisp_selftest_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < 256) return CRISP_ERR_INVALID_ARG;
  return launch_timeout_selftest(static_cast<int*>(ws), limit_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? CRISP_OK
             : CRISP_ERR_CUDA;
}

}  // extern "C"
