// noalloc.cu — index selection that allocates nothing, for callers that must not call
// cudaMalloc: code that runs under a memory manager that owns every device byte (a serving
// engine's pre-reserved pool), and latency-critical paths where an allocation's implicit device
// synchronisation is not acceptable. The scratch lives in one file-scope device array instead of
// a caller-provided workspace; inputs, outputs and the optional status word stay the caller's.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "crisp_internal.h"

namespace crisp {
namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, fetched once per device (with that device current).
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];

int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CRISP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CRISP_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CRISP_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
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

// bf16 [heads][n][128] with 64x128x1 boxes and 128-byte swizzle, as the selection kernels expect
// (a head's rows past n read as zeros).
int encode_heads(CUtensorMap* m, const void* base, uint64_t n, uint64_t heads) {
  auto fn = encode_tiled();
  if (fn == nullptr) return CRISP_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)n, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kD * 2 * n};
  cuuint32_t box[3] = {64, (cuuint32_t)kB, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? CRISP_OK
             : CRISP_ERR_CUDA;
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace crisp

using namespace crisp;

extern "C" int crisp_select_noalloc(const void* q, const void* k, int h_q, int h_kv, int n, int d,
                                    const crisp_params* p, const crisp_index* out, int* device_status,
                                    void* stream) {
  if (h_q <= 0 || h_kv <= 0 || n <= 0 || d <= 0 || p == nullptr || out == nullptr) return CRISP_ERR_INVALID_ARG;
  if (d != kD || n < kB || h_q % h_kv != 0 || p->block != kB || p->anchors != kB) return CRISP_ERR_UNSUPPORTED;
  if (!std::isfinite(p->tau_proxy) || !std::isfinite(p->alpha) || !std::isfinite(p->gamma) || p->alpha < 0.f ||
      p->gamma <= 0.f || p->min_blocks < 0)
    return CRISP_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || !is_aligned(q, 16) || !is_aligned(k, 16)) return CRISP_ERR_INVALID_ARG;
  if (out->route == nullptr || out->c_struct == nullptr || out->row_ptr == nullptr || out->cols == nullptr ||
      !is_aligned(out->row_ptr, 4) || !is_aligned(out->cols, 4))
    return CRISP_ERR_INVALID_ARG;
  const long long nb = (n + kB - 1) / kB;  // a partial last block when n is not a multiple of 128
  const long long cap = nb * (nb + 1) / 2;
  if (cap > 0x7fffffffLL || (long long)h_q * n > 0x7fffffffLL) return CRISP_ERR_OVERFLOW;
  if (nb > kMaxSelectBlocks) return CRISP_ERR_UNSUPPORTED;
  if ((p->route_rule != 0 && p->route_rule != 1) || (p->vs_rule != 0 && p->vs_rule != 1) ||
      (p->floor_rule != 0 && p->floor_rule != 1) || !std::isfinite(p->tau_jsd) || p->tau_jsd < 0.f)
    return CRISP_ERR_INVALID_ARG;
  Shape s;
  s.h_q = h_q;
  s.h_kv = h_kv;
  s.n = n;
  s.ld = n;
  s.nb = (int)nb;
  s.G = h_q / h_kv;
  s.n_chunks = (int)((nb + kProxyChunk - 1) / kProxyChunk);
  s.cap = cap;
  const Workspace w = workspace_layout(s);
  if (w.total > kNoAllocScratchBytes) return CRISP_ERR_WORKSPACE;  // shape needs more scratch than the array

  void* ws = nullptr;
  int rc = scratch_address(&ws);
  if (rc != CRISP_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto at = [&](size_t off) { return static_cast<uint8_t*>(ws) + off; };

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
  a.status = device_status != nullptr ? device_status : reinterpret_cast<int*>(at(w.status));
  a.trace = reinterpret_cast<unsigned long long*>(at(w.trace));
  a.part = reinterpret_cast<float2*>(at(w.part));
  a.chunk_max = reinterpret_cast<float*>(at(w.chunk_max));
  a.chunk_tot = reinterpret_cast<float*>(at(w.chunk_tot));
  a.row_w = reinterpret_cast<float*>(at(w.row_w));
  a.pv = reinterpret_cast<double*>(at(w.pv));
  a.ps_lo = reinterpret_cast<double*>(at(w.ps_lo));
  a.ps_hi = reinterpret_cast<double*>(at(w.ps_hi));
  a.ps_x = reinterpret_cast<double*>(at(w.ps_x));
  a.rec_extra = reinterpret_cast<float*>(at(w.rec_extra));
  a.kbar = reinterpret_cast<float*>(at(w.kbar));
  a.qbar = reinterpret_cast<float*>(at(w.qbar));
  a.pbuf = reinterpret_cast<float*>(at(w.pbuf));
  a.hist_cnt = reinterpret_cast<uint32_t*>(at(w.hist_cnt));
  a.hist_mass = reinterpret_cast<unsigned long long*>(at(w.hist_mass));
  a.cut = reinterpret_cast<CutState*>(at(w.cut));
  a.keep_v = at(w.keep_v);
  a.keep_s = at(w.keep_s);
  a.cnt = reinterpret_cast<int*>(at(w.cnt));
  a.eqcnt = reinterpret_cast<int*>(at(w.eqcnt));
  a.eqbase = reinterpret_cast<int*>(at(w.eqbase));
  a.selmask = reinterpret_cast<uint32_t*>(at(w.selmask));
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.route = out->route;
  a.c_struct = out->c_struct;
  a.row_ptr = out->row_ptr;
  a.cols = out->cols;
  a.debug = out->debug;

  CUtensorMap qm, km;
  rc = encode_heads(&qm, q, (uint64_t)n, (uint64_t)h_q);
  if (rc == CRISP_OK) rc = encode_heads(&km, k, (uint64_t)n, (uint64_t)h_kv);
  if (rc != CRISP_OK) return rc;
  // The array keeps the previous call's contents: clear what the kernels accumulate into.
  if (cudaMemsetAsync(at(w.status), 0, 256, st) != cudaSuccess ||
      cudaMemsetAsync(a.hist_cnt, 0, (size_t)h_q * kHistBins * 4, st) != cudaSuccess ||
      cudaMemsetAsync(a.hist_mass, 0, (size_t)h_q * kHistBins * 8, st) != cudaSuccess ||
      cudaMemsetAsync(a.cut, 0, (size_t)h_q * sizeof(CutState), st) != cudaSuccess)
    return CRISP_ERR_CUDA;
  if (launch_proxy_pass(qm, km, a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  if (launch_route_threshold(a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  if (launch_pe(a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  if (launch_merge(a, st) != cudaSuccess) return CRISP_ERR_CUDA;
  return CRISP_OK;
}
