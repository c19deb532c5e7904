// noalloc.cu — index selection that allocates nothing, for callers that must not call
// cudaMalloc: code that runs under a memory manager that owns every device byte (a serving
// engine's pre-reserved pool), and latency-critical paths where an allocation's implicit device
// synchronisation is not acceptable. The scratch lives in one file-scope device array instead of
// a caller-provided workspace; inputs, outputs and the optional status word stay the caller's.
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

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace crisp

using namespace crisp;

extern "C" int crisp_select_noalloc(const void* q, const void* k, int h_q, int h_kv, int n, int d,
                                    const crisp_params* p, const crisp_index* out, int* device_status,
                                    void* stream) {
  // the same checks as crisp_select, then the size of the array instead of a workspace
  Shape s;
  int rc = check_shape(h_q, h_kv, n, d, &s);
  if (rc == CRISP_OK) rc = check_params(p);
  if (rc == CRISP_OK && (s.nb > kMaxSelectBlocks || n < kB)) rc = CRISP_ERR_UNSUPPORTED;
  if (rc == CRISP_OK && (q == nullptr || k == nullptr || !is_aligned(q, 16) || !is_aligned(k, 16)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc == CRISP_OK && (out == nullptr || out->route == nullptr || out->c_struct == nullptr ||
                         out->row_ptr == nullptr || out->cols == nullptr || !is_aligned(out->row_ptr, 4) ||
                         !is_aligned(out->cols, 4)))
    rc = CRISP_ERR_INVALID_ARG;
  if (rc != CRISP_OK) return rc;
  if (workspace_layout(s).total > kNoAllocScratchBytes) return CRISP_ERR_WORKSPACE;  // needs more than the array

  void* ws = nullptr;
  rc = scratch_address(&ws);
  if (rc != CRISP_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the status word in it starts from zero here,
  // and the selection sequence clears what its kernels accumulate into.
  if (device_status == nullptr && cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return CRISP_ERR_CUDA;
  return run_select(q, k, s, p, *out, ws, device_status, st);
}
