// Decode step for callers that cannot allocate device memory.
//
// Some callers of this library never call cudaMalloc themselves: code that
// runs inside a framework whose caching allocator owns all device memory (a
// private cudaMalloc there can fail once the pool has reserved the GPU, and it
// bypasses the framework's accounting), engines that capture their decode
// loop into CUDA graphs and must not allocate between captures, and plugin
// hosts that hand a kernel only its input and output pointers. For them,
// resa_decode_sparse_noalloc keeps its scratch in a fixed array that lives in
// the library's own device memory.
//
// The array is a file-scope __device__ variable of kScratchBytes: every GPU
// that loads libresa.so holds it until the process exits. In host code its
// name only stands in for the symbol, so the device address is looked up with
// cudaGetSymbolAddress once per device (on that device's first call) and
// cached. A failed call drops the cached address, so a context rebuilt after
// cudaDeviceReset looks it up again.
//
// The array's first 256 bytes are the same control block a caller workspace
// starts with: its error word is sticky across calls (a timed-out wait or a
// bad block id raised by one call stays set until resa_noalloc_status reads
// and clears it); the arrival counters after it are cleared by every call.
#include <mutex>

#include "../../include/resa.h"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = 16ull << 20;   // 16 MiB per GPU
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {nullptr};

// device address of g_scratch on the current device (nullptr on failure)
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) return nullptr;
    g_addr[dev] = p;
  }
  return g_addr[dev];
}

// forget the current device's cached address (after a CUDA failure)
void drop_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lk(g_mu);
  g_addr[dev] = nullptr;
}

}  // namespace

extern "C" {

int resa_decode_sparse_noalloc(const resa_dims* dims, const void* q, const void* k_new,
                               const void* v_new, void* k_cache, void* v_cache, void* desc,
                               int64_t len, double r, int32_t n_min, float softmax_scale,
                               void* out, float* lse, int32_t* sel, void* stream) {
  const size_t need = resa_workspace_bytes(dims, len, 0);
  if (need == 0) return RESA_ERR_INVALID_ARG;
  if (need > kScratchBytes) return RESA_ERR_WORKSPACE;
  resa::Shape s;
  s.B = dims->batch;
  s.H = dims->n_kv_heads;
  s.Hq = dims->n_q_heads;
  s.G = dims->n_q_heads / dims->n_kv_heads;
  s.D = dims->head_dim;
  s.L_max = dims->max_len;
  s.Mmax = static_cast<int>(dims->max_len / 16);
  s.bf16 = dims->dtype == RESA_BF16;
  void* ws = scratch_address();
  if (ws == nullptr) return RESA_ERR_CUDA;
  // the arrival counters must start at zero; the error word (the first bytes
  // of the control block) is left for resa_noalloc_status to read
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t zero_end = resa::workspace_zero_prefix(s);
  if (cudaMemsetAsync(static_cast<unsigned char*>(ws) + resa::kCtrlBytes, 0,
                      zero_end - resa::kCtrlBytes, st) != cudaSuccess) {
    drop_scratch_address();
    return RESA_ERR_CUDA;
  }
  const int rc = resa_decode_sparse(dims, q, k_new, v_new, k_cache, v_cache, desc, len, r, n_min,
                                    softmax_scale, out, lse, sel, ws, kScratchBytes, stream);
  if (rc == RESA_ERR_CUDA) drop_scratch_address();
  return rc;
}

int resa_noalloc_status(void* stream) {
  void* ws = scratch_address();
  if (ws == nullptr) return RESA_ERR_CUDA;
  const int rc = resa_workspace_status(ws, stream);
  if (rc == RESA_ERR_CUDA) drop_scratch_address();
  return rc;
}

}  // extern "C"
