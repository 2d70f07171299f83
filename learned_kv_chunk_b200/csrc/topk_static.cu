// topk_static.cu -- fm_select_topk_static: the top-K keep mask of
// fm_select_topk with its scratch memory compiled into the library, for
// callers that cannot allocate device memory.
//
// Who cannot allocate: a serving process that hands all free device memory to
// its KV-cache pool at start-up has nothing left for cudaMalloc when a decode
// step runs; a plugin hosted inside another framework must leave device memory
// to that framework's allocator and may not call cudaMalloc at all; and
// cudaMalloc / cudaFree may synchronise the device, which a per-token decode
// loop cannot afford.  Such callers pass only inputs and outputs; the scratch
// (row states, digit histograms, tie counts) lives in the array below.
//
// The array is one per GPU that loads the library and stays allocated until
// the process exits.  Every call on a device shares it: calls whose kernels
// overlap on the GPU (two streams, two threads) race on it and produce wrong
// masks, so a caller must order them (one stream, or events).  Nothing needs
// to be cleared by the host: the first kernel of every call zeroes the row
// states and histograms it uses, whatever the previous call left there.
#include <mutex>

#include "fm_internal.cuh"

// The scratch.  In host code this name is only a host-side stand-in for the
// device variable, never a device address: its address is obtained per device
// with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char fm_topk_scratch[FM_TOPK_STATIC_SCRATCH_BYTES];

namespace fm {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// A failed runtime call: its error is the runtime's last error, which
// check_launch records for fm_last_cuda_error.
fm_status runtime_fail() {
  const fm_status s = check_launch();
  return s != FM_OK ? s : FM_ERR_CUDA;
}

// Device address of the scratch on the calling thread's current device; looked
// up on the first call on each device (with that device current) and cached.
fm_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return runtime_fail();
  if (dev < 0 || dev >= kMaxDevices) return FM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, fm_topk_scratch) != cudaSuccess) return runtime_fail();
    if (p == nullptr) return FM_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FM_OK;
}

}  // namespace
}  // namespace fm

using namespace fm;

extern "C" fm_status fm_select_topk_static(const float* ens, const int32_t* n_valid, int B, int N,
                                           int k, uint8_t* keep, cudaStream_t stream) {
  if (!ens || !keep || B < 1 || N < 1 || k < 1 || B > 65535) return FM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ens) & 3u) != 0) return FM_ERR_ALIGNMENT;
  if (topk_workspace_bytes(B, N) > (size_t)FM_TOPK_STATIC_SCRATCH_BYTES) return FM_ERR_UNSUPPORTED;
  void* ws = nullptr;
  const fm_status st = scratch_address(&ws);
  if (st != FM_OK) return st;
  return launch_topk(ens, n_valid, B, N, k, keep, ws, (size_t)FM_TOPK_STATIC_SCRATCH_BYTES, stream);
}
