// clsa_topk_noalloc: the exact TopK of clsa_topk for callers that cannot
// allocate device memory.  It runs the same kernel as clsa_topk; the only
// difference is where its scratch lives.
//
// Scratch: one file-scope __device__ array of kScratchBytes (2 MiB).  Every GPU
// that loads this library holds it until the process exits.  Host code cannot
// use the array's name as a device address (on the host it names a stand-in
// object), so the device address is looked up with cudaGetSymbolAddress, once
// per device, with that device current, on the first call made there.  That
// first call should therefore happen before any stream capture.
//
// Every call shares the array and it keeps the last call's contents, so each
// call first clears the part it uses (error word, histograms, barrier state)
// with cudaMemsetAsync on the caller's stream.  Calls whose work overlaps on
// the GPU (different streams, or different host threads) race on the array.
//
// The looked-up address belongs to the device's primary context.  A process that
// destroys that context (cudaDeviceReset) must not call this entry point on that
// device again: the cached address would no longer be mapped.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;
constexpr int kMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char clsa_topk_scratch[kScratchBytes];

namespace {

std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, clsa_topk_scratch);
    if (e != cudaSuccess) return e;
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" clsa_status clsa_topk_noalloc(const float* scores, const int32_t* seq_lens, int B, int n_max, int k,
                                         int32_t* idx, int32_t* count, void* stream) {
  using namespace clsa;
  CallScope scope(stream);
  if (!scores || !seq_lens || !idx || !count || B < 1 || n_max < 1 || k < 1) return CLSA_ERR_INVALID_ARG;
  if (k > 4096) return CLSA_ERR_UNSUPPORTED;
  for (const void* p : {(const void*)scores, (const void*)seq_lens, (const void*)idx, (const void*)count})
    if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0) return CLSA_ERR_INVALID_ARG;
  const size_t need = kWsHeader + topk_ws_bytes(B, n_max, k);
  if (need > kScratchBytes) return CLSA_ERR_UNSUPPORTED;  // more rows than the fixed scratch holds
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return CLSA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return CLSA_ERR_CUDA;
  char* w = static_cast<char*>(scratch);
  return launch_topk(scores, seq_lens, B, n_max, k, idx, count, w, w + kWsHeader, s) == cudaSuccess
             ? CLSA_OK
             : CLSA_ERR_CUDA;
}
