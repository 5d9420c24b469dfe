// bsa_decode_noalloc: the decode attention step for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: code that runs inside a host
// framework which owns every device allocation and hands out no scratch, plugins
// loaded into a process whose memory budget was fixed when it started, or paths
// where a cudaMalloc would stall or synchronise the device at the wrong moment.
// For them this entry point keeps the split-K partials of bsa_decode in a
// file-scope device array of fixed size, BSA_NOALLOC_SCRATCH_BYTES, that the
// CUDA runtime reserves on every device where this library's code is loaded and
// keeps until the process exits. Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
//
// Every call made outside stream capture looks up the array's device address
// on the current device with cudaGetSymbolAddress and remembers it per device,
// so a context that was reset and re-created gets its own address. A call whose
// stream is capturing cannot make that lookup part of a graph and uses the
// address remembered by the last uncaptured call on the device: make one call
// before capturing (a capture with none returns BSA_ERR_UNSUPPORTED). Every call
// on a device shares the one array,
// so calls whose work overlaps on the GPU (different streams, or concurrent host
// threads) race on it: serialise them. The array keeps whatever the last call
// wrote; the decode kernels write every partial they later read, so nothing has
// to be cleared between calls.
#include <mutex>

#include "bsa_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[BSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device: looked up again on
// every call outside stream capture, taken from the last lookup while capturing.
bsa_status_t scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return bsa::record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return bsa::record_cuda_error(e);
  std::lock_guard<std::mutex> lock(g_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr)
      return bsa::record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    g_scratch_addr[dev] = p;
  } else if (g_scratch_addr[dev] == nullptr) {
    return BSA_ERR_UNSUPPORTED;
  }
  *out = g_scratch_addr[dev];
  return BSA_OK;
}

}  // namespace

extern "C" bsa_status_t bsa_decode_noalloc(const bsa_problem_t* prob, const void* q,
                                           bsa_cache_t k, bsa_cache_t v, const int32_t* kept,
                                           const int32_t* kept_count, void* o, float* lse,
                                           float* o_f32, int32_t* dev_status, void* stream) {
  size_t need = 0;
  bsa_status_t st = bsa_workspace_size(prob, BSA_OP_DECODE, &need);
  if (st != BSA_OK) return st;
  if (need > static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES)) return BSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = scratch_address(static_cast<cudaStream_t>(stream), &scratch)) != BSA_OK) return st;
  return bsa_decode(prob, q, k, v, kept, kept_count, o, lse, o_f32, scratch,
                    static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES), dev_status, stream);
}
