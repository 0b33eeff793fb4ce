// kvq_sparse_decode_attn_noalloc: the sparse decode attention of kvq_sparse_decode_attn
// with its split-K scratch held in this library's own static device memory, for callers
// that cannot allocate device memory at decode time.
//
// Who needs it: a serving engine that hands (nearly) all device memory to its own KV
// page pool at start-up has no allocator left to call when a decode step runs, and a
// plugin loaded into another runtime may have no allocation hook at all; cudaMalloc on
// the decode path would also synchronise the device.  Such callers still pass their
// inputs and outputs; the scratch comes from the array below.
//
// The array lives in every GPU that loads the library, for the life of the process.
// Host code cannot pass the array's name to a kernel (on the host it is a stand-in, not
// a device address), so its device address is looked up with cudaGetSymbolAddress while
// the device is current: on every call made outside a stream capture (so a context that
// was reset and re-created gets the new address), and from the last such lookup during a
// capture.  Make the first call on each device before any stream capture.  Every call
// shares the array, which keeps the last call's contents: each call clears the
// per-segment arrival counters at its head (an asynchronous memset on the caller's
// stream; the split-K partials behind them are rewritten before they are read).  Two
// calls whose work overlaps on the GPU (different streams) race on the scratch.
#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_attn_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_attn_scratch on the current device: looked up again on every call
// outside a stream capture, taken from the last lookup while `stream` is capturing.
cudaError_t scratch_address(int device, cudaStream_t stream, void** out) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const bool capturing = cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!capturing || g_scratch_addr[device] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return cudaSuccess;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

size_t kvq_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

kvq_status kvq_sparse_decode_attn_noalloc(const kvq_cache* cache, const void* q, const int32_t* sel,
                                          const int32_t* cnt, int32_t kmax, float sm_scale, void* out,
                                          float* lse, kvq_stream_t stream) {
  size_t need = 0;
  kvq_status st = kvq_workspace_size(cache, kmax, &need);
  if (st != KVQ_OK) return st;
  const long long segments = (long long)cache->B * cache->Hkv;
  if (segments >= kMaxSegments) return KVQ_ERR_UNSUPPORTED;   // as kvq_sparse_decode_attn
  if (need > kNoAllocScratchBytes) return KVQ_ERR_WORKSPACE;  // batch too large for the static scratch
  if (q == nullptr || sel == nullptr || cnt == nullptr || out == nullptr || !(sm_scale > 0.f))
    return KVQ_ERR_INVALID_ARG;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return KVQ_ERR_CUDA;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  if (scratch_address(device, s, &scratch) != cudaSuccess) return KVQ_ERR_CUDA;
  // the arrival counters start at zero whatever an earlier call left behind
  if (cudaMemsetAsync(scratch, 0, (size_t)segments * sizeof(unsigned), s) != cudaSuccess) return KVQ_ERR_CUDA;
  return kvq_sparse_decode_attn(cache, q, sel, cnt, kmax, sm_scale, out, lse, scratch, kNoAllocScratchBytes,
                                stream);
}

}  // extern "C"
