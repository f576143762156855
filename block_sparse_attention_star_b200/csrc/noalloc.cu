// Decode without caller-provided scratch.
//
// star_decode_step needs a workspace for its per-chunk (O, LSE) partials, which
// the caller normally allocates once and passes in.  Some callers cannot call
// cudaMalloc at all: a serving runtime that reserves every byte of device memory
// for its own pool at start-up and allows no allocation afterwards, or a plugin
// that is handed only its input and output buffers by a host application that
// owns the allocator.  star_decode_step_noalloc serves them: the partials live in
// the file-scope device array below, which exists on every GPU that loads this
// library, for as long as the process runs.
//
// Host code must not pass the array's name to a kernel (on the host it names a
// host-side shadow, not device memory).  The device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first call
// made on it.
#include "star.h"
#include "common.cuh"
#include "internal.h"

#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

namespace {

// 16 MiB.  The decode step keeps at most 8 work items per CTA, so its chunk
// partials are bounded by the item count, not by the cache length: 0.61 MB for the
// Llama-3.1-8B shapes at 32K, 128K and 1M tokens, 2.4 MB for two 70B sequences.
constexpr size_t kNoAllocScratchBytes = 16u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_lock;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once).
// The lookup is not allowed while `stream` is being captured into a CUDA graph, so
// a first call made during a capture is refused with a message instead.
int scratch_for_current_device(cudaStream_t stream, void** out, char* why, size_t why_len) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(why, why_len, "cudaGetDevice: %s", cudaGetErrorString(e));
    return STAR_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(why, why_len, "device ordinal %d is beyond the %d devices this entry point tracks", dev, kMaxDevices);
    return STAR_ERR_UNSUPPORTED_SHAPE;
  }
  std::lock_guard<std::mutex> g(g_lock);
  if (!g_scratch_addr[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) {
      snprintf(why, why_len, "cudaStreamIsCapturing: %s", cudaGetErrorString(e));
      return STAR_ERR_CUDA;
    }
    if (cap != cudaStreamCaptureStatusNone) {
      snprintf(why, why_len,
               "the first star_decode_step_noalloc call on device %d was made during stream capture; make one "
               "call on this device before capturing",
               dev);
      return STAR_ERR_INVALID_ARG;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      snprintf(why, why_len, "cudaGetSymbolAddress of the decode scratch failed: %s", cudaGetErrorString(e));
      return STAR_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return STAR_OK;
}

thread_local char g_why[256];

}  // namespace

extern "C" int star_decode_step_noalloc(const star_shape* shape, const star_cache* cache, const void* q,
                                        const void* k, const void* v, const int32_t* pos, int32_t cur_len, void* out,
                                        float* lse_out, star_stream_t stream) {
  size_t need = 0;
  int rc = star_workspace_size(shape, STAR_OP_DECODE, 0, &need);
  if (rc != STAR_OK) return rc;  // star_last_error() already describes the shape problem
  if (need > kNoAllocScratchBytes) {
    snprintf(g_why, sizeof(g_why),
             "decode partials need %zu bytes, more than the %zu-byte built-in scratch of "
             "star_decode_step_noalloc; use star_decode_step with a caller workspace",
             need, kNoAllocScratchBytes);
    return star::set_last_error(STAR_ERR_CAPACITY, g_why);
  }
  void* scratch = nullptr;
  rc = scratch_for_current_device((cudaStream_t)stream, &scratch, g_why, sizeof(g_why));
  if (rc != STAR_OK) return star::set_last_error(rc, g_why);
  // Every partial the merge reads is written by the same call first, so nothing in
  // the array has to start at zero.
  return star_decode_step(shape, cache, q, k, v, pos, cur_len, out, lse_out, scratch, kNoAllocScratchBytes, stream);
}
