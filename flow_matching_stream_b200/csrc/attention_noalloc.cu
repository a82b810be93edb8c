// krea2_gqa_attention_noalloc: the GQA attention entry point for callers that cannot allocate
// device memory.
//
// krea2_gqa_attention needs a caller workspace, where it writes the RMS-normalised, rotated
// q|k before the flash-attention core reads them. Some callers cannot provide one: a plugin
// interface that hands the library only the input and output buffers, or a runtime whose
// allocator owns all device memory and forbids side allocations while it serves. This variant
// keeps that scratch in a file-scope device array of fixed size instead. It runs the same
// kernels, so its results equal krea2_gqa_attention's.
//
// The array (KREA2_NOALLOC_SCRATCH_BYTES) stays resident on every GPU that loads this part of
// the library, until the process exits. Host code cannot use the array's name as a device
// address: the first call on each device looks the address up with cudaGetSymbolAddress while
// that device is current, and caches it; the stream must belong to the current device. All
// calls share the array, so calls that overlap on the GPU (for example on two streams) race on
// it. Nothing in it needs to start at zero: the prep kernel writes every element the attention
// core reads, on every call.
#include <mutex>

#include "krea2_internal.h"

namespace krea2 {
namespace {

__device__ __align__(256) unsigned char g_attn_scratch[KREA2_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[MAX_DEVICES] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device). The
// kernels run on `stream`, so the stream must belong to that device: a stream of another GPU
// would make them use this device's array from that GPU.
int scratch_on_current_device(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= MAX_DEVICES) return set_error(KREA2_ERR_UNSUPPORTED, "device ordinal %d is out of range", dev);
  int stream_dev = -1;
  e = cudaStreamGetDevice(stream, &stream_dev);
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "cudaStreamGetDevice failed: %s", cudaGetErrorString(e));
  if (stream_dev != dev)
    return set_error(KREA2_ERR_ARG, "the stream belongs to device %d but device %d is current; make the stream's "
                     "device current before the call", stream_dev, dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess || !p)
      return set_error(KREA2_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed on device %d: %s", dev,
                       cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KREA2_OK;
}

}  // namespace
}  // namespace krea2

using namespace krea2;

extern "C" int krea2_gqa_attention_noalloc(const Krea2Dims* dims, int B, int T, int N, int dtype, const void* qkvg,
                                           const float* q_norm_w, const float* k_norm_w, const float* cos,
                                           const float* sin, const uint8_t* text_mask, void* out, void* stream) {
  // 0 for invalid arguments (the wrapped call then reports them) and for the SIMT path
  const size_t need = krea2_attention_workspace_size(dims, B, T, N, dtype);
  if (need > KREA2_NOALLOC_SCRATCH_BYTES)
    return set_error(KREA2_ERR_WORKSPACE,
                     "attention without allocation needs %zu bytes of scratch for B=%d, S=%d, but the static "
                     "scratch holds %zu; use krea2_gqa_attention with a caller workspace",
                     need, B, T + N, (size_t)KREA2_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (need) {
    int rc = scratch_on_current_device(reinterpret_cast<cudaStream_t>(stream), &scratch);
    if (rc) return rc;
  }
  return krea2_gqa_attention(dims, B, T, N, dtype, qkvg, q_norm_w, k_norm_w, cos, sin, text_mask, out, scratch,
                             need, stream);
}
