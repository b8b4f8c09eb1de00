// veda_tile_scores_noalloc: the tile-score step for callers that may not
// allocate device memory at all, not even through their own allocator. Some
// host applications load this library as a plug-in and own every byte of
// device memory themselves (a fixed pool planned ahead of time), and
// real-time loops are not allowed to call into an allocator between frames;
// both can still pass their inputs and outputs, but not a scratch buffer.
//
// The scratch that veda_tile_scores takes from its caller (the query and key
// embeddings between the MLP and the score GEMM) lives here instead in a
// file-scope device array of VEDA_NOALLOC_SCRATCH_BYTES. Every GPU that loads
// the library keeps that array until the process exits. All calls share it:
// calls whose kernels can overlap on the GPU (different streams, or different
// host threads) race on it and must be serialised by the caller. Nothing in
// it needs clearing between calls: each call overwrites every embedding it
// reads before reading it.
#include <mutex>

#include "veda_internal.cuh"

namespace veda {
void set_last_error(const char* fmt, ...);
}

#define VEDA_NOALLOC_SCRATCH_BYTES (16u << 20)
#define VEDA_NOALLOC_MAX_DEVICES 64

namespace {

static __device__ __align__(256) unsigned char g_scores_scratch[VEDA_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[VEDA_NOALLOC_MAX_DEVICES] = {};

// Device address of this device's copy of the array. In host code the array's
// name only stands for it; the address comes from cudaGetSymbolAddress, called
// once per device with that device current (first call on each device). With
// lazy module loading that first lookup is also what loads this module on the
// device, and with it reserves the array. The address is cached for the life
// of the process: a cudaDeviceReset would leave it stale, so the entry point
// is documented as unsupported across one.
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= VEDA_NOALLOC_MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scores_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int veda_tile_scores_noalloc(const veda_layer* L, const float* dq, const float* dk, const float* w1q,
                                        const float* b1q, const float* w2q, const float* b2q, const float* w1k,
                                        const float* b1k, const float* w2k, const float* b2k, int32_t hidden,
                                        int32_t out_dim, float scale, float* scores, cudaStream_t stream) {
  const size_t need = veda_tile_scores_ws_bytes(L, out_dim);
  if (need == 0) {
    const int rc = veda_layout(L, nullptr, nullptr, nullptr, nullptr);  // reports a bad layer
    if (rc != VEDA_OK) return rc;
    veda::set_last_error("out_dim=%d must be a multiple of 4 in [4, 128]", out_dim);
    return VEDA_ERR_UNSUPPORTED;
  }
  if (need > VEDA_NOALLOC_SCRATCH_BYTES) {
    veda::set_last_error(
        "veda_tile_scores_noalloc: the embeddings need %zu bytes, more than the built-in %u-byte scratch "
        "(2*B*heads*nt_cap*out_dim*4 bytes must fit); use veda_tile_scores with a caller buffer",
        need, (unsigned)VEDA_NOALLOC_SCRATCH_BYTES);
    return VEDA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  const cudaError_t e = scratch_for_current_device(&ws);
  if (e != cudaSuccess) {
    veda::set_last_error("veda_tile_scores_noalloc: scratch address: %s", cudaGetErrorString(e));
    return VEDA_ERR_CUDA;
  }
  return veda_tile_scores(L, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden, out_dim, scale, scores,
                          static_cast<float*>(ws), stream);
}
