// Temporal caching of tile scores across diffusion steps (Veda summary 5:
// the pages name temporal caching of tile scores and adaptive sparsity across
// timesteps as future work; the rule below is this library's reading).
//
// Per (batch element, head) the call keeps the TripPool descriptors of the
// step whose scores and top-k mask are cached, and the number of steps since
// then (age). A step reuses the cached mask of a head when its descriptors
// moved little:
//   drift^2 = (|Dq - Dq_ref|^2 + |Dk - Dk_ref|^2) / (|Dq_ref|^2 + |Dk_ref|^2)
// over the head's valid tiles, and refreshes it (new scores and top-k, the
// descriptors become the reference, age 0) when the head was never scored
// (age < 0), when age + 1 >= max_age, or when drift^2 > tau^2. The decision
// stays on the device: the score and top-k kernels read the per-head flag
// and skip heads whose mask is reused, so the step needs no host round trip.
// Three small launches: chunked partial sums over ~4 CTAs per SM, the
// per-head decision (the partials summed in a fixed order, so decisions are
// reproducible), and the chunked copy of refreshed heads' descriptors.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int SC_THREADS = 256;

// Chunks per (batch element, head): enough CTAs for ~4 per SM in all.
__host__ __device__ inline int cache_chunks(const LayerGeom& g) {
  const int bh = g.B * g.heads;
  const int c = (592 + bh - 1) / bh;
  return c < 1 ? 1 : (c > 64 ? 64 : c);
}

// Element range [lo, hi) of chunk c of the n valid descriptor floats.
__device__ __forceinline__ void chunk_range(long long n, int c, int nc, long long& lo, long long& hi) {
  lo = n * c / nc;
  hi = n * (c + 1) / nc;
}

// Grid (chunks, B*heads): fp32 partial sums per thread, combined in fp64 in a
// fixed order into ws[bh][chunk] = (num, den).
__global__ void __launch_bounds__(SC_THREADS)
    cache_partial_kernel(const __grid_constant__ LayerGeom g, const float* __restrict__ dq,
                         const float* __restrict__ dk, const float* __restrict__ dq_ref,
                         const float* __restrict__ dk_ref, double2* __restrict__ ws) {
  __shared__ double red[2][SC_THREADS / 32];
  const int c = blockIdx.x, nc = gridDim.x, bh = blockIdx.y;
  const int din = 3 * g.d;
  const long long base = (long long)bh * g.nt_cap * din;
  long long lo, hi;
  chunk_range((long long)g.h[bh % g.heads].nt * din, c, nc, lo, hi);
  float num = 0.f, den = 0.f;
  for (long long i = lo + threadIdx.x; i < hi; i += SC_THREADS) {
    const float q = dq[base + i], k = dk[base + i], qr = dq_ref[base + i], kr = dk_ref[base + i];
    num = fmaf(q - qr, q - qr, num);
    num = fmaf(k - kr, k - kr, num);
    den = fmaf(qr, qr, den);
    den = fmaf(kr, kr, den);
  }
  double dn = num, dd = den;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dn += __shfl_xor_sync(0xffffffffu, dn, off);
    dd += __shfl_xor_sync(0xffffffffu, dd, off);
  }
  if (threadIdx.x % 32 == 0) {
    red[0][threadIdx.x / 32] = dn;
    red[1][threadIdx.x / 32] = dd;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double N = 0.0, D = 0.0;
    for (int w = 0; w < SC_THREADS / 32; ++w) {
      N += red[0][w];
      D += red[1][w];
    }
    ws[(long long)bh * nc + c] = make_double2(N, D);
  }
}

// One thread per (batch element, head): the chunks' sums in order, then the
// refresh decision and the new age.
__global__ void cache_decide_kernel(int n_bh, int nc, const double2* __restrict__ ws, float tau, int max_age,
                                    int32_t* __restrict__ age, int32_t* __restrict__ refresh) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= n_bh) return;
  double N = 0.0, D = 0.0;
  for (int c = 0; c < nc; ++c) {
    const double2 p = ws[(long long)bh * nc + c];
    N += p.x;
    D += p.y;
  }
  const int a = age[bh];
  const bool fresh = a < 0 || a + 1 >= max_age || !(N <= (double)tau * (double)tau * D);
  refresh[bh] = fresh ? 1 : 0;
  age[bh] = fresh ? 0 : a + 1;
}

// Grid (chunks, B*heads): refreshed heads take the step's descriptors as
// their new reference.
__global__ void __launch_bounds__(SC_THREADS)
    cache_copy_kernel(const __grid_constant__ LayerGeom g, const float* __restrict__ dq,
                      const float* __restrict__ dk, float* __restrict__ dq_ref, float* __restrict__ dk_ref,
                      const int32_t* __restrict__ refresh) {
  const int c = blockIdx.x, nc = gridDim.x, bh = blockIdx.y;
  if (!refresh[bh]) return;
  const int din = 3 * g.d;
  const long long base = (long long)bh * g.nt_cap * din;
  long long lo, hi;
  chunk_range((long long)g.h[bh % g.heads].nt * din, c, nc, lo, hi);
  for (long long i = lo + threadIdx.x; i < hi; i += SC_THREADS) {
    dq_ref[base + i] = dq[base + i];
    dk_ref[base + i] = dk[base + i];
  }
}

}  // namespace

size_t score_cache_ws_bytes(const LayerGeom& g) {
  return (size_t)g.B * g.heads * cache_chunks(g) * sizeof(double2);
}

cudaError_t launch_score_cache(const LayerGeom& g, const float* dq, const float* dk, float* dq_ref, float* dk_ref,
                               float tau, int max_age, int32_t* age, int32_t* refresh, void* ws, cudaStream_t s) {
  const int nc = cache_chunks(g), n_bh = g.B * g.heads;
  double2* w = reinterpret_cast<double2*>(ws);
  cache_partial_kernel<<<dim3(nc, n_bh), SC_THREADS, 0, s>>>(g, dq, dk, dq_ref, dk_ref, w);
  cache_decide_kernel<<<(n_bh + 127) / 128, 128, 0, s>>>(n_bh, nc, w, tau, max_age, age, refresh);
  cache_copy_kernel<<<dim3(nc, n_bh), SC_THREADS, 0, s>>>(g, dq, dk, dq_ref, dk_ref, refresh);
  return cudaGetLastError();
}

}  // namespace veda
