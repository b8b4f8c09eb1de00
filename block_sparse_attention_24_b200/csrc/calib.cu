// Calibration metric for the head-aware tiling search (Veda summary 2.2:
// each head's tiling is chosen offline to fit its locality): per head, the
// squared Frobenius distance between two attention outputs in the original
// token order, e.g. full attention and the tile-skipping result under one
// candidate tiling.
//
// One CTA per head reads both tensors once (16-byte vectors, two rows of
// d = 128 per warp pass); each thread accumulates in fp32 over a fixed set
// of rows and the block combines the thread sums in fp64 in a fixed order,
// so the result is bit-reproducible. HBM-bound: 2*B*N*d*2 bytes per head.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int CAL_THREADS = 1024;

template <int VPR>
__global__ void __launch_bounds__(CAL_THREADS) output_sq_error_kernel(const __grid_constant__ LayerGeom g,
                                                                      const uint4* __restrict__ a,
                                                                      const uint4* __restrict__ b,
                                                                      float* __restrict__ err) {
  __shared__ double part[CAL_THREADS / 32];
  const int h = blockIdx.x;
  const long long N = (long long)g.T * g.H * g.W;
  const long long rows = (long long)g.B * N;
  constexpr int RPP = CAL_THREADS / VPR;  // rows per pass
  const int v = threadIdx.x % VPR;
  float acc = 0.f;
  for (long long r = threadIdx.x / VPR; r < rows; r += RPP) {
    const long long off = (r * g.heads + h) * VPR + v;  // row r = b*N + n of head h
    const uint4 ua = __ldg(a + off), ub = __ldg(b + off);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&ua);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&ub);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(pa[e]), fb = __bfloat1622float2(pb[e]);
      const float dx = fa.x - fb.x, dy = fa.y - fb.y;
      acc = fmaf(dx, dx, acc);
      acc = fmaf(dy, dy, acc);
    }
  }
  double s = acc;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) part[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < CAL_THREADS / 32; ++w) t += part[w];
    err[h] = (float)t;
  }
}

}  // namespace

cudaError_t launch_output_sq_error(const LayerGeom& g, const void* a, const void* b, float* err, cudaStream_t s) {
  if (g.d == 128)
    output_sq_error_kernel<16><<<g.heads, CAL_THREADS, 0, s>>>(g, (const uint4*)a, (const uint4*)b, err);
  else
    output_sq_error_kernel<8><<<g.heads, CAL_THREADS, 0, s>>>(g, (const uint4*)a, (const uint4*)b, err);
  return cudaGetLastError();
}

}  // namespace veda
