// TripPool tile descriptors (Veda summary 2.1, Statistic-Aware Estimator):
// per tile and channel, [mean | max | min] over the tile's valid tokens.
//
// One CTA (128 threads) reduces one tile of one head. Each thread loads
// 16-byte vectors (8 channels) from a strided set of rows and keeps running
// sum/max/min; partial results are combined with warp shuffles, then across
// warps through shared memory. HBM-bound: tile*d*2 bytes read per tile.
#include "veda_internal.cuh"

namespace veda {
namespace {

template <int D>
__global__ void __launch_bounds__(128) trippool_kernel(const __grid_constant__ LayerGeom g,
                                                       const uint4* __restrict__ xp, float* __restrict__ desc) {
  constexpr int VPR = D / 8;          // vectors per row
  constexpr int RG = 128 / VPR;       // row groups
  constexpr int GPW = 32 / VPR;       // row groups per warp
  __shared__ float part[4][VPR][24];
  const int tid = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const HeadGeom& hg = g.h[h];
  float* out = desc + (((long long)b * g.heads + h) * g.nt_cap + tid) * (3 * D);
  if (tid >= hg.nt) {
    for (int i = threadIdx.x; i < 3 * D; i += blockDim.x) out[i] = 0.f;
    return;
  }
  const int len = tile_len(hg, g.T, tid);
  const uint4* rows = xp + (((long long)b * g.heads + h) * g.n_cap + (long long)tid * g.tile) * VPR;
  const int v = threadIdx.x % VPR;
  const int rg = threadIdx.x / VPR;

  float sum[8], mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    sum[e] = 0.f;
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
  for (int r = rg; r < len; r += RG) {
    uint4 u = __ldg(rows + (long long)r * VPR + v);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(p[e]);
      sum[2 * e] += f.x;
      sum[2 * e + 1] += f.y;
      mx[2 * e] = fmaxf(mx[2 * e], f.x);
      mx[2 * e + 1] = fmaxf(mx[2 * e + 1], f.y);
      mn[2 * e] = fminf(mn[2 * e], f.x);
      mn[2 * e + 1] = fminf(mn[2 * e + 1], f.y);
    }
  }
  // combine the row groups that share a warp (lanes v, v+VPR, ...)
#pragma unroll
  for (int off = VPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], off);
      mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], off));
      mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], off));
    }
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane < VPR) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      part[warp][lane][e] = sum[e];
      part[warp][lane][8 + e] = mx[e];
      part[warp][lane][16 + e] = mn[e];
    }
  }
  __syncthreads();
  (void)GPW;
  if (threadIdx.x < D) {
    const int c = threadIdx.x, cv = c / 8, ce = c % 8;
    // fixed combination order keeps the result bit-reproducible
    float s = part[0][cv][ce], M = part[0][cv][8 + ce], m = part[0][cv][16 + ce];
#pragma unroll
    for (int w = 1; w < 4; ++w) {
      s += part[w][cv][ce];
      M = fmaxf(M, part[w][cv][8 + ce]);
      m = fminf(m, part[w][cv][16 + ce]);
    }
    out[c] = s / (float)len;
    out[D + c] = M;
    out[2 * D + c] = m;
  }
}

}  // namespace

cudaError_t launch_trippool(const LayerGeom& g, const void* xp, float* desc, cudaStream_t s) {
  const dim3 grid(g.nt_cap, g.heads, g.B);
  if (g.d == 128)
    trippool_kernel<128><<<grid, 128, 0, s>>>(g, (const uint4*)xp, desc);
  else
    trippool_kernel<64><<<grid, 128, 0, s>>>(g, (const uint4*)xp, desc);
  return cudaGetLastError();
}

}  // namespace veda
