// Head-aware tiling permutation (Veda summary 2.2, Head-Aware Tiling).
//
// Forward: x [B,N,heads,d] -> xp [B,heads,n_cap,d]; inverse: xp -> x.
// One CTA moves one tile (64 or 128 rows of d bf16) of one head. The CTA
// first tabulates, for each in-tile position, its offset from the tile's
// origin in the original grid; after that each row costs one shared-memory
// lookup. Each thread moves 16-byte vectors, so every row (128 or 256 bytes)
// is read and written as whole 32-byte sectors. HBM-bound: 2*d*2 bytes per
// row moved.
#include "veda_internal.cuh"

namespace veda {
namespace {

template <int VPR>  // 16-byte vectors per row (d*2/16)
__global__ void __launch_bounds__(256) permute_kernel(const __grid_constant__ LayerGeom g, const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, int32_t* __restrict__ perm,
                                                      int inverse) {
  __shared__ int s_off[128];
  __shared__ int s_lt[128];
  const int tid = blockIdx.x;  // tile of head h
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const HeadGeom& hg = g.h[h];
  const int tile = g.tile;
  const long long N = (long long)g.T * g.H * g.W;
  const long long slot0 = ((long long)b * g.heads + h) * g.n_cap + (long long)tid * tile;  // permuted row

  if (tid >= hg.nt) {  // tiles beyond this head's count are padding
    if (!inverse) {
      for (int i = threadIdx.x; i < tile * VPR; i += blockDim.x) dst[slot0 * VPR + i] = make_uint4(0u, 0u, 0u, 0u);
      if (perm && b == 0)
        for (int i = threadIdx.x; i < tile; i += blockDim.x) perm[(long long)h * g.n_cap + tid * tile + i] = -1;
    }
    return;
  }
  const int slab = hg.ph * hg.pw;
  if (threadIdx.x < tile) {
    const int loc = threadIdx.x;
    const int lt = loc / slab;
    const int lr = loc - lt * slab;
    const int ly = lr / hg.pw;
    const int lx = lr - ly * hg.pw;
    s_lt[loc] = lt;
    s_off[loc] = (lt * g.H + ly) * g.W + lx;
  }
  const int tt = tid / hg.tps;
  const int rem = tid - tt * hg.tps;
  const int th = rem / hg.nwt;
  const int tw = rem - th * hg.nwt;
  const int t0 = tt * hg.pt;
  const int n0 = (t0 * g.H + th * hg.ph) * g.W + tw * hg.pw;
  __syncthreads();

  constexpr int RPP = 256 / VPR;  // rows per pass
  const int v = threadIdx.x % VPR;
  for (int r = threadIdx.x / VPR; r < tile; r += RPP) {
    const bool valid = t0 + s_lt[r] < g.T;
    const int n = n0 + s_off[r];
    const long long prow = slot0 + r;                                       // row in xp
    const long long orow = ((long long)b * N + n) * g.heads + h;            // row in x
    if (!inverse) {
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (valid) val = __ldg(src + orow * VPR + v);
      dst[prow * VPR + v] = val;
      if (perm && b == 0 && v == 0) perm[(long long)h * g.n_cap + tid * tile + r] = valid ? n : -1;
    } else if (valid) {
      dst[orow * VPR + v] = __ldg(src + prow * VPR + v);
    }
  }
}

}  // namespace

cudaError_t launch_permute(const LayerGeom& g, const void* x, void* xp, int32_t* perm, int inverse, cudaStream_t s) {
  const dim3 grid(g.nt_cap, g.heads, g.B);
  const uint4* src = (const uint4*)(inverse ? xp : x);
  uint4* dst = (uint4*)(inverse ? x : xp);
  if (g.d == 128)
    permute_kernel<16><<<grid, 256, 0, s>>>(g, src, dst, perm, inverse);
  else
    permute_kernel<8><<<grid, 256, 0, s>>>(g, src, dst, perm, inverse);
  return cudaGetLastError();
}

}  // namespace veda
