// Head-aware tiling permutation (Veda summary 2.2, Head-Aware Tiling), and
// the same permutation fused with TripPool (summary 2.1).
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

// Forward permutation fused with TripPool (Veda summary 2.1 and 2.2): the
// CTA that moves a tile's rows also reduces them to the tile descriptor
// [mean | max | min] per channel, so the permuted tensor is never read back.
// Each thread keeps sum / max / min of its 8 channels over the valid rows it
// moves; threads holding the same channels are combined with warp shuffles
// and then across the 8 warps through shared memory in a fixed order.
template <int VPR>
__global__ void __launch_bounds__(256) permute_pool_kernel(const __grid_constant__ LayerGeom g,
                                                           const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           int32_t* __restrict__ perm, float* __restrict__ desc) {
  constexpr int D = VPR * 8;
  __shared__ int s_off[128];
  __shared__ int s_lt[128];
  __shared__ float part[8][VPR][24];
  const int tid = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const HeadGeom& hg = g.h[h];
  const int tile = g.tile;
  const long long N = (long long)g.T * g.H * g.W;
  const long long slot0 = ((long long)b * g.heads + h) * g.n_cap + (long long)tid * tile;
  float* out = desc + (((long long)b * g.heads + h) * g.nt_cap + tid) * (3 * D);

  if (tid >= hg.nt) {  // padding tile: zero rows, -1 in the map, zero descriptor
    for (int i = threadIdx.x; i < tile * VPR; i += blockDim.x) dst[slot0 * VPR + i] = make_uint4(0u, 0u, 0u, 0u);
    if (perm && b == 0)
      for (int i = threadIdx.x; i < tile; i += blockDim.x) perm[(long long)h * g.n_cap + tid * tile + i] = -1;
    if (tid < g.nt_cap)
      for (int i = threadIdx.x; i < 3 * D; i += blockDim.x) out[i] = 0.f;
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

  float sum[8], mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    sum[e] = 0.f;
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
  // all of a thread's rows are loaded before any is stored or reduced, so
  // each thread keeps up to RPT independent 16-byte loads in flight
  constexpr int RPP = 256 / VPR;  // rows per pass
  constexpr int RPT = 128 / RPP;  // rows per thread for a 128-token tile
  const int v = threadIdx.x % VPR;
  const int r0 = threadIdx.x / VPR;
  uint4 val[RPT];
  bool ok[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = r0 + i * RPP;
    ok[i] = r < tile && t0 + s_lt[r < tile ? r : 0] < g.T;
    val[i] = make_uint4(0u, 0u, 0u, 0u);
    if (ok[i]) {
      const long long orow = ((long long)b * N + n0 + s_off[r]) * g.heads + h;
      val[i] = __ldg(src + orow * VPR + v);
    }
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = r0 + i * RPP;
    if (r < tile) {
      dst[(slot0 + r) * VPR + v] = val[i];
      if (perm && b == 0 && v == 0) perm[(long long)h * g.n_cap + tid * tile + r] = ok[i] ? n0 + s_off[r] : -1;
    }
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    if (ok[i]) {
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&val[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p2[e]);
        sum[2 * e] += f.x;
        sum[2 * e + 1] += f.y;
        mx[2 * e] = fmaxf(mx[2 * e], f.x);
        mx[2 * e + 1] = fmaxf(mx[2 * e + 1], f.y);
        mn[2 * e] = fminf(mn[2 * e], f.x);
        mn[2 * e + 1] = fminf(mn[2 * e + 1], f.y);
      }
    }
  }
  // lanes v, v+VPR, ... of a warp hold the same channels
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
  if (threadIdx.x < D) {
    const int c = threadIdx.x, cv = c / 8, ce = c % 8;
    float S = part[0][cv][ce], M = part[0][cv][8 + ce], m = part[0][cv][16 + ce];
#pragma unroll
    for (int w = 1; w < 8; ++w) {  // fixed order: bit-reproducible
      S += part[w][cv][ce];
      M = fmaxf(M, part[w][cv][8 + ce]);
      m = fminf(m, part[w][cv][16 + ce]);
    }
    out[c] = S / (float)tile_len(hg, g.T, tid);
    out[D + c] = M;
    out[2 * D + c] = m;
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

cudaError_t launch_permute_pool(const LayerGeom& g, const void* x, void* xp, int32_t* perm, float* desc,
                                cudaStream_t s) {
  const dim3 grid(g.nt_cap, g.heads, g.B);
  if (g.d == 128)
    permute_pool_kernel<16><<<grid, 256, 0, s>>>(g, (const uint4*)x, (uint4*)xp, perm, desc);
  else
    permute_pool_kernel<8><<<grid, 256, 0, s>>>(g, (const uint4*)x, (uint4*)xp, perm, desc);
  return cudaGetLastError();
}

}  // namespace veda
