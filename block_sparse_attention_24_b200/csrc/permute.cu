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
// Each valid row of the tile (one token's slice of this head: D bf16, a
// 16-byte multiple) is copied into shared memory by cp.async.bulk on one
// mbarrier, so a CTA keeps its whole tile in flight with few registers; the
// padding rows are zeroed in shared memory; one bulk store writes the tile to
// its contiguous permuted slots; the descriptor is reduced from shared
// memory, 256 threads over channel pairs x row groups, combined in a fixed
// order. (Holding the rows in registers took 61 registers a thread, 4 CTAs
// per SM, and was 5% slower.)
__device__ __forceinline__ void bulk_load_row(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_store_tile(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(smem_src)),
               "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

template <int VPR>
__global__ void __launch_bounds__(256) permute_pool_kernel(const __grid_constant__ LayerGeom g,
                                                                const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                int32_t* __restrict__ perm, float* __restrict__ desc) {
  constexpr int D = VPR * 8;
  constexpr uint32_t RB = D * 2;         // bytes per row
  constexpr int NCP = D / 2;             // channel pairs
  constexpr int NG = 256 / NCP;          // row groups
  extern __shared__ __align__(128) uint8_t rows_sm[];  // [tile][D] bf16
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  __shared__ float part[NG][6][NCP];
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
  const int nv = tile_len(hg, g.T, tid);  // the valid rows are a prefix of the tile
  const int tt = tid / hg.tps;
  const int rem = tid - tt * hg.tps;
  const int th = rem / hg.nwt;
  const int tw = rem - th * hg.nwt;
  const int t0 = tt * hg.pt;
  const int n0 = (t0 * g.H + th * hg.ph) * g.W + tw * hg.pw;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    s_abort = 0;
    fence_mbar_init();
    mbar_expect_tx(&bar, (uint32_t)nv * RB);
  }
  __syncthreads();  // the expected bytes are registered before any copy can complete
  if (threadIdx.x < tile) {
    const int loc = threadIdx.x;
    const int slab = hg.ph * hg.pw;
    const int lt = loc / slab;
    const int lr = loc - lt * slab;
    const int ly = lr / hg.pw;
    const int lx = lr - ly * hg.pw;
    const int n = n0 + (lt * g.H + ly) * g.W + lx;
    if (loc < nv) {
      bulk_load_row(rows_sm + loc * RB, src + (((long long)b * N + n) * g.heads + h) * VPR, RB, &bar);
    } else {
      uint4* z = reinterpret_cast<uint4*>(rows_sm + loc * RB);
#pragma unroll
      for (int e = 0; e < VPR; ++e) z[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (perm && b == 0) perm[(long long)h * g.n_cap + tid * tile + loc] = loc < nv ? n : -1;
  }
  if (!mbar_wait(&bar, 0, &s_abort, g.dev_status)) {
    mbar_wait_drain(&bar, 0, VEDA_WAIT_LIMIT_NS);  // let the copies into this CTA's memory land
    return;
  }
  fence_proxy_async_smem();  // the zeroed padding rows, before the bulk store reads them
  __syncthreads();
  if (threadIdx.x == 0) bulk_store_tile(dst + slot0 * VPR, rows_sm, (uint32_t)tile * RB);
  const int cp = threadIdx.x % NCP, grp = threadIdx.x / NCP;
  float s0 = 0.f, s1 = 0.f, hi0 = -INFINITY, hi1 = -INFINITY, lo0 = INFINITY, lo1 = INFINITY;
  for (int r = grp; r < nv; r += NG) {
    const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(rows_sm + r * RB)[cp]);
    s0 += f.x;
    s1 += f.y;
    hi0 = fmaxf(hi0, f.x);
    hi1 = fmaxf(hi1, f.y);
    lo0 = fminf(lo0, f.x);
    lo1 = fminf(lo1, f.y);
  }
  part[grp][0][cp] = s0;
  part[grp][1][cp] = s1;
  part[grp][2][cp] = hi0;
  part[grp][3][cp] = hi1;
  part[grp][4][cp] = lo0;
  part[grp][5][cp] = lo1;
  __syncthreads();
  if (threadIdx.x < NCP) {
    float S0 = part[0][0][cp], S1 = part[0][1][cp], H0 = part[0][2][cp], H1 = part[0][3][cp];
    float L0 = part[0][4][cp], L1 = part[0][5][cp];
#pragma unroll
    for (int q = 1; q < NG; ++q) {  // fixed order: bit-reproducible
      S0 += part[q][0][cp];
      S1 += part[q][1][cp];
      H0 = fmaxf(H0, part[q][2][cp]);
      H1 = fmaxf(H1, part[q][3][cp]);
      L0 = fminf(L0, part[q][4][cp]);
      L1 = fminf(L1, part[q][5][cp]);
    }
    const float cnt = (float)nv;
    out[2 * cp] = S0 / cnt;
    out[2 * cp + 1] = S1 / cnt;
    out[D + 2 * cp] = H0;
    out[D + 2 * cp + 1] = H1;
    out[2 * D + 2 * cp] = L0;
    out[2 * D + 2 * cp + 1] = L1;
  }
  if (threadIdx.x == 0) bulk_wait_read_all();  // the tile stays in shared memory until the store has read it
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
  const size_t smem = (size_t)g.tile * g.d * 2;
  if (g.d == 128)
    permute_pool_kernel<16><<<grid, 256, smem, s>>>(g, (const uint4*)x, (uint4*)xp, perm, desc);
  else
    permute_pool_kernel<8><<<grid, 256, smem, s>>>(g, (const uint4*)x, (uint4*)xp, perm, desc);
  return cudaGetLastError();
}

}  // namespace veda
