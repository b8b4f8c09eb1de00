// Head-specific MLP estimator and tile scores (Veda summary 2.1,
// Head-Specific Projections).
//
//   emb = W2^T GELU(W1^T desc + b1) + b2   per tile, per head, for Q and K
//   scores[i, j] = scale * emb_q[i] . emb_k[j]
//
// Two kernels, both fp32 FFMA (no TF32): a register-tiled MLP kernel that
// keeps 32 tile descriptors in shared memory and streams each weight once
// per CTA, and a 64x64-tiled SGEMM for the score matrix. The embeddings live
// in the caller's scratch buffer between the two.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int MLP_ROWS = 64;                 // descriptors per CTA
constexpr int MLP_THREADS = 256;             // 8 warps
constexpr int MLP_RPT = MLP_ROWS / (MLP_THREADS / 32);  // layer-1 rows per thread (one row group per warp)
constexpr int MLP_RPT2 = 4;                  // layer-2 rows per thread (16 row groups x 16 column groups)

__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

// Shared memory of one CTA: the descriptors transposed [din][MLP_ROWS], and
// the hidden activations [hidden][MLP_ROWS], which reuse the descriptors'
// space when layer 1 is a single chunk of at most 128 units (then the
// descriptors are no longer read once the hidden units are written).
__host__ __device__ inline bool mlp_alias(int din, int hidden) { return hidden <= 128 && hidden <= din; }
__host__ __device__ inline int mlp_smem_floats(int din, int hidden) {
  return MLP_ROWS * (din + (mlp_alias(din, hidden) ? 0 : hidden));
}

// grid (ceil(nt_cap/MLP_ROWS), heads, B*2): z%2 == 0 -> query side, 1 -> key
// side. MLP_ROWS tile descriptors per CTA, kept transposed in shared memory
// (input-major) so that a thread's rows are 16-byte loads; every weight row
// is read once per CTA (the eight warps share it through L1) and feeds
// MLP_ROWS rows. Layer 1: each thread owns an MLP_RPT-row x 4-column
// register tile of a 128-unit chunk (4*MLP_RPT FMAs per 16-byte weight
// load, issued as packed fp32x2 FMAs, which round every lane like fmaf),
// GELU'd and transposed into shared memory. Layer 2: 4 rows x 4
// columns per thread over chunks of 64 outputs, so no lane idles at
// out_dim = 64. (32 rows per CTA with 4 warps streamed each weight twice as
// often per row and was L2-bound.)
__global__ void __launch_bounds__(MLP_THREADS) mlp_kernel(const __grid_constant__ LayerGeom g, const float* __restrict__ dq,
                                                          const float* __restrict__ dk, const float* __restrict__ w1q,
                                                          const float* __restrict__ b1q, const float* __restrict__ w2q,
                                                          const float* __restrict__ b2q, const float* __restrict__ w1k,
                                                          const float* __restrict__ b1k, const float* __restrict__ w2k,
                                                          const float* __restrict__ b2k, int hidden, int out_dim,
                                                          float* __restrict__ emb, const int32_t* __restrict__ head_on) {
  // head_on (may be NULL): per (batch element, head), 0 = keep the cached scores
  if (head_on && !head_on[(blockIdx.z >> 1) * g.heads + blockIdx.y]) return;
  extern __shared__ float4 sm4[];
  float* sm = reinterpret_cast<float*>(sm4);
  const int din = 3 * g.d;
  const bool alias = mlp_alias(din, hidden);
  float* xsT = sm;                                    // [din][MLP_ROWS]
  float* hsT = alias ? sm : sm + din * MLP_ROWS;      // [hidden][MLP_ROWS]
  const int h = blockIdx.y;
  const int b = blockIdx.z >> 1;
  const int side = blockIdx.z & 1;
  const int r0 = blockIdx.x * MLP_ROWS;
  const int nt = g.h[h].nt;
  const float* desc = (side ? dk : dq) + (((long long)b * g.heads + h) * g.nt_cap) * din;
  const float* W1 = (side ? w1k : w1q) + (long long)h * din * hidden;
  const float* B1 = (side ? b1k : b1q) + (long long)h * hidden;
  const float* W2 = (side ? w2k : w2q) + (long long)h * hidden * out_dim;
  const float* B2 = (side ? b2k : b2q) + (long long)h * out_dim;
  float* out = emb + ((long long)side * g.B * g.heads + (long long)b * g.heads + h) * g.nt_cap * out_dim;

  // transpose-load the descriptors: consecutive threads take consecutive rows
  for (int i = threadIdx.x; i < MLP_ROWS * (din / 4); i += MLP_THREADS) {
    const int r = i % MLP_ROWS, c4 = i / MLP_ROWS;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < nt) v = __ldg(reinterpret_cast<const float4*>(desc + (long long)(r0 + r) * din) + c4);
    xsT[(4 * c4 + 0) * MLP_ROWS + r] = v.x;
    xsT[(4 * c4 + 1) * MLP_ROWS + r] = v.y;
    xsT[(4 * c4 + 2) * MLP_ROWS + r] = v.z;
    xsT[(4 * c4 + 3) * MLP_ROWS + r] = v.w;
  }
  __syncthreads();
  {
    const int rg = threadIdx.x / 32;  // rows rg*MLP_RPT .. (one warp per row group)
    const int cg = threadIdx.x % 32;  // columns cg*4 .. cg*4+3 of a 128-column chunk
    // layer 1 + GELU
    for (int cb = 0; cb < hidden; cb += 128) {
      const int c = cb + cg * 4;
      const bool act = c < hidden;
      float acc[MLP_RPT][4];
      if (act) {
        const float4 bias = __ldg(reinterpret_cast<const float4*>(B1 + c));
#pragma unroll
        for (int r = 0; r < MLP_RPT; ++r) {
          acc[r][0] = bias.x;
          acc[r][1] = bias.y;
          acc[r][2] = bias.z;
          acc[r][3] = bias.w;
        }
#pragma unroll 4
        for (int i = 0; i < din; ++i) {
          const float4 wv = __ldg(reinterpret_cast<const float4*>(W1 + (long long)i * hidden + c));
          float xr[MLP_RPT];
#pragma unroll
          for (int q = 0; q < MLP_RPT / 4; ++q) {
            const float4 x4 = *reinterpret_cast<const float4*>(xsT + i * MLP_ROWS + rg * MLP_RPT + 4 * q);
            xr[4 * q] = x4.x; xr[4 * q + 1] = x4.y; xr[4 * q + 2] = x4.z; xr[4 * q + 3] = x4.w;
          }
          const uint64_t w01 = f2(wv.x, wv.y), w23 = f2(wv.z, wv.w);
#pragma unroll
          for (int r = 0; r < MLP_RPT; ++r) {
            const uint64_t xx = f2(xr[r], xr[r]);
            uint64_t a01 = f2(acc[r][0], acc[r][1]), a23 = f2(acc[r][2], acc[r][3]);
            a01 = f2_fma(xx, w01, a01);
            a23 = f2_fma(xx, w23, a23);
            f2_split(a01, acc[r][0], acc[r][1]);
            f2_split(a23, acc[r][2], acc[r][3]);
          }
        }
      }
      if (alias) __syncthreads();  // every thread is done with the descriptors (single chunk)
      if (act) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int q = 0; q < MLP_RPT / 4; ++q) {
            float4 v;
            v.x = gelu_erf(acc[4 * q][e]);
            v.y = gelu_erf(acc[4 * q + 1][e]);
            v.z = gelu_erf(acc[4 * q + 2][e]);
            v.w = gelu_erf(acc[4 * q + 3][e]);
            *reinterpret_cast<float4*>(hsT + (c + e) * MLP_ROWS + rg * MLP_RPT + 4 * q) = v;
          }
      }
    }
  }
  __syncthreads();
  // layer 2
  const int rg2 = threadIdx.x / 16;  // rows rg2*4 .. rg2*4+3
  const int cg2 = threadIdx.x % 16;  // columns cg2*4 .. of a 64-column chunk
  for (int cb = 0; cb < out_dim; cb += 64) {
    const int c = cb + cg2 * 4;
    if (c >= out_dim) continue;
    float acc[MLP_RPT2][4];
    const float4 bias = __ldg(reinterpret_cast<const float4*>(B2 + c));
#pragma unroll
    for (int r = 0; r < MLP_RPT2; ++r) {
      acc[r][0] = bias.x;
      acc[r][1] = bias.y;
      acc[r][2] = bias.z;
      acc[r][3] = bias.w;
    }
#pragma unroll 4
    for (int i = 0; i < hidden; ++i) {
      const float4 wv = __ldg(reinterpret_cast<const float4*>(W2 + (long long)i * out_dim + c));
      const float4 x4 = *reinterpret_cast<const float4*>(hsT + i * MLP_ROWS + rg2 * MLP_RPT2);
      const float xr[4] = {x4.x, x4.y, x4.z, x4.w};
      const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int r = 0; r < MLP_RPT2; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][e] = fmaf(xr[r], wr[e], acc[r][e]);
    }
#pragma unroll
    for (int r = 0; r < MLP_RPT2; ++r) {
      const int row = r0 + rg2 * MLP_RPT2 + r;
      if (row < g.nt_cap) {
        const bool v = row < nt;
        *reinterpret_cast<float4*>(out + (long long)row * out_dim + c) =
            v ? make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

// scores[b,h,i,j] = scale * q[i].k[j]; 128x128 output tile per CTA, 8x8 per
// thread (rows ty*4.. and 64+ty*4.., columns tx*4.. and 64+tx*4..), the
// embeddings staged 32 dimensions at a time. Every score is one fma chain
// from 0 over the dimensions in ascending order, then times scale (the fused
// scores + top-k kernel builds its scores the same way).
constexpr int SG_TILE = 128, SG_KC = 32, SG_LD = SG_TILE + 4;

__global__ void __launch_bounds__(256) score_gemm_kernel(const __grid_constant__ LayerGeom g, const float* __restrict__ emb,
                                                         int out_dim, float scale, float* __restrict__ scores,
                                                         const int32_t* __restrict__ head_on) {
  if (head_on && !head_on[blockIdx.z]) return;  // blockIdx.z = b * heads + h
  __shared__ __align__(16) float As[SG_KC][SG_LD];
  __shared__ __align__(16) float Bs[SG_KC][SG_LD];
  const int h = blockIdx.z % g.heads;
  const int b = blockIdx.z / g.heads;
  const int nt = g.h[h].nt;
  const int i0 = blockIdx.y * SG_TILE, j0 = blockIdx.x * SG_TILE;
  const long long bh = (long long)b * g.heads + h;
  const float* Q = emb + bh * g.nt_cap * out_dim;
  const float* K = emb + ((long long)g.B * g.heads + bh) * g.nt_cap * out_dim;
  float* C = scores + bh * (long long)g.nt_cap * g.nt_cap;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][8];
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int w = 0; w < 8; ++w) acc[u][w] = 0.f;
  if (i0 < nt && j0 < nt) {
    for (int e0 = 0; e0 < out_dim; e0 += SG_KC) {
      for (int t = threadIdx.x; t < SG_TILE * SG_KC; t += 256) {
        const int r = t / SG_KC, e = t % SG_KC;
        const bool ein = e0 + e < out_dim;
        As[e][r] = (i0 + r < nt && ein) ? Q[(long long)(i0 + r) * out_dim + e0 + e] : 0.f;
        Bs[e][r] = (j0 + r < nt && ein) ? K[(long long)(j0 + r) * out_dim + e0 + e] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int e = 0; e < SG_KC; ++e) {
        const float4 a0 = *reinterpret_cast<const float4*>(&As[e][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&As[e][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[e][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[e][64 + tx * 4]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int w = 0; w < 8; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
      }
      __syncthreads();
    }
  }
  const bool vec = (g.nt_cap & 3) == 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = i0 + (u < 4 ? ty * 4 + u : 64 + ty * 4 + (u - 4));
    if (i >= g.nt_cap) continue;
    float* crow = C + (long long)i * g.nt_cap;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = j0 + half * 64 + tx * 4;
      float v[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) v[w] = (i < nt && j + w < nt) ? acc[u][half * 4 + w] * scale : 0.f;
      if (vec && j + 3 < g.nt_cap) {
        *reinterpret_cast<float4*>(crow + j) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (j + w < g.nt_cap) crow[j + w] = v[w];
      }
    }
  }
}

}  // namespace

cudaError_t launch_mlp(const LayerGeom& g, const float* dq, const float* dk, const float* w1q, const float* b1q,
                       const float* w2q, const float* b2q, const float* w1k, const float* b1k, const float* w2k,
                       const float* b2k, int hidden, int out_dim, float* emb_ws, cudaStream_t s,
                       const int32_t* head_on) {
  const size_t smem = (size_t)mlp_smem_floats(3 * g.d, hidden) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 g1((g.nt_cap + MLP_ROWS - 1) / MLP_ROWS, g.heads, g.B * 2);
  mlp_kernel<<<g1, MLP_THREADS, smem, s>>>(g, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden, out_dim, emb_ws,
                                   head_on);
  return cudaGetLastError();
}

cudaError_t launch_tile_scores(const LayerGeom& g, const float* dq, const float* dk, const float* w1q,
                               const float* b1q, const float* w2q, const float* b2q, const float* w1k,
                               const float* b1k, const float* w2k, const float* b2k, int hidden, int out_dim,
                               float scale, float* scores, float* emb_ws, cudaStream_t s,
                               const int32_t* head_on) {
  cudaError_t e = launch_mlp(g, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden, out_dim, emb_ws, s,
                             head_on);
  if (e != cudaSuccess) return e;
  const int nb = (g.nt_cap + SG_TILE - 1) / SG_TILE;
  const dim3 g2(nb, nb, g.heads * g.B);
  score_gemm_kernel<<<g2, 256, 0, s>>>(g, emb_ws, out_dim, scale, scores, head_on);
  return cudaGetLastError();
}

}  // namespace veda
