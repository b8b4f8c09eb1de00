// Estimator training: gradient of the distillation loss with respect to the
// per-head MLP weights (Veda summary 2.1, Optimization: the head-specific
// projections learn from a row-wise KL against the oracle tile map, with
// stop-gradient on the pooled descriptors; 2.3, Training Efficiency: on
// random subsets of query tiles).
//
// For each selected head, with q_r = MLP_q(dq[row r]) for the sampled query
// tiles and k_j = MLP_k(dk[j]) for all key tiles:
//   s_rj = scale q_r . k_j,  p_r = softmax_j(s_r),  t_r = M_r / sum M_r,
//   loss = mean over heads of mean over rows of KL(t_r || p_r),
//   G = dloss/ds = (p - t) / (rows * heads),
//   dq = scale G k,  dk = scale G^T q,
//   per side: dz = (dy W2^T) * GELU'(z),  dW1 = x^T dz,  db1 = sum dz,
//             dW2 = GELU(z)^T dy,  db2 = sum dy.
// Every reduction runs in a fixed order (no atomics), so results are
// bit-reproducible. fp32 FFMA throughout.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int FW_ROWS = 8;   // descriptors per CTA in the forward recompute (small: many CTAs, latency-bound loops)
constexpr int WG_SPLIT = 8;  // row chunks of the weight-gradient GEMMs (fixed-order partial sums)

__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float x) {
  return 0.5f * (1.0f + erff(x * 0.70710678118654752f)) + x * 0.39894228040143268f * expf(-0.5f * x * x);
}

struct GradWs {
  // per selected head hs (all row-major):
  float* zq;  // [n_rows][hidden]   pre-activations, query side
  float* yq;  // [n_rows][out]      query embeddings
  float* zk;  // [nt_cap][hidden]
  float* yk;  // [nt_cap][out]
  float* G;   // [n_rows][nt_cap]   dloss/ds
  float* dyq; // [n_rows][out]
  float* dyk; // [nt_cap][out]
  float* dzq; // [n_rows][hidden]
  float* dzk; // [nt_cap][hidden]
  float* kl;  // [n_rows]
  float* part;  // [2 sides][WG_SPLIT][(3d+1)*hidden + (hidden+1)*out]  weight-gradient partial sums
};

struct GradArgs {
  const float* dq;
  const float* dk;
  const float* w1[2];  // [side]: 0 query, 1 key
  const float* b1[2];
  const float* w2[2];
  const float* b2[2];
  float* gw1[2];
  float* gb1[2];
  float* gw2[2];
  float* gb2[2];
  const int32_t* rows;  // [n_heads_sel][n_rows] or NULL (tiles 0..n_rows-1)
  const float* tilemap; // [n_heads_sel][n_rows][nt_cap]
  float* loss;
  int hidden, out_dim, n_rows, n_heads_sel;
  float scale, coef;    // coef = 1 / (n_rows * n_heads_sel)
  int heads_sel[VEDA_MAX_HEADS];
  size_t ws_per_head;   // floats
  float* ws;
};

__device__ __forceinline__ GradWs head_ws(const GradArgs& a, int nt_cap, int hs) {
  float* p = a.ws + (size_t)hs * a.ws_per_head;
  GradWs w;
  w.zq = p;  p += (size_t)a.n_rows * a.hidden;
  w.yq = p;  p += (size_t)a.n_rows * a.out_dim;
  w.zk = p;  p += (size_t)nt_cap * a.hidden;
  w.yk = p;  p += (size_t)nt_cap * a.out_dim;
  w.G = p;   p += (size_t)a.n_rows * nt_cap;
  w.dyq = p; p += (size_t)a.n_rows * a.out_dim;
  w.dyk = p; p += (size_t)nt_cap * a.out_dim;
  w.dzq = p; p += (size_t)a.n_rows * a.hidden;
  w.dzk = p; p += (size_t)nt_cap * a.hidden;
  w.kl = p;  p += (size_t)a.n_rows;
  w.part = p;
  return w;
}

// descriptor row i of side `side` for selected head hs: the sampled query tile
// (query side) or key tile i (key side); -1 when i is past the head's tiles
__device__ __forceinline__ int desc_row(const GradArgs& a, const LayerGeom& g, int side, int hs, int i) {
  const int nt = g.h[a.heads_sel[hs]].nt;
  if (side == 0) {
    if (i >= a.n_rows) return -1;
    const int t = a.rows ? a.rows[hs * a.n_rows + i] : i;
    return (t >= 0 && t < nt) ? t : -1;
  }
  return i < nt ? i : -1;
}

// 1. MLP forward keeping the pre-activations: grid (ceil(N/FW_ROWS), heads_sel,
// 2 sides), 128 threads. Thread u of layer 1 owns hidden unit u (and u+128)
// for the CTA's FW_ROWS descriptors held in shared memory; layer 2 likewise per
// output unit. Rows past the side's count are written as zeros.
__global__ void __launch_bounds__(128) fwd_save_kernel(const __grid_constant__ LayerGeom g,
                                                       const __grid_constant__ GradArgs a) {
  extern __shared__ float sm[];
  const int din = 3 * g.d;
  float* xs = sm;                      // [FW_ROWS][din]
  float* hs_ = sm + FW_ROWS * din;     // [FW_ROWS][hidden], GELU(z)
  const int hs = blockIdx.y, side = blockIdx.z;
  const int h = a.heads_sel[hs];
  const int n_out = side == 0 ? a.n_rows : g.nt_cap;
  const int r0 = blockIdx.x * FW_ROWS;
  if (r0 >= n_out) return;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const float* X = (side == 0 ? a.dq : a.dk) + (long long)h * g.nt_cap * din;
  const float* W1 = a.w1[side] + (long long)h * din * a.hidden;
  const float* B1 = a.b1[side] + (long long)h * a.hidden;
  const float* W2 = a.w2[side] + (long long)h * a.hidden * a.out_dim;
  const float* B2 = a.b2[side] + (long long)h * a.out_dim;
  float* Z = side == 0 ? w.zq : w.zk;
  float* Y = side == 0 ? w.yq : w.yk;
  bool valid[FW_ROWS];
  for (int t = threadIdx.x; t < FW_ROWS * din; t += blockDim.x) {
    const int r = t / din, c = t % din;
    const int row = desc_row(a, g, side, hs, r0 + r);
    xs[t] = row >= 0 ? X[(long long)row * din + c] : 0.f;
  }
#pragma unroll
  for (int r = 0; r < FW_ROWS; ++r) valid[r] = desc_row(a, g, side, hs, r0 + r) >= 0;
  __syncthreads();
  for (int u = threadIdx.x; u < a.hidden; u += blockDim.x) {
    float acc[FW_ROWS];
#pragma unroll
    for (int r = 0; r < FW_ROWS; ++r) acc[r] = B1[u];
    for (int c = 0; c < din; ++c) {
      const float wv = __ldg(W1 + (long long)c * a.hidden + u);
#pragma unroll
      for (int r = 0; r < FW_ROWS; ++r) acc[r] = fmaf(xs[r * din + c], wv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < FW_ROWS; ++r) {
      const float z = valid[r] ? acc[r] : 0.f;
      hs_[r * a.hidden + u] = valid[r] ? gelu_f(z) : 0.f;
      if (r0 + r < n_out) Z[(long long)(r0 + r) * a.hidden + u] = z;
    }
  }
  __syncthreads();
  for (int o = threadIdx.x; o < a.out_dim; o += blockDim.x) {
    float acc[FW_ROWS];
#pragma unroll
    for (int r = 0; r < FW_ROWS; ++r) acc[r] = B2[o];
    for (int u = 0; u < a.hidden; ++u) {
      const float wv = __ldg(W2 + (long long)u * a.out_dim + o);
#pragma unroll
      for (int r = 0; r < FW_ROWS; ++r) acc[r] = fmaf(hs_[r * a.hidden + u], wv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < FW_ROWS; ++r)
      if (r0 + r < n_out) Y[(long long)(r0 + r) * a.out_dim + o] = valid[r] ? acc[r] : 0.f;
  }
}

// 2. Per sampled row: scores against every key tile, softmax, normalised
// map row, G = (p - t) * coef and the row's KL. One CTA (256 threads) per
// (row, head); the row lives in shared memory.
__global__ void __launch_bounds__(256) kl_grad_kernel(const __grid_constant__ LayerGeom g,
                                                      const __grid_constant__ GradArgs a) {
  extern __shared__ float srow[];  // [nt_cap] scores, then reused
  __shared__ float red[8];
  const int r = blockIdx.x, hs = blockIdx.y;
  const int h = a.heads_sel[hs];
  const int nt = g.h[h].nt;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const float* q = w.yq + (long long)r * a.out_dim;
  const float* M = a.tilemap + ((long long)hs * a.n_rows + r) * g.nt_cap;
  float* G = w.G + (long long)r * g.nt_cap;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto block_sum = [&](float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) t += red[i];
    return t;
  };
  auto block_max = [&](float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) t = fmaxf(t, red[i]);
    return t;
  };
  float mx = -INFINITY, msum = 0.f;
  for (int j = threadIdx.x; j < nt; j += blockDim.x) {
    const float* k = w.yk + (long long)j * a.out_dim;
    float acc = 0.f;
    for (int o = 0; o < a.out_dim; ++o) acc = fmaf(q[o], k[o], acc);
    srow[j] = acc * a.scale;
    mx = fmaxf(mx, srow[j]);
    msum += M[j];
  }
  mx = block_max(mx);
  msum = block_sum(msum);
  float esum = 0.f;
  for (int j = threadIdx.x; j < nt; j += blockDim.x) esum += expf(srow[j] - mx);
  esum = block_sum(esum);
  const float lse = mx + logf(esum);
  float kl = 0.f;
  const bool row_ok = msum > 0.f;  // a map row of zeros (no valid query tile) contributes nothing
  for (int j = threadIdx.x; j < g.nt_cap; j += blockDim.x) {
    float gj = 0.f;
    if (row_ok && j < nt) {
      const float logp = srow[j] - lse;
      const float t = M[j] / msum;
      gj = (expf(logp) - t) * a.coef;
      if (t > 0.f) kl += t * (logf(t) - logp);
    }
    G[j] = gj;
  }
  kl = block_sum(kl);
  if (threadIdx.x == 0) w.kl[r] = kl;
}

// 3. Embedding gradients: dy_q[r] = scale * sum_j G[r, j] k_j (grid rows x
// heads) and dy_k[j] = scale * sum_r G[r, j] q_r (grid key tiles x heads);
// thread o owns output unit o.
__global__ void dy_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ GradArgs a) {
  const int i = blockIdx.x, hs = blockIdx.y, side = blockIdx.z;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const int nt = g.h[a.heads_sel[hs]].nt;
  if (i >= (side == 0 ? a.n_rows : g.nt_cap)) return;
  for (int o = threadIdx.x; o < a.out_dim; o += blockDim.x) {
    float acc = 0.f;
    if (side == 0) {
      const float* G = w.G + (long long)i * g.nt_cap;
      for (int j = 0; j < nt; ++j) acc = fmaf(G[j], w.yk[(long long)j * a.out_dim + o], acc);
      w.dyq[(long long)i * a.out_dim + o] = acc * a.scale;
    } else {
      if (i < nt)
        for (int r = 0; r < a.n_rows; ++r) acc = fmaf(w.G[(long long)r * g.nt_cap + i], w.yq[(long long)r * a.out_dim + o], acc);
      w.dyk[(long long)i * a.out_dim + o] = acc * a.scale;
    }
  }
}

// 4. dz = (dy W2^T) * GELU'(z) for every descriptor row of both sides:
// grid (ceil(rows / DZ_ROWS), heads, sides); thread u owns hidden unit u for
// the CTA's DZ_ROWS rows (their dy in shared memory), so each W2 entry is
// loaded once per DZ_ROWS rows.
constexpr int DZ_ROWS = 8;

__global__ void __launch_bounds__(128) dz_kernel(const __grid_constant__ LayerGeom g,
                                                 const __grid_constant__ GradArgs a) {
  extern __shared__ float dys[];  // [DZ_ROWS][out_dim]
  const int i0 = blockIdx.x * DZ_ROWS, hs = blockIdx.y, side = blockIdx.z;
  const int n_out = side == 0 ? a.n_rows : g.nt_cap;
  if (i0 >= n_out) return;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const int h = a.heads_sel[hs];
  const float* W2 = a.w2[side] + (long long)h * a.hidden * a.out_dim;
  const float* dy = side == 0 ? w.dyq : w.dyk;
  const float* Z = side == 0 ? w.zq : w.zk;
  float* dz = side == 0 ? w.dzq : w.dzk;
  for (int t = threadIdx.x; t < DZ_ROWS * a.out_dim; t += blockDim.x) {
    const int r = t / a.out_dim;
    dys[t] = i0 + r < n_out ? dy[(long long)i0 * a.out_dim + t] : 0.f;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < a.hidden; u += blockDim.x) {
    float acc[DZ_ROWS] = {};
    for (int o = 0; o < a.out_dim; ++o) {
      const float wv = __ldg(W2 + (long long)u * a.out_dim + o);
#pragma unroll
      for (int r = 0; r < DZ_ROWS; ++r) acc[r] = fmaf(dys[r * a.out_dim + o], wv, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < DZ_ROWS; ++r) {
      const int i = i0 + r;
      if (i >= n_out) break;
      const bool valid = desc_row(a, g, side, hs, i) >= 0;
      dz[(long long)i * a.hidden + u] = valid ? acc[r] * gelu_grad_f(Z[(long long)i * a.hidden + u]) : 0.f;
    }
  }
}

// 5. Weight gradients of one side of one selected head, as tiled GEMMs over
// the descriptor rows:
// out[(K+1) x N] = A^T B with A = [x | 1] (layer 1: K = 3d, N = hidden,
// B = dz) or A = [GELU(z) | 1] (layer 2: K = hidden, N = out_dim, B = dy);
// the extra row of ones makes the last output row the bias gradient. A CTA
// computes a 64 x 64 output tile (4 x 4 per thread) and walks the rows in
// chunks of 16 in order, so results are bit-reproducible.
constexpr int WG_TILE = 64, WG_CHUNK = 16;

template <int LAYER>
__global__ void __launch_bounds__(256) wgrad_gemm_kernel(const __grid_constant__ LayerGeom g,
                                                         const __grid_constant__ GradArgs a) {
  __shared__ __align__(16) float As[WG_CHUNK][WG_TILE];
  __shared__ __align__(16) float Bs[WG_CHUNK][WG_TILE];
  const int chunk = blockIdx.z % WG_SPLIT;
  const int hs = (blockIdx.z / WG_SPLIT) >> 1, side = (blockIdx.z / WG_SPLIT) & 1;
  const int h = a.heads_sel[hs];
  const int din = 3 * g.d;
  const int K = LAYER == 1 ? din : a.hidden;
  const int N = LAYER == 1 ? a.hidden : a.out_dim;
  const int k0 = blockIdx.x * WG_TILE, n0 = blockIdx.y * WG_TILE;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const int n_rows_side = side == 0 ? a.n_rows : g.nt_cap;
  // this CTA's rows: chunk `chunk` of WG_SPLIT, in whole WG_CHUNK steps
  const int steps = (n_rows_side + WG_CHUNK - 1) / WG_CHUNK;
  const int i_begin = (int)((long long)steps * chunk / WG_SPLIT) * WG_CHUNK;
  const int n_in = min(n_rows_side, (int)((long long)steps * (chunk + 1) / WG_SPLIT) * WG_CHUNK);
  const float* X = (side == 0 ? a.dq : a.dk) + (long long)h * g.nt_cap * din;
  const float* Z = side == 0 ? w.zq : w.zk;
  const float* Bsrc = LAYER == 1 ? (side == 0 ? w.dzq : w.dzk) : (side == 0 ? w.dyq : w.dyk);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int i0 = i_begin; i0 < n_in; i0 += WG_CHUNK) {
    for (int t = threadIdx.x; t < WG_CHUNK * WG_TILE; t += blockDim.x) {
      const int ii = t / WG_TILE, cc = t % WG_TILE;
      const int i = i0 + ii, kk = k0 + cc, nn = n0 + cc;
      const int row = i < n_in ? desc_row(a, g, side, hs, i) : -1;
      float av = 0.f, bv = 0.f;
      if (row >= 0) {
        if (kk < K) av = LAYER == 1 ? X[(long long)row * din + kk] : gelu_f(Z[(long long)i * a.hidden + kk]);
        else if (kk == K) av = 1.f;
        if (nn < N) bv = Bsrc[(long long)i * N + nn];
      }
      As[ii][cc] = av;
      Bs[ii][cc] = bv;
    }
    __syncthreads();
#pragma unroll
    for (int ii = 0; ii < WG_CHUNK; ++ii) {
      const float4 av = *reinterpret_cast<const float4*>(&As[ii][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[ii][tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w}, br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(ar[u], br[v], acc[u][v]);
    }
    __syncthreads();
  }
  // partial sums of this row chunk: [(K+1) x N] block of the side's partials
  const long long per_chunk = (long long)(din + 1) * a.hidden + (long long)(a.hidden + 1) * a.out_dim;
  float* P = w.part + ((long long)side * WG_SPLIT + chunk) * per_chunk +
             (LAYER == 1 ? 0 : (long long)(din + 1) * a.hidden);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int kk = k0 + ty * 4 + u;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int nn = n0 + tx * 4 + v;
      if (nn < N && kk <= K) P[(long long)kk * N + nn] = acc[u][v];
    }
  }
}

// Sum of the row chunks' partials in chunk order: weight and bias gradients
// of one side of one selected head (grid: elements, heads x sides).
__global__ void wgrad_reduce_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ GradArgs a) {
  const int hs = blockIdx.y >> 1, side = blockIdx.y & 1;
  const int h = a.heads_sel[hs];
  const int din = 3 * g.d;
  const long long n1 = (long long)(din + 1) * a.hidden, per_chunk = n1 + (long long)(a.hidden + 1) * a.out_dim;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= per_chunk) return;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const float* P = w.part + (long long)side * WG_SPLIT * per_chunk + t;
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < WG_SPLIT; ++c) acc += P[c * per_chunk];
  if (t < n1) {
    const int kk = (int)(t / a.hidden), nn = (int)(t % a.hidden);
    if (kk < din) a.gw1[side][((long long)h * din + kk) * a.hidden + nn] = acc;
    else a.gb1[side][(long long)h * a.hidden + nn] = acc;
  } else {
    const long long e = t - n1;
    const int kk = (int)(e / a.out_dim), nn = (int)(e % a.out_dim);
    if (kk < a.hidden) a.gw2[side][((long long)h * a.hidden + kk) * a.out_dim + nn] = acc;
    else a.gb2[side][(long long)h * a.out_dim + nn] = acc;
  }
}

// 6. Loss: mean over rows, then over heads, in a fixed order (one thread).
__global__ void loss_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ GradArgs a) {
  if (threadIdx.x != 0 || !a.loss) return;
  float total = 0.f;
  for (int hs = 0; hs < a.n_heads_sel; ++hs) {
    const GradWs w = head_ws(a, g.nt_cap, hs);
    float s = 0.f;
    for (int r = 0; r < a.n_rows; ++r) s += w.kl[r];
    total += s / (float)a.n_rows;
  }
  *a.loss = total / (float)a.n_heads_sel;
}

}  // namespace

size_t estimator_ws_floats_per_head(int nt_cap, int n_rows, int hidden, int out_dim, int din) {
  return 2 * (size_t)n_rows * hidden + 2 * (size_t)n_rows * out_dim + 2 * (size_t)nt_cap * hidden +
         2 * (size_t)nt_cap * out_dim + (size_t)n_rows * nt_cap + (size_t)n_rows +
         2 * (size_t)WG_SPLIT * ((size_t)(din + 1) * hidden + (size_t)(hidden + 1) * out_dim);
}

cudaError_t launch_estimator_grad(const LayerGeom& g, const float* dq, const float* dk, const float* const w[8],
                                  float* const gw[8], int hidden, int out_dim, float scale, const int32_t* heads_sel,
                                  int n_heads_sel, const int32_t* rows, int n_rows, const float* tilemap,
                                  float* loss, float* ws, cudaStream_t s) {
  GradArgs a;
  a.dq = dq;
  a.dk = dk;
  for (int side = 0; side < 2; ++side) {
    a.w1[side] = w[4 * side + 0];
    a.b1[side] = w[4 * side + 1];
    a.w2[side] = w[4 * side + 2];
    a.b2[side] = w[4 * side + 3];
    a.gw1[side] = gw[4 * side + 0];
    a.gb1[side] = gw[4 * side + 1];
    a.gw2[side] = gw[4 * side + 2];
    a.gb2[side] = gw[4 * side + 3];
  }
  a.rows = rows;
  a.tilemap = tilemap;
  a.loss = loss;
  a.hidden = hidden;
  a.out_dim = out_dim;
  a.n_rows = n_rows;
  a.n_heads_sel = n_heads_sel;
  a.scale = scale;
  a.coef = 1.0f / ((float)n_rows * (float)n_heads_sel);
  for (int i = 0; i < n_heads_sel; ++i) a.heads_sel[i] = heads_sel[i];
  a.ws_per_head = estimator_ws_floats_per_head(g.nt_cap, n_rows, hidden, out_dim, 3 * g.d);
  a.ws = ws;
  const int din = 3 * g.d;
  // gradients of heads that are not selected are zero
  const size_t n1 = (size_t)din * hidden, n2 = hidden, n3 = (size_t)hidden * out_dim, n4 = out_dim;
  const size_t per[4] = {n1, n2, n3, n4};
  for (int i = 0; i < 8; ++i) {
    cudaError_t e = cudaMemsetAsync(gw[i], 0, per[i % 4] * g.heads * sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  const size_t smem_fw = (size_t)FW_ROWS * (din + hidden) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(fwd_save_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_fw);
  if (e != cudaSuccess) return e;
  const int n_side_max = g.nt_cap > n_rows ? g.nt_cap : n_rows;
  fwd_save_kernel<<<dim3((n_side_max + FW_ROWS - 1) / FW_ROWS, n_heads_sel, 2), 128, smem_fw, s>>>(g, a);
  const size_t smem_kl = (size_t)g.nt_cap * sizeof(float);
  e = cudaFuncSetAttribute(kl_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kl);
  if (e != cudaSuccess) return e;
  kl_grad_kernel<<<dim3(n_rows, n_heads_sel), 256, smem_kl, s>>>(g, a);
  dy_kernel<<<dim3(n_side_max, n_heads_sel, 2), 128, 0, s>>>(g, a);
  dz_kernel<<<dim3((n_side_max + DZ_ROWS - 1) / DZ_ROWS, n_heads_sel, 2), 128,
              (size_t)DZ_ROWS * out_dim * sizeof(float), s>>>(g, a);
  wgrad_gemm_kernel<1><<<dim3((din + 1 + WG_TILE - 1) / WG_TILE, (hidden + WG_TILE - 1) / WG_TILE,
                              2 * n_heads_sel * WG_SPLIT),
                         256, 0, s>>>(g, a);
  wgrad_gemm_kernel<2><<<dim3((hidden + 1 + WG_TILE - 1) / WG_TILE, (out_dim + WG_TILE - 1) / WG_TILE,
                              2 * n_heads_sel * WG_SPLIT),
                         256, 0, s>>>(g, a);
  const long long per_chunk = (long long)(din + 1) * hidden + (long long)(hidden + 1) * out_dim;
  wgrad_reduce_kernel<<<dim3((unsigned)((per_chunk + 255) / 256), 2 * n_heads_sel), 256, 0, s>>>(g, a);
  loss_kernel<<<1, 32, 0, s>>>(g, a);
  return cudaGetLastError();
}

}  // namespace veda
