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

constexpr int FW_ROWS = 32;  // descriptors per CTA in the forward recompute

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
  w.kl = p;
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

// 1. MLP forward keeping the pre-activations: grid (ceil(N/32), heads_sel,
// 2 sides), 128 threads. Thread u of layer 1 owns hidden unit u (and u+128)
// for the CTA's 32 descriptors held in shared memory; layer 2 likewise per
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
// grid (rows, heads, sides), thread u owns hidden unit u.
__global__ void dz_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ GradArgs a) {
  const int i = blockIdx.x, hs = blockIdx.y, side = blockIdx.z;
  const int n_out = side == 0 ? a.n_rows : g.nt_cap;
  if (i >= n_out) return;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const int h = a.heads_sel[hs];
  const float* W2 = a.w2[side] + (long long)h * a.hidden * a.out_dim;
  const float* dy = (side == 0 ? w.dyq : w.dyk) + (long long)i * a.out_dim;
  const float* Z = (side == 0 ? w.zq : w.zk) + (long long)i * a.hidden;
  float* dz = (side == 0 ? w.dzq : w.dzk) + (long long)i * a.hidden;
  const bool valid = desc_row(a, g, side, hs, i) >= 0;
  for (int u = threadIdx.x; u < a.hidden; u += blockDim.x) {
    float acc = 0.f;
    for (int o = 0; o < a.out_dim; ++o) acc = fmaf(dy[o], __ldg(W2 + (long long)u * a.out_dim + o), acc);
    dz[u] = valid ? acc * gelu_grad_f(Z[u]) : 0.f;
  }
}

// 5. Weight gradients of one side of one selected head: one thread per
// weight, each summing over that side's descriptor rows in order.
//   index < din*hidden            : dW1[c][u] = sum_i x[i][c] dz[i][u]
//   next hidden                    : db1[u]    = sum_i dz[i][u]
//   next hidden*out_dim            : dW2[u][o] = sum_i GELU(z[i][u]) dy[i][o]
//   next out_dim                   : db2[o]    = sum_i dy[i][o]
__global__ void wgrad_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ GradArgs a) {
  const int hs = blockIdx.y, side = blockIdx.z;
  const int h = a.heads_sel[hs];
  const int din = 3 * g.d;
  const long long n1 = (long long)din * a.hidden, n2 = n1 + a.hidden, n3 = n2 + (long long)a.hidden * a.out_dim,
                  n4 = n3 + a.out_dim;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n4) return;
  const GradWs w = head_ws(a, g.nt_cap, hs);
  const int n_in = side == 0 ? a.n_rows : g.nt_cap;
  const float* X = (side == 0 ? a.dq : a.dk) + (long long)h * g.nt_cap * din;
  const float* dz = side == 0 ? w.dzq : w.dzk;
  const float* dy = side == 0 ? w.dyq : w.dyk;
  const float* Z = side == 0 ? w.zq : w.zk;
  float acc = 0.f;
  if (t < n1) {
    const int c = (int)(t / a.hidden), u = (int)(t % a.hidden);
    for (int i = 0; i < n_in; ++i) {
      const int row = desc_row(a, g, side, hs, i);
      if (row >= 0) acc = fmaf(X[(long long)row * din + c], dz[(long long)i * a.hidden + u], acc);
    }
    a.gw1[side][(long long)h * n1 + t] = acc;
  } else if (t < n2) {
    const int u = (int)(t - n1);
    for (int i = 0; i < n_in; ++i)
      if (desc_row(a, g, side, hs, i) >= 0) acc += dz[(long long)i * a.hidden + u];
    a.gb1[side][(long long)h * a.hidden + u] = acc;
  } else if (t < n3) {
    const long long e = t - n2;
    const int u = (int)(e / a.out_dim), o = (int)(e % a.out_dim);
    for (int i = 0; i < n_in; ++i) {
      if (desc_row(a, g, side, hs, i) < 0) continue;
      acc = fmaf(gelu_f(Z[(long long)i * a.hidden + u]), dy[(long long)i * a.out_dim + o], acc);
    }
    a.gw2[side][(long long)h * a.hidden * a.out_dim + e] = acc;
  } else {
    const int o = (int)(t - n3);
    for (int i = 0; i < n_in; ++i)
      if (desc_row(a, g, side, hs, i) >= 0) acc += dy[(long long)i * a.out_dim + o];
    a.gb2[side][(long long)h * a.out_dim + o] = acc;
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

size_t estimator_ws_floats_per_head(int nt_cap, int n_rows, int hidden, int out_dim) {
  return 2 * (size_t)n_rows * hidden + 2 * (size_t)n_rows * out_dim + 2 * (size_t)nt_cap * hidden +
         2 * (size_t)nt_cap * out_dim + (size_t)n_rows * nt_cap + (size_t)n_rows;
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
  a.ws_per_head = estimator_ws_floats_per_head(g.nt_cap, n_rows, hidden, out_dim);
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
  dz_kernel<<<dim3(n_side_max, n_heads_sel, 2), 128, 0, s>>>(g, a);
  const long long nw = (long long)n1 + n2 + n3 + n4;
  wgrad_kernel<<<dim3((unsigned)((nw + 255) / 256), n_heads_sel, 2), 256, 0, s>>>(g, a);
  loss_kernel<<<1, 32, 0, s>>>(g, a);
  return cudaGetLastError();
}

}  // namespace veda
