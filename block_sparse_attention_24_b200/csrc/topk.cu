// Top-k key tiles per query tile (Veda summary 2.1 and 4: only the highest
// scoring key tiles are kept).
//
// One warp per score row; scores become order-preserving 32-bit keys (larger
// float -> larger key, -0.0 folded into +0.0). The exact k-th largest key T
// is found, then a final pass in column order keeps every key > T and the
// lowest-index keys == T, so exact ties go to the lower tile index and the
// output list comes out ascending without a sort.
//
// Rows of up to 2048 tiles (every layer of the pages' sizes) keep their keys
// in registers, and T is built bit by bit from the top in 32 steps: a bit is
// kept when at least k keys are >= T with it set. Each step counts the lane's
// keys >= the candidate through an add-with-carry (two instructions per key)
// and takes one warp reduction, with no shared memory and no atomics. Longer rows are staged in shared memory and take a 4-pass,
// 8-bit radix select whose histogram updates are warp-aggregated
// (__match_any_sync) shared atomics; the same radix selection also runs inside
// the fused scores + top-k kernel.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int TOPK_WARPS = 4;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;  // -0.0 ties +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Selection on one row staged as order keys in shared memory (warp-wide):
// writes the k kept column indices ascending (-1 beyond k, up to k_cap) and
// the 0/1 mask over nt_cap columns (when mask_row is not NULL). `hist` is 256
// words of this warp's shared memory.
__device__ __forceinline__ void warp_select_row(const uint32_t* keys, uint32_t* hist, int nt, int k, int k_cap,
                                                int nt_cap, int32_t* idx_row, uint8_t* mask_row, int lane) {
  uint32_t prefix = 0u, pmask = 0u;
  int remaining = k;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[lane * 8 + q] = 0u;
    __syncwarp();
    for (int c0 = 0; c0 < nt; c0 += 32) {
      const int c = c0 + lane;
      const bool in = c < nt;
      const uint32_t key = in ? keys[c] : 0u;
      const bool match = in && ((key & pmask) == prefix);
      const uint32_t active = __ballot_sync(0xffffffffu, match);
      if (match) {
        const uint32_t bin = (key >> shift) & 255u;
        const uint32_t same = __match_any_sync(active, bin);
        if ((__ffs(same) - 1) == lane) atomicAdd(&hist[bin], (uint32_t)__popc(same));
      }
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l (descending); scan from the top
    uint32_t cnt = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) cnt += hist[255 - 8 * lane - q];
    uint32_t incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    const uint32_t excl = incl - cnt;
    const bool here = excl < (uint32_t)remaining && (uint32_t)remaining <= incl;
    const uint32_t who = __ballot_sync(0xffffffffu, here);
    const int L = __ffs(who) - 1;  // exactly one lane: the class holds >= remaining keys
    uint32_t digit = 0, above = 0;
    if (lane == L) {
      uint32_t acc = excl;
      for (int q = 0; q < 8; ++q) {
        const uint32_t bin = 255 - 8 * lane - q;
        if (acc + hist[bin] >= (uint32_t)remaining) {
          digit = bin;
          above = acc;
          break;
        }
        acc += hist[bin];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, L);
    above = __shfl_sync(0xffffffffu, above, L);
    remaining -= (int)above;
    prefix |= digit << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  // prefix is now the k-th largest key; keep all larger keys and the first
  // `remaining` equal keys in column order.
  const uint32_t T = prefix;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0, eq_seen = 0;
  for (int c0 = 0; c0 < nt; c0 += 32) {
    const int c = c0 + lane;
    const bool in = c < nt;
    const uint32_t key = in ? keys[c] : 0u;
    const bool eq = in && key == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eqm & lt_mask);
    const bool sel = in && (key > T || (eq && eq_rank < remaining));
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (sel) idx_row[base + __popc(selm & lt_mask)] = c;
    if (mask_row && in) mask_row[c] = sel ? 1 : 0;
    base += __popc(selm);
    eq_seen += __popc(eqm);
  }
  for (int p = k + lane; p < k_cap; p += 32) idx_row[p] = -1;
  if (mask_row)
    for (int c = nt + lane; c < nt_cap; c += 32) mask_row[c] = 0;
}

__global__ void __launch_bounds__(TOPK_WARPS * 32) topk_radix_kernel(const __grid_constant__ LayerGeom g,
                                                               const float* __restrict__ scores, int k_cap,
                                                               int32_t* __restrict__ idx, uint8_t* __restrict__ mask,
                                                               const int32_t* __restrict__ head_on) {
  extern __shared__ uint32_t sm_u32[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint32_t* keys = sm_u32 + warp * (g.nt_cap + 256);
  uint32_t* hist = keys + g.nt_cap;
  const long long rows = (long long)g.B * g.heads * g.nt_cap;
  const long long row = (long long)blockIdx.x * TOPK_WARPS + warp;
  if (row >= rows) return;
  const int a = (int)(row % g.nt_cap);
  const int h = (int)((row / g.nt_cap) % g.heads);
  // head_on (may be NULL): per (batch element, head), 0 = keep the cached mask
  if (head_on && !head_on[row / g.nt_cap]) return;
  const int nt = g.h[h].nt;
  const int k = g.h[h].k;
  int32_t* idx_row = idx + row * k_cap;
  uint8_t* mask_row = mask ? mask + row * g.nt_cap : nullptr;
  if (a >= nt) {
    for (int p = lane; p < k_cap; p += 32) idx_row[p] = -1;
    if (mask_row)
      for (int c = lane; c < g.nt_cap; c += 32) mask_row[c] = 0;
    return;
  }
  const float* srow = scores + row * g.nt_cap;
  for (int c = lane; c < nt; c += 32) keys[c] = order_key(__ldg(srow + c));
  __syncwarp();

  warp_select_row(keys, hist, nt, k, k_cap, g.nt_cap, idx_row, mask_row, lane);
}

// Register-resident selection: KPL keys per lane (column 32 i + lane in key
// i; columns at or past nt hold key 0, which is below the key of every float,
// so no candidate T >= 1 ever counts them).
constexpr int BIS_WARPS = 8;

// #(keys >= cand) over one lane's keys, cand >= 1: key + (2^32 - cand)
// carries out exactly when key >= cand, and the carry is added straight into
// the count (two instructions per key).
template <int KPL>
__device__ __forceinline__ uint32_t count_ge(const uint32_t (&key)[KPL], uint32_t cand) {
  const uint32_t neg = 0u - cand;
  uint32_t c0 = 0u, c1 = 0u;
#pragma unroll
  for (int i = 0; i < KPL; i += 2) {
    uint32_t t0, t1;
    asm("add.cc.u32 %0, %2, %3;\n\taddc.u32 %1, %1, 0;" : "=r"(t0), "+r"(c0) : "r"(key[i]), "r"(neg));
    asm("add.cc.u32 %0, %2, %3;\n\taddc.u32 %1, %1, 0;" : "=r"(t1), "+r"(c1) : "r"(key[i + 1]), "r"(neg));
  }
  return c0 + c1;
}

template <int KPL>
__global__ void __launch_bounds__(BIS_WARPS * 32) topk_bisect_kernel(const __grid_constant__ LayerGeom g,
                                                                     const float* __restrict__ scores, int k_cap,
                                                                     int32_t* __restrict__ idx,
                                                                     uint8_t* __restrict__ mask,
                                                                     const int32_t* __restrict__ head_on) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long rows = (long long)g.B * g.heads * g.nt_cap;
  const long long row = (long long)blockIdx.x * BIS_WARPS + warp;
  if (row >= rows) return;
  const int a = (int)(row % g.nt_cap);
  const int h = (int)((row / g.nt_cap) % g.heads);
  if (head_on && !head_on[row / g.nt_cap]) return;
  const int nt = g.h[h].nt;
  const int k = g.h[h].k;
  int32_t* idx_row = idx + row * k_cap;
  uint8_t* mask_row = mask ? mask + row * g.nt_cap : nullptr;
  if (a >= nt) {
    for (int p = lane; p < k_cap; p += 32) idx_row[p] = -1;
    if (mask_row)
      for (int c = lane; c < g.nt_cap; c += 32) mask_row[c] = 0;
    return;
  }
  const float* srow = scores + row * g.nt_cap;
  uint32_t key[KPL];
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int c = 32 * i + lane;
    key[i] = c < nt ? order_key(__ldg(srow + c)) : 0u;
  }
  // T = the largest value with #(key >= T) >= k, i.e. the k-th largest key
  // (the count only drops as T grows, so the top-down greedy choice is exact)
  uint32_t T = 0u;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    if (__reduce_add_sync(0xffffffffu, count_ge(key, cand)) >= (unsigned)k) T = cand;
  }
  int gt = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) gt += key[i] > T;
  const int remaining = k - (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);  // keys == T to keep, >= 1
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    if (32 * i >= nt) break;
    const int c = 32 * i + lane;
    const bool in = c < nt;
    const bool eq = in && key[i] == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eqm & lt_mask);
    const bool sel = in && (key[i] > T || (eq && eq_rank < remaining));
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (sel) idx_row[base + __popc(selm & lt_mask)] = c;
    if (mask_row && in) mask_row[c] = sel ? 1 : 0;
    base += __popc(selm);
    eq_seen += __popc(eqm);
  }
  for (int p = k + lane; p < k_cap; p += 32) idx_row[p] = -1;
  if (mask_row)
    for (int c = nt + lane; c < g.nt_cap; c += 32) mask_row[c] = 0;
}

template <int KPL>
cudaError_t launch_bisect(const LayerGeom& g, const float* scores, int k_cap, int32_t* idx, uint8_t* mask,
                          cudaStream_t s, const int32_t* head_on) {
  const long long rows = (long long)g.B * g.heads * g.nt_cap;
  const long long blocks = (rows + BIS_WARPS - 1) / BIS_WARPS;
  if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
  topk_bisect_kernel<KPL><<<(unsigned)blocks, BIS_WARPS * 32, 0, s>>>(g, scores, k_cap, idx, mask, head_on);
  return cudaGetLastError();
}

// Tile scores and top-k in one pass (Veda summary 2.1; the pages name
// tighter kernel fusion as future work). A CTA takes R query tiles of one
// head, computes their whole score rows scale * q_i . k_j into shared memory
// with the same fma order as the score GEMM kernel (so scores and selections
// are bit-identical to the unfused path) and selects from there: the score
// matrix reaches HBM only when the caller asks for it. Measured 1.07 ms
// against 0.85 ms for the score GEMM plus top-k kernels on the 153,600-token
// layer (the per-thread dot products with broadcast shared-memory operands
// cannot match the register-tiled GEMM), so the layer uses the unfused pair.
constexpr int ST_THREADS = 256, ST_WARPS = ST_THREADS / 32, ST_RMAX = 8;

__global__ void __launch_bounds__(ST_THREADS) score_topk_kernel(const __grid_constant__ LayerGeom g,
                                                                const float* __restrict__ emb, int out_dim,
                                                                float scale, int R, int k_cap,
                                                                int32_t* __restrict__ idx,
                                                                uint8_t* __restrict__ mask,
                                                                float* __restrict__ scores) {
  extern __shared__ uint32_t sm_u32[];
  float* qs = reinterpret_cast<float*>(sm_u32);                  // [R][out_dim], 16-byte rows (out_dim % 4 == 0)
  uint32_t* hist = sm_u32 + R * out_dim;                         // [ST_WARPS][256]
  uint32_t* keys = hist + ST_WARPS * 256;                        // [R][nt_cap] order keys
  const int h = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * R;
  const HeadGeom& hg = g.h[h];
  const int nt = hg.nt;
  const long long bh = (long long)b * g.heads + h;
  const float* Q = emb + bh * g.nt_cap * out_dim;
  const float* K = emb + ((long long)g.B * g.heads + bh) * g.nt_cap * out_dim;
  for (int t = threadIdx.x; t < R * out_dim; t += ST_THREADS) {
    const int r = t / out_dim;
    qs[t] = i0 + r < nt ? Q[(long long)i0 * out_dim + t] : 0.f;
  }
  __syncthreads();
  // one key tile per thread at a time, all R rows against it
  for (int j = threadIdx.x; j < g.nt_cap; j += ST_THREADS) {
    float acc[ST_RMAX];
#pragma unroll
    for (int r = 0; r < ST_RMAX; ++r) acc[r] = 0.f;
    if (j < nt) {
      const float4* kr = reinterpret_cast<const float4*>(K + (long long)j * out_dim);
      for (int e4 = 0; e4 < out_dim / 4; ++e4) {
        const float4 kv = __ldg(kr + e4);
#pragma unroll
        for (int r = 0; r < ST_RMAX; ++r) {
          if (r < R) {
            const float4 qv = *reinterpret_cast<const float4*>(qs + r * out_dim + 4 * e4);
            acc[r] = fmaf(qv.x, kv.x, acc[r]);
            acc[r] = fmaf(qv.y, kv.y, acc[r]);
            acc[r] = fmaf(qv.z, kv.z, acc[r]);
            acc[r] = fmaf(qv.w, kv.w, acc[r]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < ST_RMAX; ++r) {
      if (r < R) {
        const int i = i0 + r;
        const float sc = (i < nt && j < nt) ? acc[r] * scale : 0.f;
        keys[r * g.nt_cap + j] = order_key(sc);
        if (scores && i < g.nt_cap) scores[(bh * g.nt_cap + i) * g.nt_cap + j] = sc;
      }
    }
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int r = warp; r < R; r += ST_WARPS) {
    const int i = i0 + r;
    if (i >= g.nt_cap) break;
    int32_t* idx_row = idx + (bh * g.nt_cap + i) * k_cap;
    uint8_t* mask_row = mask ? mask + (bh * g.nt_cap + i) * g.nt_cap : nullptr;
    if (i >= nt) {  // query tile beyond this head's tiles
      for (int p = lane; p < k_cap; p += 32) idx_row[p] = -1;
      if (mask_row)
        for (int c = lane; c < g.nt_cap; c += 32) mask_row[c] = 0;
      continue;
    }
    warp_select_row(keys + r * g.nt_cap, hist + warp * 256, nt, hg.k, k_cap, g.nt_cap, idx_row, mask_row, lane);
  }
}

// Recall of the predicted top-k lists against the tile map's own top-k
// (Veda summary 2.1, Target Construction: the max-pooled full-attention map
// is the target the estimator is aligned to). One warp per (selected head,
// sampled query tile): the map row is ranked exactly as a score row is ranked
// here (order keys, the head's k, exact ties to the lower tile index) into a
// list in shared memory; the hits are the tiles held both by that list and
// by the predicted list of the same query tile, counted over two kept-tile
// bitmaps (set semantics, so a repeated predicted entry counts once).
struct RecallParams {
  int32_t heads_sel[VEDA_MAX_HEADS];
  const int32_t* rows;    // [n_sel, n_rows] query tiles, or NULL: 0..n_rows-1
  const float* tilemap;   // [n_sel, n_rows, nt_cap]
  const int32_t* idx;     // predicted lists [B = 1, heads, nt_cap, k_cap]
  int32_t* map_idx;       // [n_sel, n_rows, k_cap] or NULL
  int32_t* hits;          // [n_sel, n_rows]
  float* recall;          // [n_sel + 1]
  int32_t n_sel, n_rows, k_cap, warps;
};

// 32-bit words of one warp's shared area: order keys, radix histogram, the
// map's selected list, and two kept-tile bitmaps.
__host__ __device__ inline int recall_warp_words(int nt_cap, int k_cap) {
  return nt_cap + 256 + k_cap + 2 * ((nt_cap + 31) / 32);
}

__global__ void __launch_bounds__(128) recall_rows_kernel(const __grid_constant__ LayerGeom g,
                                                          const __grid_constant__ RecallParams prm) {
  extern __shared__ uint32_t sm_u32[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int words = (g.nt_cap + 31) / 32;
  uint32_t* keys = sm_u32 + warp * recall_warp_words(g.nt_cap, prm.k_cap);
  uint32_t* hist = keys + g.nt_cap;
  int32_t* sel = reinterpret_cast<int32_t*>(hist + 256);
  uint32_t* bm_map = reinterpret_cast<uint32_t*>(sel + prm.k_cap);
  uint32_t* bm_pred = bm_map + words;
  const long long row = (long long)blockIdx.x * prm.warps + warp;
  if (warp >= prm.warps || row >= (long long)prm.n_sel * prm.n_rows) return;
  const int s = (int)(row / prm.n_rows), r = (int)(row % prm.n_rows);
  const int h = prm.heads_sel[s];
  const int nt = g.h[h].nt, k = g.h[h].k;
  const int a = prm.rows ? __ldg(prm.rows + row) : r;
  int32_t* mrow = prm.map_idx ? prm.map_idx + row * prm.k_cap : nullptr;
  if (a < 0 || a >= nt) {  // not a query tile of this head: no hits, empty list
    if (lane == 0) {
      prm.hits[row] = 0;
      report(g.dev_status, VEDA_ERR_BAD_INDEX);
    }
    if (mrow)
      for (int p = lane; p < prm.k_cap; p += 32) mrow[p] = -1;
    return;
  }
  const float* M = prm.tilemap + row * g.nt_cap;
  for (int c = lane; c < nt; c += 32) keys[c] = order_key(__ldg(M + c));
  for (int w = lane; w < words; w += 32) bm_map[w] = bm_pred[w] = 0u;
  __syncwarp();
  warp_select_row(keys, hist, nt, k, prm.k_cap, g.nt_cap, sel, nullptr, lane);
  __syncwarp();
  const int32_t* pred = prm.idx + ((long long)h * g.nt_cap + a) * prm.k_cap;
  bool bad = false;
  for (int p = lane; p < k; p += 32) {
    const int t = sel[p];
    atomicOr(bm_map + (t >> 5), 1u << (t & 31));
    const int u = __ldg(pred + p);
    if (u >= 0 && u < nt) atomicOr(bm_pred + (u >> 5), 1u << (u & 31));
    else bad = true;
  }
  __syncwarp();
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(g.dev_status, VEDA_ERR_BAD_INDEX);
  unsigned c = 0;
  for (int w = lane; w < words; w += 32) c += __popc(bm_map[w] & bm_pred[w]);
  c = __reduce_add_sync(0xffffffffu, c);
  if (lane == 0) prm.hits[row] = (int32_t)c;
  if (mrow)
    for (int p = lane; p < prm.k_cap; p += 32) mrow[p] = sel[p];
}

// recall[s] = (sum of head s's hits) / (n_rows * k_h); recall[n_sel] = the
// mean over the selected heads, in head order. Hit sums are integers, so the
// result does not depend on the order of the additions.
__global__ void __launch_bounds__(256) recall_mean_kernel(const __grid_constant__ LayerGeom g,
                                                          const __grid_constant__ RecallParams prm) {
  __shared__ unsigned long long part[256];
  __shared__ double per_head[VEDA_MAX_HEADS];
  for (int s = 0; s < prm.n_sel; ++s) {
    unsigned long long c = 0;
    for (int r = threadIdx.x; r < prm.n_rows; r += 256) c += (unsigned long long)prm.hits[(long long)s * prm.n_rows + r];
    part[threadIdx.x] = c;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
      if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0) {
      const double v = (double)part[0] / ((double)prm.n_rows * g.h[prm.heads_sel[s]].k);
      per_head[s] = v;
      prm.recall[s] = (float)v;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    double m = 0.0;
    for (int s = 0; s < prm.n_sel; ++s) m += per_head[s];
    prm.recall[prm.n_sel] = (float)(m / prm.n_sel);
  }
}

}  // namespace

cudaError_t launch_topk(const LayerGeom& g, const float* scores, int k_cap, int32_t* idx, uint8_t* mask,
                        cudaStream_t s, const int32_t* head_on) {
  // register-resident keys: the smallest multiple of 8 keys per lane that
  // holds a row
  const int kpl = (g.nt_cap + 32 * 8 - 1) / (32 * 8) * 8;
  switch (kpl) {
    case 8: return launch_bisect<8>(g, scores, k_cap, idx, mask, s, head_on);
    case 16: return launch_bisect<16>(g, scores, k_cap, idx, mask, s, head_on);
    case 24: return launch_bisect<24>(g, scores, k_cap, idx, mask, s, head_on);
    case 32: return launch_bisect<32>(g, scores, k_cap, idx, mask, s, head_on);
    case 40: return launch_bisect<40>(g, scores, k_cap, idx, mask, s, head_on);
    case 48: return launch_bisect<48>(g, scores, k_cap, idx, mask, s, head_on);
    case 56: return launch_bisect<56>(g, scores, k_cap, idx, mask, s, head_on);
    case 64: return launch_bisect<64>(g, scores, k_cap, idx, mask, s, head_on);
    default: break;
  }
  const size_t smem = (size_t)TOPK_WARPS * (g.nt_cap + 256) * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)g.B * g.heads * g.nt_cap;
  const long long blocks = (rows + TOPK_WARPS - 1) / TOPK_WARPS;
  if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
  topk_radix_kernel<<<(unsigned)blocks, TOPK_WARPS * 32, smem, s>>>(g, scores, k_cap, idx, mask, head_on);
  return cudaGetLastError();
}

// Rows per CTA: as many as fit 200 KB of shared memory with the order keys
// of whole rows, at most 8 (4 and 16 measured slower on the 153,600-token
// layer: fewer rows re-read the key embeddings more often, more rows leave
// too few CTAs per SM for the latency-bound selection).
cudaError_t launch_score_topk(const LayerGeom& g, const float* emb_ws, int out_dim, float scale, int k_cap,
                              int32_t* idx, uint8_t* mask, float* scores, cudaStream_t s) {
  const size_t fixed = (size_t)ST_WARPS * 256 * 4;
  const size_t per_row = (size_t)g.nt_cap * 4 + (size_t)out_dim * 4;
  int R = (int)((200 * 1024 - fixed) / per_row);
  R = R > ST_RMAX ? ST_RMAX : R;
  if (R < 1) return cudaErrorInvalidValue;
  const size_t smem = fixed + (size_t)R * per_row;
  cudaError_t e = cudaFuncSetAttribute(score_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((g.nt_cap + R - 1) / R, g.heads, g.B);
  score_topk_kernel<<<grid, ST_THREADS, smem, s>>>(g, emb_ws, out_dim, scale, R, k_cap, idx, mask, scores);
  return cudaGetLastError();
}

cudaError_t launch_recall(const LayerGeom& g, const int32_t* heads_sel, int n_sel, const int32_t* rows, int n_rows,
                          const float* tilemap, const int32_t* idx, int k_cap, int32_t* hits, int32_t* map_idx,
                          float* recall, cudaStream_t s) {
  RecallParams prm;
  for (int i = 0; i < VEDA_MAX_HEADS; ++i) prm.heads_sel[i] = i < n_sel ? heads_sel[i] : 0;
  prm.rows = rows;
  prm.tilemap = tilemap;
  prm.idx = idx;
  prm.map_idx = map_idx;
  prm.hits = hits;
  prm.recall = recall;
  prm.n_sel = n_sel;
  prm.n_rows = n_rows;
  prm.k_cap = k_cap;
  const size_t per_warp = (size_t)recall_warp_words(g.nt_cap, k_cap) * sizeof(uint32_t);
  int warps = (int)((200 * 1024) / per_warp);
  warps = warps > 4 ? 4 : warps;
  if (warps < 1) return cudaErrorInvalidValue;
  prm.warps = warps;
  const size_t smem = (size_t)warps * per_warp;
  cudaError_t e = cudaFuncSetAttribute(recall_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long total = (long long)n_sel * n_rows;
  recall_rows_kernel<<<(unsigned)((total + warps - 1) / warps), 128, smem, s>>>(g, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  recall_mean_kernel<<<1, 256, 0, s>>>(g, prm);
  return cudaGetLastError();
}

}  // namespace veda
