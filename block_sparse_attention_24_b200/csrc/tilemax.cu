// Oracle tile map and row-wise KL (Veda summary 2.1, Target Construction and
// Optimization; 2.3, Training Efficiency: the heat map is built in two
// passes, on a subset of query tiles).
//
// Two 128-row blocks of selected query tiles share one CTA and every K block
// load. M[a, b] = max over the tile region of the softmax probability =
// exp2(max over the tile's valid rows of (row's largest logit in key tile b
// * C - row's log2-sum-exp)). Without a workspace each CTA sweeps all key
// blocks twice with tcgen05 S = Q K^T:
//   pass 1: per row, log2-domain log-sum-exp over all valid keys;
//   pass 2: per row and key tile, the largest logit minus lse, then the
//           maximum over the tile's valid rows (warp shuffle, then a shared
//           order-preserving atomicMax).
// With a workspace the key range may be split over several CTAs and there is
// one sweep: it writes each row's partial (reference, sum) and its largest
// logit per key tile; map_finish_kernel combines the partial sums in a fixed
// order and reduces the stored maxima over rows (the same values pass 2 would
// recompute, so the same map).
// A further kernel turns map rows and score rows into KL values, another
// averages them in a fixed order.
#include <climits>

#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int BM = 128, BN = 128;
constexpr int KST = 3;                 // K ring stages
constexpr uint32_t TMEM_COLS = 512;    // S buffers: row-block r, buffer b at (2r + b) * 128
constexpr int NUM_THREADS = 384;
constexpr int MAP_MAX_SPLIT = 8;       // most CTAs one row pair's key range is split over
// softmax warpgroups 216 registers, producer/MMA warpgroup 72:
// 2*128*216 + 128*72 = 64,512 = the 384*168 the launch reserves (208/88
// removes the producer warps' few spills but measured 10% slower)
constexpr int REGS_SOFTMAX = 216, REGS_ROLES = 72;
constexpr float OVERFLOW_SUM = 1.8446744e19f;  // 2^64: a tile's exp sum above this moves the reference

template <int D>
struct MapLayout {
  static constexpr int QB = BM * D * 2;  // one 128-row block of Q
  static constexpr int KB = BN * D * 2;
  static constexpr int OFF_Q = 0;        // row blocks A, B
  static constexpr int OFF_K = 2 * QB;
  static constexpr int OFF_BAR = OFF_K + KST * KB;
  // q_full, k_full[KST], k_empty[KST], s_full[4], s_free[4], drain
  static constexpr int NUM_BARS = 1 + 2 * KST + 4 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_PART = (OFF_MISC + 16 + 15) / 16 * 16;
  static int bytes(int nt_cap, int nsub) { return OFF_PART + 2 * nsub * nt_cap * 4 + 1024; }
};

struct MapParams {
  float scale_log2;
  int mode;             // 0: both passes; 1: one sweep, partial sums and row maxima to ws
  int n_split;          // CTAs sharing one row pair's key range (blockIdx.z); 1 for mode 0
  float2* ws;           // [n_heads_sel][n_rows][tile][n_split] (reference m, sum l) in log2 units
  float* rowmax;        // [n_heads_sel][n_rows][nt_cap][tile] largest logit per row and key tile
  int n_rows;
  const int32_t* rows;  // [n_heads_sel, n_rows] or NULL
  float* tilemap;       // [n_heads_sel, n_rows, nt_cap]
  float* lse;           // [n_heads_sel, n_rows, tile] or NULL
  int heads_sel[VEDA_MAX_HEADS];
};

__device__ __forceinline__ uint32_t ord_f32(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_f32(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Maximum of columns [c0, c0+TILE) of a row of S over the first `klen` of
// them (all when FULL).
template <int TILE, bool FULL>
__device__ __forceinline__ float tile_max(const uint32_t (&u)[BN], int c0, int klen) {
  float pm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < TILE; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k0 = c + i, k1 = k0 + 8;
      const float v0 = (FULL || k0 < klen) ? __uint_as_float(u[c0 + k0]) : -INFINITY;
      const float v1 = (FULL || k1 < klen) ? __uint_as_float(u[c0 + k1]) : -INFINITY;
      pm[i] = fmax3(pm[i], v0, v1);
    }
  return fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
}

// Sum over columns [c0, c0+TILE) (the first `klen`, all when FULL) of
// 2^(s*C - mref); packed fp32x2 math, exponentials on MUFU.
template <int TILE, bool FULL>
__device__ __forceinline__ float tile_expsum(const uint32_t (&u)[BN], int c0, int klen, uint64_t C2, uint64_t NM) {
  uint64_t acc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = f2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < TILE / 2; ++w) {
    const int k0 = 2 * w;
    const uint64_t y = f2_fma(f2(__uint_as_float(u[c0 + k0]), __uint_as_float(u[c0 + k0 + 1])), C2, NM);
    float y0, y1;
    f2_split(y, y0, y1);
    uint64_t p = f2(fast_exp2(y0), fast_exp2(y1));
    if (!FULL) {
      float p0, p1;
      f2_split(p, p0, p1);
      p = f2(k0 < klen ? p0 : 0.f, k0 + 1 < klen ? p1 : 0.f);
    }
    acc[w & 3] = f2_add(acc[w & 3], p);
  }
  float lo, hi;
  f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lo, hi);
  return lo + hi;
}

// One CTA owns two 128-row blocks (A, B) of selected query rows of one head:
// one 128-token query tile each, or two 64-token query tiles each. Both
// sweep every key block of the CTA's range, twice in mode 0 (pass 1:
// log-sum-exp; pass 2: per key tile max of logit - lse, then max over the
// tile's rows), once in mode 1 (partial log-sum-exp and per key tile row
// maxima to the workspace); each K block is loaded once for both. S of each row block is double-buffered in TMEM, so the MMA
// for the next key block overlaps the softmax of the current one.
//   warps 0-3 / 4-7  row block A / B (thread = row = TMEM lane)
//   warp 8           TMA producer (Q once, then K blocks, 3-stage ring)
//   warp 9           MMA issuer (one thread)
//   warps 10-11      idle
template <int D, int TILE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tilemax_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ MapParams prm) {
  using Lay = MapLayout<D>;
  constexpr int NSUB = BM / TILE;  // query tiles per row block
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

  const int hs = blockIdx.y;
  const int h = prm.heads_sel[hs];
  const int bh = h;  // B == 1
  const HeadGeom& hg = g.h[h];
  const int nt = hg.nt;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_kb = (nt * TILE + BN - 1) / BN;
  // this CTA's share of the key blocks (all of them unless the key range is
  // split over blockIdx.z)
  const int split = blockIdx.z;
  const int kb_begin = (int)((long long)n_kb * split / prm.n_split);
  const int kb_end = (int)((long long)n_kb * (split + 1) / prm.n_split);
  const int nkb = kb_end - kb_begin;
  const int iters = (prm.mode == 0 ? 2 : 1) * nkb;

  // selected query tiles: entry (2*blockIdx.x + r)*NSUB + s of the row list
  int qt[2][NSUB];
  bool qv[2][NSUB];
  bool rb_valid[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    rb_valid[r] = false;
#pragma unroll
    for (int s = 0; s < NSUB; ++s) {
      const int e = (2 * blockIdx.x + r) * NSUB + s;
      qv[r][s] = e < prm.n_rows;
      int a = qv[r][s] ? (prm.rows ? __ldg(prm.rows + (long long)hs * prm.n_rows + e) : e) : 0;
      if (a < 0 || a >= nt) {
        if (qv[r][s]) report(g.dev_status, VEDA_ERR_BAD_INDEX);
        a = 0;
        qv[r][s] = false;
      }
      qt[r][s] = a;
      rb_valid[r] = rb_valid[r] || qv[r][s];
    }
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* s_full = k_empty + KST;  // [row block * 2 + buffer]
  uint64_t* s_free = s_full + 4;     // [row block * 2 + buffer], 128 arrivals each
  uint64_t* drain = s_free + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);
  uint32_t* part = reinterpret_cast<uint32_t*>(smem + Lay::OFF_PART);  // [2][NSUB][nt_cap] ordered maxima

  if (threadIdx.x == 0) {
    for (int i = 0; i < Lay::NUM_BARS; ++i) {
      uint64_t* bar = bars + i;
      mbar_init(bar, (bar >= s_free && bar < s_free + 4) ? 128 : 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * NSUB * g.nt_cap; i += NUM_THREADS) part[i] = 0u;  // 0 = no contribution
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_lower<REGS_ROLES>();
    if (warp == 8 && lane == 0) {
      // ------------------------------------------------------- producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_expect_tx(q_full, 2 * Lay::QB);
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int s = 0; s < NSUB; ++s)
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_3d(smem + Lay::OFF_Q + r * Lay::QB + bx * BM * 128 + s * TILE * 128, &tmQ, q_full, bx * 64,
                        qt[r][s] * TILE, bh);
      int issued = 0;
      for (int it = 0; it < iters; ++it) {
        const int st = it % KST;
        if (it >= KST && !mbar_wait(k_empty + st, ((it - KST) / KST) & 1, abort_flag, g.dev_status)) break;
        mbar_expect_tx(k_full + st, Lay::KB);
        const int kb = kb_begin + it % nkb;
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_3d(smem + Lay::OFF_K + st * Lay::KB + bx * BN * 128, &tmK, k_full + st, bx * 64, kb * BN, bh);
        issued = it + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(q_full, 0, VEDA_WAIT_LIMIT_NS);
        for (int it = issued - KST < 0 ? 0 : issued - KST; it < issued; ++it)
          mbar_wait_drain(k_full + it % KST, (it / KST) & 1, VEDA_WAIT_LIMIT_NS);
      }
    } else if (warp == 9 && lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      const uint32_t aQ = smem_u32(smem + Lay::OFF_Q);
      const uint32_t aK = smem_u32(smem + Lay::OFF_K);
      if (mbar_wait(q_full, 0, abort_flag, g.dev_status)) {
        tc_fence_after();
        bool ok = true;
        for (int it = 0; it < iters && ok; ++it) {
          const int st = it % KST, buf = it & 1;
          if (!mbar_wait(k_full + st, (it / KST) & 1, abort_flag, g.dev_status)) break;
          tc_fence_after();
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            if (!rb_valid[r]) continue;
            const int sb = 2 * r + buf;
            if (it >= 2 && !(ok = mbar_wait(s_free + sb, ((it - 2) >> 1) & 1, abort_flag, g.dev_status))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
              umma_bf16_ss(tmem + sb * BN, sdesc_sw128(aQ + r * Lay::QB + off, 16, 1024),
                           sdesc_sw128(aK + st * Lay::KB + off, 16, 1024), idesc, kk > 0);
            }
            umma_commit(s_full + sb);
          }
          if (ok) umma_commit(k_empty + st);
        }
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0, VEDA_WAIT_LIMIT_NS);
    }
  } else {
    regs_raise<REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    const int r = warp / 4;                 // row block
    const int row = threadIdx.x % BM;       // TMEM lane
    const int qs = row / TILE;              // query tile within the row block
    const bool row_valid = qv[r][qs] && (row % TILE) < tile_len(hg, g.T, qt[r][qs]);
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const float C = prm.scale_log2;
    const uint64_t C2 = f2(C, C);
    float m = -INFINITY, l = 0.f, lse2 = 0.f;
    const int e_row = (2 * blockIdx.x + r) * NSUB + qs;  // this row's entry in the row list
    // partial (reference, sum) of row `row` of entry e_row from split sp
    auto part_ws = [&](int sp) -> float2* {
      return prm.ws + (((long long)hs * prm.n_rows + e_row) * TILE + (row % TILE)) * prm.n_split + sp;
    };
    const bool keep_max = prm.mode == 1 && e_row < prm.n_rows;
    for (int it = 0; it < (rb_valid[r] ? iters : 0); ++it) {
      const int sb = 2 * r + (it & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + sb, (it >> 1) & 1, abort_flag, g.dev_status))) break;
      tc_fence_after();
      uint32_t u[BN];
      tmem_ld128(lane_addr + sb * BN, u);
      tc_fence_before();
      mbar_arrive(s_free + sb);  // S buffer may be overwritten now
      const int kb = kb_begin + it % nkb;
      const bool pass2 = prm.mode == 0 && it >= nkb;
#pragma unroll
      for (int uu = 0; uu < NSUB; ++uu) {
        const int kt = kb * NSUB + uu;
        const int klen = kt < nt ? tile_len(hg, g.T, kt) : 0;
        const bool full = klen >= TILE;
        auto block_max = [&]() {
          return full ? tile_max<TILE, true>(u, uu * TILE, klen) : tile_max<TILE, false>(u, uu * TILE, klen);
        };
        auto block_sum = [&](float mref) {
          const uint64_t NM = f2(-mref, -mref);
          return full ? tile_expsum<TILE, true>(u, uu * TILE, klen, C2, NM)
                      : tile_expsum<TILE, false>(u, uu * TILE, klen, C2, NM);
        };
        if (!pass2) {
          // Only the row's first key tile is max-reduced; later tiles sum
          // 2^(s*C - m) against that reference, which fp32 carries at full
          // relative precision, and move it only when a tile's sum nears the
          // top of the range (rare).
          if (klen > 0) {
            float mx = 0.f;
            if (keep_max) {  // the row's largest logit in key tile kt, for the map
              mx = block_max();
              prm.rowmax[(((long long)hs * prm.n_rows + e_row) * g.nt_cap + kt) * TILE + (row % TILE)] = mx;
            }
            if (m == -INFINITY) m = (keep_max ? mx : block_max()) * C;
            float sum = block_sum(m);
            if (!(sum <= OVERFLOW_SUM)) {
              const float mnew = fmaxf(m, (keep_max ? mx : block_max()) * C);
              l *= fast_exp2(m - mnew);
              m = mnew;
              sum = block_sum(m);
            }
            l += sum;
          }
        } else {
          const float mx = block_max();
          float v = (row_valid && klen > 0) ? fmaf(mx, C, -lse2) : -INFINITY;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0 && kt < nt && v > -INFINITY) atomicMax(part + (r * NSUB + qs) * g.nt_cap + kt, ord_f32(v));
        }
      }
      if (prm.mode == 0 && it == nkb - 1) {
        lse2 = m + __log2f(l);
        if (prm.lse && e_row < prm.n_rows)
          prm.lse[((long long)hs * prm.n_rows + e_row) * TILE + (row % TILE)] = row_valid ? lse2 * 0.69314718055994531f : 0.f;
      }
    }
    if (prm.mode == 1 && e_row < prm.n_rows) *part_ws(split) = make_float2(m, l);
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // mode 0: write the map rows (zero columns past nt included)
  const int kt_begin = 0, kt_end = g.nt_cap;
  if (!*abort_flag && prm.mode == 0) {
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int s = 0; s < NSUB; ++s) {
        const int e = (2 * blockIdx.x + r) * NSUB + s;
        if (e >= prm.n_rows) continue;
        float* out = prm.tilemap + ((long long)hs * prm.n_rows + e) * g.nt_cap;
        for (int b = kt_begin + threadIdx.x; b < kt_end; b += NUM_THREADS) {
          const uint32_t k = part[(r * NSUB + s) * g.nt_cap + b];
          out[b] = (b < nt && k != 0u && qv[r][s]) ? fast_exp2(unord_f32(k)) : 0.f;
        }
      }
  }
}

constexpr int FIN_THREADS = 256;
constexpr int FIN_KT = 64;  // key tiles per finishing CTA

// Finishes a mode-1 map: per row, the fixed-order combination of the splits'
// partial (reference, sum) into the log2-sum-exp; per key tile, the maximum
// over the query tile's valid rows of (largest logit * C - lse), as 2^max.
// Grid: (key-tile chunks, selected rows, selected heads); warp per key tile.
template <int TILE>
__global__ void __launch_bounds__(FIN_THREADS)
    map_finish_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ MapParams prm) {
  __shared__ float lse2s[TILE];
  const int hs = blockIdx.z;
  const int h = prm.heads_sel[hs];
  const HeadGeom& hg = g.h[h];
  const int nt = hg.nt;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float C = prm.scale_log2;
  const int kt_end = min(g.nt_cap, (int)(blockIdx.x + 1) * FIN_KT);
  for (int e = blockIdx.y; e < prm.n_rows; e += gridDim.y) {
    const int a = prm.rows ? __ldg(prm.rows + (long long)hs * prm.n_rows + e) : e;
    const bool qv = a >= 0 && a < nt;  // a bad entry was reported by the sweep
    const int len = qv ? tile_len(hg, g.T, a) : 0;
    const long long er = (long long)hs * prm.n_rows + e;
    __syncthreads();  // lse2s of the previous row is no longer read
    if (threadIdx.x < TILE) {
      const int row = threadIdx.x;
      const float2* part = prm.ws + (er * TILE + row) * prm.n_split;
      float M = -INFINITY;
      for (int sp = 0; sp < prm.n_split; ++sp) M = fmaxf(M, part[sp].x);
      float L = 0.f;
      for (int sp = 0; sp < prm.n_split; ++sp) {
        const float2 pr = part[sp];
        if (pr.y > 0.f) L += pr.y * fast_exp2(pr.x - M);
      }
      const float lse2 = M + __log2f(L);
      lse2s[row] = lse2;
      if (prm.lse && blockIdx.x == 0) prm.lse[er * TILE + row] = row < len ? lse2 * 0.69314718055994531f : 0.f;
    }
    __syncthreads();
    for (int kt = blockIdx.x * FIN_KT + warp; kt < kt_end; kt += FIN_THREADS / 32) {
      float out = 0.f;
      if (kt < nt && qv) {
        const float* mx = prm.rowmax + (er * g.nt_cap + kt) * TILE;
        float v = -INFINITY;
#pragma unroll
        for (int j = 0; j < TILE / 32; ++j) {
          const int row = lane + 32 * j;
          if (row < len) v = fmaxf(v, fmaf(__ldg(mx + row), C, -lse2s[row]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        out = v > -INFINITY ? fast_exp2(v) : 0.f;
      }
      if (lane == 0) prm.tilemap[er * g.nt_cap + kt] = out;
    }
  }
}

__global__ void kl_rows_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ MapParams prm,
                               int n_heads_sel, const float* __restrict__ scores, float* __restrict__ kl_rows) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32, lane = threadIdx.x % 32;
  if (warp >= n_heads_sel * prm.n_rows) return;
  const int hs = warp / prm.n_rows, rr = warp % prm.n_rows;
  const int h = prm.heads_sel[hs];
  const int nt = g.h[h].nt;
  int a = prm.rows ? __ldg(prm.rows + (long long)hs * prm.n_rows + rr) : rr;
  if (a < 0 || a >= nt) {
    if (lane == 0) kl_rows[warp] = 0.f;
    return;
  }
  const float* M = prm.tilemap + (long long)warp * g.nt_cap;
  const float* S = scores + ((long long)h * g.nt_cap + a) * g.nt_cap;
  float msum = 0.f, smax = -INFINITY;
  for (int b = lane; b < nt; b += 32) {
    msum += M[b];
    smax = fmaxf(smax, S[b]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    msum += __shfl_xor_sync(0xffffffffu, msum, off);
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
  }
  float z = 0.f;
  for (int b = lane; b < nt; b += 32) z += expf(S[b] - smax);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float logz = logf(z), log_msum = logf(msum);
  float kl = 0.f;
  for (int b = lane; b < nt; b += 32) {
    const float mb = M[b];
    if (mb > 0.f) {
      const float t = mb / msum;
      kl += t * ((logf(mb) - log_msum) - (S[b] - smax - logz));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kl += __shfl_xor_sync(0xffffffffu, kl, off);
  if (lane == 0) kl_rows[warp] = kl;
}

__global__ void kl_mean_kernel(const float* __restrict__ kl_rows, int n_heads_sel, int n_rows, float* __restrict__ out) {
  __shared__ float red[32];
  float total = 0.f;
  for (int hs = 0; hs < n_heads_sel; ++hs) {
    float acc = 0.f;
    for (int r = threadIdx.x; r < n_rows; r += blockDim.x) acc += kl_rows[(long long)hs * n_rows + r];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
      for (int w = 0; w < (int)(blockDim.x / 32); ++w) s += red[w];
      total += s / (float)n_rows;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = total / (float)n_heads_sel;
}

template <int D, int TILE>
cudaError_t launch_map_t(const LayerGeom& g, const void* qp, const void* kp, MapParams prm, int n_heads_sel,
                         cudaStream_t s) {
  CUtensorMap tq, tk;
  const uint64_t rows = (uint64_t)g.n_cap, planes = (uint64_t)g.B * g.heads;
  if (encode_tensor_map_3d_bf16(&tq, qp, D, rows, planes, 64, TILE) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&tk, kp, D, rows, planes, 64, BN) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = tilemax_kernel<D, TILE>;
  constexpr int NSUB = BM / TILE;
  const int smem = MapLayout<D>::bytes(g.nt_cap, NSUB);
  if (smem > 232448) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int pairs = (prm.n_rows + 2 * NSUB - 1) / (2 * NSUB);
  // With a workspace: one sweep (mode 1), with each row pair's key range split
  // over n_split CTAs when that fills the SMs' waves noticeably better (one
  // CTA per SM), then map_finish_kernel.
  int n_split = 1;
  if (prm.ws) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int n_kb_min = INT_MAX;
    for (int i = 0; i < n_heads_sel; ++i) {
      const int nt = g.h[prm.heads_sel[i]].nt;
      const int nkb = (nt * TILE + BN - 1) / BN;
      n_kb_min = nkb < n_kb_min ? nkb : n_kb_min;
    }
    const long long base = (long long)pairs * n_heads_sel;
    auto fill = [&](int sp) {
      const long long ctas = base * sp, waves = (ctas + sms - 1) / sms;
      return (double)ctas / (double)(waves * sms);
    };
    double best = fill(1);
    for (int sp = 2; sp <= MAP_MAX_SPLIT && n_kb_min / sp >= 4; ++sp)
      if (fill(sp) > best + 0.05) {
        best = fill(sp);
        n_split = sp;
      }
  }
  if (!prm.ws) {
    prm.mode = 0;
    prm.n_split = 1;
    kern<<<dim3(pairs, n_heads_sel, 1), NUM_THREADS, smem, s>>>(g, tq, tk, prm);
    return cudaGetLastError();
  }
  prm.n_split = n_split;
  prm.mode = 1;
  kern<<<dim3(pairs, n_heads_sel, n_split), NUM_THREADS, smem, s>>>(g, tq, tk, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 fgrid((g.nt_cap + FIN_KT - 1) / FIN_KT, prm.n_rows < 65535 ? prm.n_rows : 65535, n_heads_sel);
  map_finish_kernel<TILE><<<fgrid, FIN_THREADS, 0, s>>>(g, prm);
  return cudaGetLastError();
}

}  // namespace

// partial sums [heads][rows][tile][MAP_MAX_SPLIT] float2, then the row
// maxima [heads][rows][nt_cap][tile] float
size_t tilemax_ws_bytes(int n_heads_sel, int n_rows, int tile, int nt_cap) {
  const size_t rows = (size_t)n_heads_sel * n_rows * tile;
  return rows * MAP_MAX_SPLIT * sizeof(float2) + rows * nt_cap * sizeof(float);
}

cudaError_t launch_tilemax(const LayerGeom& g, const void* qp, const void* kp, const int32_t* heads_sel,
                           int n_heads_sel, const int32_t* rows, int n_rows, float scale, float* tilemap, float* lse,
                           const float* scores, float* kl_rows, float* kl_out, float* ws, cudaStream_t s) {
  MapParams prm;
  prm.mode = 0;
  prm.n_split = 1;
  prm.ws = reinterpret_cast<float2*>(ws);
  prm.rowmax = ws ? ws + (size_t)n_heads_sel * n_rows * g.tile * MAP_MAX_SPLIT * 2 : nullptr;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.n_rows = n_rows;
  prm.rows = rows;
  prm.tilemap = tilemap;
  prm.lse = lse;
  for (int i = 0; i < VEDA_MAX_HEADS; ++i) prm.heads_sel[i] = i < n_heads_sel ? heads_sel[i] : 0;
  cudaError_t e;
  if (g.d == 128 && g.tile == 128) e = launch_map_t<128, 128>(g, qp, kp, prm, n_heads_sel, s);
  else if (g.d == 128 && g.tile == 64) e = launch_map_t<128, 64>(g, qp, kp, prm, n_heads_sel, s);
  else if (g.d == 64 && g.tile == 128) e = launch_map_t<64, 128>(g, qp, kp, prm, n_heads_sel, s);
  else e = launch_map_t<64, 64>(g, qp, kp, prm, n_heads_sel, s);
  if (e != cudaSuccess || !scores) return e;
  const int warps = n_heads_sel * n_rows;
  kl_rows_kernel<<<(warps * 32 + 255) / 256, 256, 0, s>>>(g, prm, n_heads_sel, scores, kl_rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kl_mean_kernel<<<1, 1024, 0, s>>>(kl_rows, n_heads_sel, n_rows, kl_out);
  return cudaGetLastError();
}

// The row-wise KL of a finished map (kl_rows_kernel + kl_mean_kernel), for
// callers that build the map before the scores exist.
cudaError_t launch_tilemap_kl(const LayerGeom& g, const int32_t* heads_sel, int n_heads_sel, const int32_t* rows,
                              int n_rows, const float* tilemap, const float* scores, float* kl_rows, float* kl_out,
                              cudaStream_t s) {
  MapParams prm;
  prm.mode = 0;
  prm.n_split = 1;
  prm.ws = nullptr;
  prm.rowmax = nullptr;
  prm.scale_log2 = 0.f;
  prm.n_rows = n_rows;
  prm.rows = rows;
  prm.tilemap = const_cast<float*>(tilemap);
  prm.lse = nullptr;
  for (int i = 0; i < VEDA_MAX_HEADS; ++i) prm.heads_sel[i] = i < n_heads_sel ? heads_sel[i] : 0;
  const int warps = n_heads_sel * n_rows;
  kl_rows_kernel<<<(warps * 32 + 255) / 256, 256, 0, s>>>(g, prm, n_heads_sel, scores, kl_rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kl_mean_kernel<<<1, 1024, 0, s>>>(kl_rows, n_heads_sel, n_rows, kl_out);
  return cudaGetLastError();
}

}  // namespace veda
