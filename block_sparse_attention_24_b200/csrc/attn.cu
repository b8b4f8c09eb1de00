// Tile-skipping sparse attention on sm_100a (Veda summary 2.3, Hardware-
// Efficient Implementation): each CTA owns 128 query rows of one head and
// walks only the key/value tiles its query tiles kept; skipped tiles are
// never loaded.
//
// Roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r. Reads S from
//              TMEM, keeps the running max / sum in fp32, writes P (bf16) to
//              shared memory, rescales O in TMEM when the max grows by more
//              than 2^8, and finally normalises O and stores it.
//   warp 4     producer: TMA loads of Q once and of the selected K and V tiles
//              into two-stage rings (128B-swizzled).
//   warp 5     MMA issuer (one thread): S = Q K^T into one of two TMEM
//              buffers, O += P V into a TMEM accumulator, tcgen05.commit to
//              mbarriers.
// Pipeline per key block j: S_j is computed while softmax j-1 runs, PV_j and
// S_{j+2} are queued as soon as P_j is written.
//
// Tiles of 64 tokens: a CTA still computes 128x128 blocks; its two 64-row
// query tiles each pair with their own 64-key tile, so only the two diagonal
// 64x64 blocks of S are used (the others are masked to zero in P).
//
// Every mbarrier wait is bounded (VEDA_WAIT_LIMIT_NS); on expiry the CTA
// records VEDA_ERR_TIMEOUT, drains the copies and MMAs it issued, frees its
// TMEM and exits.
#include "veda_internal.cuh"

namespace veda {
namespace {

constexpr int BM = 128;               // query rows per CTA
constexpr int BN = 128;               // keys per block
constexpr float RESCALE_LOG2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_THREADS = 192;

template <int D>
struct AttnLayout {
  static constexpr int QB = BM * D * 2;       // Q block bytes (D/64 boxes of 16 KB)
  static constexpr int KB = BN * D * 2;       // K or V block bytes
  static constexpr int PB = BM * BN * 2;      // P block bytes (2 boxes of 16 KB)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QB;
  static constexpr int OFF_V = OFF_K + 2 * KB;
  static constexpr int OFF_P = OFF_V + 2 * KB;
  static constexpr int OFF_BAR = OFF_P + 2 * PB;
  static constexpr int NUM_BARS = 16;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
};

struct AttnParams {
  int32_t k_cap;
  float scale_log2;  // scale * log2(e)
  const int32_t* idx;
  __nv_bfloat16* op;
  float* lse;
};

// Tile index of query sub-tile `sub` at key block `j` (clamped into range;
// an out-of-range entry is reported once).
__device__ __forceinline__ int key_tile(const int32_t* row, int j, int nt, int32_t* status) {
  if (!row) return j;
  int t = __ldg(row + j);
  if (t < 0 || t >= nt) {
    report(status, VEDA_ERR_BAD_INDEX);
    t = 0;
  }
  return t;
}

template <int D, int TILE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ LayerGeom g, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const AttnParams prm) {
  using Lay = AttnLayout<D>;
  constexpr int NSUB = BM / TILE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * g.heads + h;
  const HeadGeom& hg = g.h[h];
  const int nt = hg.nt;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qb = (nt + NSUB - 1) / NSUB;
  const long long row0 = (long long)bh * g.n_cap + (long long)qb * BM;  // first output row

  if (qb >= n_qb) {  // padding rows of this head: zero output
    for (int i = threadIdx.x; i < BM * D / 8; i += NUM_THREADS) {
      const int r = i / (D / 8);
      if (qb * BM + r < g.n_cap) reinterpret_cast<uint4*>(prm.op + (row0 + r) * D)[i % (D / 8)] = make_uint4(0, 0, 0, 0);
    }
    if (prm.lse)
      for (int r = threadIdx.x; r < BM; r += NUM_THREADS)
        if (qb * BM + r < g.n_cap) prm.lse[row0 + r] = 0.f;
    return;
  }

  uint8_t* sQ = smem + Lay::OFF_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* p_full = bars + 11;  // [2]
  uint64_t* pv_done = bars + 13; // [2]
  uint64_t* mma_drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);

  const int n = hg.k;  // key blocks (kept tiles per query tile)
  const int32_t* lists[NSUB];
#pragma unroll
  for (int s = 0; s < NSUB; ++s) {
    int a = qb * NSUB + s;
    if (a >= nt) a = qb * NSUB;  // missing second query tile: reuse the first list
    lists[s] = prm.idx ? prm.idx + ((long long)bh * g.nt_cap + a) * prm.k_cap : nullptr;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < Lay::NUM_BARS; ++i) mbar_init(bars + i, (i == 11 || i == 12) ? 128 : 1);  // p_full: 128
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(q_full, Lay::QB);
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) tma_load_3d(sQ + bx * BM * 128, &tmQ, q_full, bx * 64, qb * BM, bh);
      int kt_issued = 0, vt_issued = 0;
      for (int t = 0; t < n; ++t) {
        const int s = t & 1;
        int kts[NSUB];
#pragma unroll
        for (int u = 0; u < NSUB; ++u) kts[u] = key_tile(lists[u], t, nt, g.dev_status);
        if (t >= 2 && !mbar_wait(k_empty + s, ((t - 2) >> 1) & 1, abort_flag, g.dev_status)) break;
        mbar_expect_tx(k_full + s, Lay::KB);
        uint8_t* dK = smem + Lay::OFF_K + s * Lay::KB;
#pragma unroll
        for (int u = 0; u < NSUB; ++u)
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_3d(dK + bx * BN * 128 + u * TILE * 128, &tmK, k_full + s, bx * 64, kts[u] * TILE, bh);
        kt_issued = t + 1;
        if (t >= 2 && !mbar_wait(v_empty + s, ((t - 2) >> 1) & 1, abort_flag, g.dev_status)) break;
        mbar_expect_tx(v_full + s, Lay::KB);
        uint8_t* dV = smem + Lay::OFF_V + s * Lay::KB;
#pragma unroll
        for (int u = 0; u < NSUB; ++u)
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_3d(dV + bx * BN * 128 + u * TILE * 128, &tmV, v_full + s, bx * 64, kts[u] * TILE, bh);
        vt_issued = t + 1;
      }
      if (*abort_flag) {  // let every copy this CTA started land before exiting
        mbar_wait_drain(q_full, 0, VEDA_WAIT_LIMIT_NS);
        for (int t = kt_issued - 2 < 0 ? 0 : kt_issued - 2; t < kt_issued; ++t)
          mbar_wait_drain(k_full + (t & 1), (t >> 1) & 1, VEDA_WAIT_LIMIT_NS);
        for (int t = vt_issued - 2 < 0 ? 0 : vt_issued - 2; t < vt_issued; ++t)
          mbar_wait_drain(v_full + (t & 1), (t >> 1) & 1, VEDA_WAIT_LIMIT_NS);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(BM, D, false, true);
      const uint32_t aQ = smem_u32(sQ);
      const uint32_t aK = smem_u32(smem + Lay::OFF_K);
      const uint32_t aV = smem_u32(smem + Lay::OFF_V);
      const uint32_t aP = smem_u32(smem + Lay::OFF_P);
      auto issue_s = [&](int t) -> bool {
        const int s = t & 1;
        if (!mbar_wait(k_full + s, (t >> 1) & 1, abort_flag, g.dev_status)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_bf16_ss(tmem + s * BN, sdesc_sw128(aQ + off, 16, 1024),
                       sdesc_sw128(aK + s * Lay::KB + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(s_full + s);
        umma_commit(k_empty + s);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, g.dev_status);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2 && t < n && ok; ++t) ok = issue_s(t);
        for (int j = 0; j < n && ok; ++j) {
          const int s = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (!mbar_wait(p_full + s, ph, abort_flag, g.dev_status)) break;
          if (!mbar_wait(v_full + s, ph, abort_flag, g.dev_status)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t offp = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
            umma_bf16_ss(tmem + 2 * BN, sdesc_sw128(aP + s * Lay::PB + offp, 16, 1024),
                         sdesc_sw128(aV + s * Lay::KB + kk * 2048, BN * 128, 1024), idesc_o,
                         (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(pv_done + s);
          umma_commit(v_empty + s);
          if (j + 2 < n) ok = issue_s(j + 2);
        }
      }
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0, VEDA_WAIT_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = threadIdx.x;                 // query row in the block
    const int sub = r / TILE;                  // query sub-tile
    const int a = qb * NSUB + sub;             // query tile
    const int32_t* my_list = (NSUB == 1 || sub == 0) ? lists[0] : lists[NSUB - 1];
    const bool row_valid = a < nt && (r % TILE) < tile_len(hg, g.T, a);
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const float C = prm.scale_log2;
    uint8_t* sP = smem + Lay::OFF_P;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      const int kt = key_tile(my_list, j, nt, nullptr);
      const int klen = tile_len(hg, g.T, kt);
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + s, ph, abort_flag, g.dev_status))) { ok = false; break; }
      tc_fence_after();
      float sv[TILE];
#pragma unroll
      for (int c = 0; c < TILE / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_addr + s * BN + sub * TILE + c * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(u[e]);
      }
      float mx = -INFINITY;
      if (klen == TILE) {
#pragma unroll
        for (int c = 0; c < TILE; ++c) mx = fmaxf(mx, sv[c]);
      } else {
#pragma unroll
        for (int c = 0; c < TILE; ++c) mx = fmaxf(mx, c < klen ? sv[c] : -INFINITY);
      }
      const float mx2 = mx * C;
      if (j == 0) {
        m = mx2;
      } else {
        const bool need = mx2 > m + RESCALE_LOG2;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold PV_{j-1} before it is rescaled
          if (!__all_sync(0xffffffffu, mbar_wait(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, g.dev_status))) { ok = false; break; }
          tc_fence_after();
          const float alpha = need ? fast_exp2(m - mx2) : 1.0f;
          if (need) {
            l *= alpha;
            m = mx2;
          }
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld32(lane_addr + 2 * BN + c * 32, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(lane_addr + 2 * BN + c * 32, u);
          }
        }
      }
      // P buffer s is free once PV_{j-2} has completed
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(pv_done + s, ((j - 2) >> 1) & 1, abort_flag, g.dev_status))) { ok = false; break; }
      uint8_t* Pbuf = sP + s * Lay::PB;
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < TILE / 8; ++q) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = q * 8 + 2 * e;
          float p0 = fast_exp2(fmaf(sv[c0], C, -m));
          float p1 = fast_exp2(fmaf(sv[c0 + 1], C, -m));
          if (klen != TILE) {
            p0 = c0 < klen ? p0 : 0.f;
            p1 = c0 + 1 < klen ? p1 : 0.f;
          }
          rs += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        const int key_chunk = sub * (TILE / 8) + q;  // 8-key chunk within the 128-key block
        const int bx = key_chunk >> 3, qq = key_chunk & 7;
        *reinterpret_cast<uint4*>(Pbuf + bx * (BM * 128) + r * 128 + ((qq ^ (r & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      if (NSUB > 1) {  // the other query tile's keys: zero
#pragma unroll
        for (int q = 0; q < TILE / 8; ++q) {
          const int key_chunk = (1 - sub) * (TILE / 8) + q;
          const int bx = key_chunk >> 3, qq = key_chunk & 7;
          *reinterpret_cast<uint4*>(Pbuf + bx * (BM * 128) + r * 128 + ((qq ^ (r & 7)) << 4)) =
              make_uint4(0, 0, 0, 0);
        }
      }
      l += rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + s);
    }
    // epilogue: O / l -> bf16
    if (ok && n > 0 && __all_sync(0xffffffffu, mbar_wait(pv_done + ((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag, g.dev_status))) {
      tc_fence_after();
      const float inv = row_valid ? 1.0f / l : 0.f;
      const bool in_range = qb * BM + r < g.n_cap;
      __nv_bfloat16* orow = prm.op + (row0 + r) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_addr + 2 * BN + c * 32, u);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(u[2 * e]) * inv, __uint_as_float(u[2 * e + 1]) * inv);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (prm.lse && in_range) prm.lse[row0 + r] = row_valid ? (m + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D, int TILE>
cudaError_t launch_t(const LayerGeom& g, const void* qp, const void* kp, const void* vp, const AttnParams& prm,
                     cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)g.n_cap, planes = (uint64_t)g.B * g.heads;
  if (encode_tensor_map_3d_bf16(&tq, qp, D, rows, planes, 64, BM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&tk, kp, D, rows, planes, 64, TILE) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&tv, vp, D, rows, planes, 64, TILE) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = sparse_attn_kernel<D, TILE>;
  const int smem = AttnLayout<D>::SMEM_ALLOC;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int qblocks = (g.nt_cap * TILE + BM - 1) / BM;
  const dim3 grid(qblocks, g.heads, g.B);
  kern<<<grid, NUM_THREADS, smem, s>>>(g, tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn(const LayerGeom& g, const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, int k_cap, float scale, void* op, float* lse, cudaStream_t s) {
  AttnParams prm;
  prm.k_cap = k_cap;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.idx = idx;
  prm.op = reinterpret_cast<__nv_bfloat16*>(op);
  prm.lse = lse;
  if (g.d == 128 && g.tile == 128) return launch_t<128, 128>(g, qp, kp, vp, prm, s);
  if (g.d == 128 && g.tile == 64) return launch_t<128, 64>(g, qp, kp, vp, prm, s);
  if (g.d == 64 && g.tile == 128) return launch_t<64, 128>(g, qp, kp, vp, prm, s);
  return launch_t<64, 64>(g, qp, kp, vp, prm, s);
}

}  // namespace veda
