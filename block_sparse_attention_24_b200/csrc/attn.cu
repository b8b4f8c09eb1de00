// Tile-skipping sparse attention on sm_100a (Veda summary 2.3, Hardware-
// Efficient Implementation) for 64-token tiles: one CTA per pair of query
// tiles (a 128-row query block), walking the union of the two tiles' kept
// key-tile lists two tiles at a time; tiles neither kept are never loaded.
// 128-token tiles go to the two-tile kernel in attn_pair.cu.
//
// A 128 x 128 S block covers query tiles a0 (rows 0-63) and a1 (rows 64-127)
// against two union tiles u0 (keys 0-63) and u1 (keys 64-127). Each of the
// four 64 x 64 quarters is used when its query tile kept its key tile, and
// its P is zero otherwise. Neighbouring query tiles keep mostly the same key
// tiles, so the union is much shorter than the two lists together and most
// quarters are used: with one key tile per query tile per block (the other
// layout) only the two diagonal quarters would be.
//
// Roles (224 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r. Reads its
//              query tile's kept halves of a row of S from TMEM, keeps the row
//              reference and sum in fp32, writes P (bf16 pairs, zero in the
//              halves its query tile did not keep) back into the first half of
//              the same TMEM columns, rescales O in TMEM on the rare block
//              whose P sum nears the fp32 range, and finally normalises O and
//              stores it.
//   warp 4     K producer: TMA loads of Q once and of each step's two union
//              K tiles into a 3-stage ring (128B-swizzled).
//   warp 5     MMA issuer (one thread): S = Q K^T (A, B from shared memory)
//              into one of NS = 3 TMEM buffers; O += P V with P read from TMEM
//              and V from shared memory; tcgen05.commit to mbarriers.
//   warp 6     V producer: TMA loads of each step's two union V tiles.
// Per step j the MMA warp queues PV_j and then S_{j+3} as soon as P_j is in
// TMEM, so the tensor core works on them while softmax j+1 runs, and the
// next steps' S are already computed when their softmax starts.
//
// The union is walked over kept-tile bitmaps in shared memory when both lists
// are ascending, distinct and in range (and the bitmaps fit beside the
// rings), else by merging the lists as given; an odd union's last step loads
// its one tile into both halves, the second kept by neither query tile.
//
// Every mbarrier wait is bounded (VEDA_WAIT_LIMIT_NS); on expiry the CTA
// records VEDA_ERR_TIMEOUT, drains the copies and MMAs it issued, frees its
// TMEM and exits.
#include <type_traits>

#include "veda_internal.cuh"
#include "walk.cuh"

namespace veda {
namespace {

constexpr int BM = 128;               // query rows per CTA
constexpr int BN = 128;               // keys per block
constexpr int KST = 3, VST = 3;       // K and V ring stages
constexpr float OVERFLOW_SUM = 1.8446744e19f;  // 2^64: a block's P sum above this moves the reference
constexpr int NS = 3;                 // S buffers in TMEM: the MMA runs NS steps ahead of the softmax
constexpr uint32_t TMEM_COLS = 512;   // S_0 .. S_{NS-1} at [128 s, 128 s + 128), then O [128 NS, 128 NS + D)
constexpr int NUM_THREADS = 224;

template <int D>
struct AttnLayout {
  static constexpr int QB = BM * D * 2;       // Q block bytes (D/64 boxes of 16 KB)
  static constexpr int KB = BN * D * 2;       // K or V block bytes
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QB;
  static constexpr int OFF_V = OFF_K + KST * KB;
  static constexpr int OFF_BAR = OFF_V + VST * KB;
  // q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[NS], p_full[NS], pv_done[NS], drain
  static constexpr int NUM_BARS = 1 + 2 * KST + 2 * VST + 3 * NS + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag, list check
  static constexpr int OFF_BM = (OFF_MISC + 16 + 15) / 16 * 16;  // kept-tile bitmaps of a0 and a1
  // dynamic shared memory with bitmaps of `words` 32-bit words each
  static constexpr int alloc(int words) { return OFF_BM + 8 * words + 1024; }  // + 1024-byte alignment slack
};

struct AttnParams {
  int32_t k_cap;
  int32_t bm_words;  // 32-bit words per kept-tile bitmap; 0: merge the lists
  float scale_log2;  // scale * log2(e)
  const int32_t* idx;
  __nv_bfloat16* op;    // [B, heads, n_cap, D] (permuted order), or NULL when otok is set
  __nv_bfloat16* otok;  // [B, N, heads, D] (token order) or NULL: rows written straight to their tokens
  float* lse;
};

// Two consecutive union tiles per step. keep bit (2*s + h): query tile s of
// the block kept the step's tile h. An odd union's last step repeats its one
// tile in half 1, kept by neither (its loaded values meet only zeros in P).
template <class W>
struct StepWalk {
  W w;
  __device__ bool next(int& t0, int& t1, uint32_t& keep) {
    int t;
    bool ma, mb;
    if (!w.next(t, ma, mb)) return false;
    t0 = t;
    keep = (ma ? 1u : 0u) | (mb ? 4u : 0u);
    if (w.next(t, ma, mb)) {
      t1 = t;
      keep |= (ma ? 2u : 0u) | (mb ? 8u : 0u);
    } else {
      t1 = t0;
    }
    return true;
  }
};
template <class W>
__device__ __forceinline__ StepWalk<W> steps_of(const W& w) {
  return StepWalk<W>{w};
}

// Maximum of one 64-key half of a row of S over its first `klen` keys.
template <bool FULL>
__device__ __forceinline__ float half_row_max(const uint32_t (&u)[64], int klen) {
  float pm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v0 = (FULL || c + i < klen) ? __uint_as_float(u[c + i]) : -INFINITY;
      const float v1 = (FULL || c + 8 + i < klen) ? __uint_as_float(u[c + 8 + i]) : -INFINITY;
      pm[i] = fmax3(pm[i], v0, v1);
    }
  return fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
}

// P = 2^(s*C - m) for one 64-key half as 32 bf16 pairs into pk[32h..32h+32)
// (MUFU ex2), keys at or past `klen` zero; adds the fp32 values to acc.
template <bool FULL>
__device__ __forceinline__ void half_row_p(const uint32_t (&u)[64], int h, int klen, uint64_t C2, uint64_t NM,
                                           uint64_t (&acc)[4], uint32_t (&pk)[64]) {
#pragma unroll
  for (int w = 0; w < 32; ++w) {
    const uint64_t x = f2_fma(f2(__uint_as_float(u[2 * w]), __uint_as_float(u[2 * w + 1])), C2, NM);
    float x0, x1;
    f2_split(x, x0, x1);
    float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
    if (!FULL) {
      p0 = 2 * w < klen ? p0 : 0.f;
      p1 = 2 * w + 1 < klen ? p1 : 0.f;
    }
    acc[w & 3] = f2_add(acc[w & 3], f2(p0, p1));
    pk[32 * h + w] = pack_bf16x2_rn(p0, p1);
  }
}

// Tensor maps of the permuted layout [B*heads, n_cap, d] (Q boxes of 128
// rows, K/V boxes of one tile).
struct PermMaps {
  CUtensorMap q, k, v;
};

// TOK: Q, K, V in token order through the per-tiling 5D maps (TokenMaps).
template <int D, int TILE, bool TOK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ LayerGeom g,
                       const __grid_constant__ std::conditional_t<TOK, TokenMaps, PermMaps> maps,
                       const AttnParams prm) {
  static_assert(TILE == 64, "the union walk pairs two 64-token tiles per 128-key block");
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

  if (qb >= n_qb) {  // padding rows of this head: zero output (none in token order)
    for (int i = threadIdx.x; prm.op && i < BM * D / 8; i += NUM_THREADS) {
      const int r = i / (D / 8);
      if (qb * BM + r < g.n_cap)
        reinterpret_cast<uint4*>(prm.op + (row0 + r) * D)[i % (D / 8)] = make_uint4(0, 0, 0, 0);
    }
    if (prm.lse)
      for (int r = threadIdx.x; r < BM; r += NUM_THREADS)
        if (qb * BM + r < g.n_cap) prm.lse[row0 + r] = 0.f;
    return;
  }

  uint8_t* sQ = smem + Lay::OFF_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;  // [NS]
  uint64_t* p_full = s_full + NS;    // [NS], 128 arrivals
  uint64_t* pv_done = p_full + NS;   // [NS]
  uint64_t* mma_drain = pv_done + NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);
  volatile int* list_bad = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 8);
  uint32_t* bm0 = reinterpret_cast<uint32_t*>(smem + Lay::OFF_BM);
  uint32_t* bm1 = bm0 + prm.bm_words;

  // the block's query tiles a0 = 2 qb and a1 = 2 qb + 1 (a1 may be past the
  // head's last tile: then it keeps nothing)
  const int a0 = qb * NSUB, a1 = a0 + 1;
  const bool has1 = a1 < nt;
  const int n = hg.k;
  const int k0 = n, k1 = has1 ? n : 0;
  const int32_t* list0 = prm.idx ? prm.idx + ((long long)bh * g.nt_cap + a0) * prm.k_cap : nullptr;
  const int32_t* list1 = prm.idx ? prm.idx + ((long long)bh * g.nt_cap + (has1 ? a1 : a0)) * prm.k_cap : nullptr;
  const bool try_bm = prm.idx != nullptr && prm.bm_words > 0;  // uniform over the CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < Lay::NUM_BARS; ++i) {
      uint64_t* bar = bars + i;
      mbar_init(bar, (bar >= p_full && bar < p_full + NS) ? 128 : 1);
    }
    *abort_flag = 0;
    *list_bad = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (try_bm) {
    for (int i = threadIdx.x; i < 2 * prm.bm_words; i += NUM_THREADS) bm0[i] = 0u;
    __syncthreads();
    build_kept_bitmaps(list0, k0, list1, k1, nt, bm0, bm1, list_bad, threadIdx.x, NUM_THREADS);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool use_bm = try_bm && *list_bad == 0;
  // runs fn on the step walk of this CTA's union (one walk type instantiated
  // per call site, so only one walk's state is live)
  auto with_steps = [&](int32_t* status, auto&& fn) {
    if (use_bm) {
      auto sw = steps_of(BitWalk(bm0, bm1, prm.bm_words));
      fn(sw);
    } else {
      auto sw = steps_of(UnionWalk(list0, k0, list1, k1, nt, status));
      fn(sw);
    }
  };

  if (warp == 4 || warp == 6) {
    // ----------------------------------------------------------- producers
    if (lane == 0) {
      const bool is_k = warp == 4;
      const CUtensorMap* map;
      const CUtensorMap* qmap;
      if constexpr (TOK) {
        map = is_k ? &maps.k[hg.tmap] : &maps.v[hg.tmap];
        qmap = &maps.q[hg.tmap];
      } else {
        map = is_k ? &maps.k : &maps.v;
        qmap = &maps.q;
      }
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      uint8_t* ring = smem + (is_k ? Lay::OFF_K : Lay::OFF_V);
      const int ST = is_k ? KST : VST;  // this producer's ring depth
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(qmap);
        mbar_expect_tx(q_full, Lay::QB);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          if constexpr (TOK) {
#pragma unroll
            for (int u = 0; u < NSUB; ++u)  // the block's query tiles, one box each
              tma_load_tile_tokens(sQ + bx * BM * 128 + u * TILE * 128, qmap, q_full, g, hg, bx * 64, h, b,
                                   qb * NSUB + u);
          } else {
            tma_load_3d(sQ + bx * BM * 128, qmap, q_full, bx * 64, qb * BM, bh);
          }
        }
      }
      int issued = 0;
      with_steps(is_k ? g.dev_status : nullptr, [&](auto& sw) {
        int kt[2];
        uint32_t keep;
        for (int t = 0; sw.next(kt[0], kt[1], keep); ++t) {
          const int st = t % ST;
          if (t >= ST && !mbar_wait(empty + st, ((t - ST) / ST) & 1, abort_flag, g.dev_status)) break;
          mbar_expect_tx(full + st, Lay::KB);
          uint8_t* dst = ring + st * Lay::KB;
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int bx = 0; bx < D / 64; ++bx)
              if constexpr (TOK)
                tma_load_tile_tokens(dst + bx * BN * 128 + u * TILE * 128, map, full + st, g, hg, bx * 64, h, b,
                                     kt[u]);
              else
                tma_load_3d(dst + bx * BN * 128 + u * TILE * 128, map, full + st, bx * 64, kt[u] * TILE, bh);
          issued = t + 1;
        }
      });
      if (*abort_flag) {  // let every copy this warp started land before exiting
        if (is_k) mbar_wait_drain(q_full, 0, VEDA_WAIT_LIMIT_NS);
        for (int t = issued - ST < 0 ? 0 : issued - ST; t < issued; ++t)
          mbar_wait_drain(full + t % ST, (t / ST) & 1, VEDA_WAIT_LIMIT_NS);
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
      // the number of steps of the walk
      int n_steps = 0;
      with_steps(nullptr, [&](auto& sw) {
        int t0, t1;
        uint32_t keep;
        while (sw.next(t0, t1, keep)) ++n_steps;
      });
      auto issue_s = [&](int t) -> bool {
        const int s = t % NS, st = t % KST;
        if (!mbar_wait(k_full + st, (t / KST) & 1, abort_flag, g.dev_status)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_bf16_ss(tmem + s * BN, sdesc_sw128(aQ + off, 16, 1024),
                       sdesc_sw128(aK + st * Lay::KB + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(s_full + s);
        umma_commit(k_empty + st);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, g.dev_status);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < NS && t < n_steps && ok; ++t) ok = issue_s(t);
        for (int j = 0; j < n_steps && ok; ++j) {
          const int s = j % NS, sv = j % VST;
          if (!mbar_wait(p_full + s, (j / NS) & 1, abort_flag, g.dev_status)) break;
          if (!mbar_wait(v_full + sv, (j / VST) & 1, abort_flag, g.dev_status)) break;
          tc_fence_after();
          // P_j sits in the first 64 columns of S buffer s (two bf16 per column)
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_bf16_ts(tmem + NS * BN, tmem + s * BN + kk * 8,
                         sdesc_sw128(aV + sv * Lay::KB + kk * 2048, BN * 128, 1024), idesc_o,
                         (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(pv_done + s);
          umma_commit(v_empty + sv);
          if (j + NS < n_steps) ok = issue_s(j + NS);  // overwrites S buffer s after PV_j has read P_j
        }
      }
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0, VEDA_WAIT_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = threadIdx.x;                 // query row in the block
    const int sub = r / TILE;                  // the block's query tile (0 or 1)
    const int a = qb * NSUB + sub;             // query tile
    const bool row_valid = a < nt && (r % TILE) < tile_len(hg, g.T, a);
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const float C = prm.scale_log2;
    const uint64_t C2 = f2(C, C);
    const bool padded = hg.padded != 0;
    float m = -INFINITY, l = 0.f;
    bool have_ref = false;  // the row's reference m is set (its first kept tile seen)
    bool ok = true;
    int n_steps = 0;
    with_steps(nullptr, [&](auto& sw) {
      int kt[2];
      uint32_t keep;
      for (int j = 0; sw.next(kt[0], kt[1], keep); ++j) {
        n_steps = j + 1;
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        // this query tile's kept halves (uniform over the warp: a warp's rows
        // belong to one query tile)
        const bool kh0 = (keep >> (2 * sub)) & 1u, kh1 = (keep >> (2 * sub + 1)) & 1u;
        const int klen0 = padded ? tile_len(hg, g.T, kt[0]) : TILE;
        const int klen1 = padded ? tile_len(hg, g.T, kt[1]) : TILE;
        if (!__all_sync(0xffffffffu, mbar_wait(s_full + s, ph, abort_flag, g.dev_status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t pk[64];
        // exact maximum of the kept halves' valid keys
        auto kept_max = [&]() -> float {
          float mx = -INFINITY;
          if (kh0) {
            uint32_t u[64];
            tmem_ld64(lane_addr + s * BN, u);
            mx = klen0 >= TILE ? half_row_max<true>(u, klen0) : half_row_max<false>(u, klen0);
          }
          if (kh1) {
            uint32_t u[64];
            tmem_ld64(lane_addr + s * BN + TILE, u);
            mx = fmaxf(mx, klen1 >= TILE ? half_row_max<true>(u, klen1) : half_row_max<false>(u, klen1));
          }
          return mx;
        };
        // P of the kept halves against reference mref (zeros elsewhere);
        // returns the fp32 row sum
        auto make_p = [&](float mref) -> float {
          const uint64_t NM = f2(-mref, -mref);
          uint64_t acc[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[e] = f2(0.f, 0.f);
          if (kh0 && kh1) {  // both halves: one TMEM load of the whole row
            uint32_t u[BN];
            tmem_ld128(lane_addr + s * BN, u);
            const uint32_t (&u0)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&u[0]);
            const uint32_t (&u1)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&u[64]);
            if (klen0 >= TILE) half_row_p<true>(u0, 0, klen0, C2, NM, acc, pk);
            else half_row_p<false>(u0, 0, klen0, C2, NM, acc, pk);
            if (klen1 >= TILE) half_row_p<true>(u1, 1, klen1, C2, NM, acc, pk);
            else half_row_p<false>(u1, 1, klen1, C2, NM, acc, pk);
          } else if (kh0) {
            uint32_t u[64];
            tmem_ld64(lane_addr + s * BN, u);
            if (klen0 >= TILE) half_row_p<true>(u, 0, klen0, C2, NM, acc, pk);
            else half_row_p<false>(u, 0, klen0, C2, NM, acc, pk);
#pragma unroll
            for (int w = 0; w < 32; ++w) pk[32 + w] = 0u;
          } else {
            uint32_t u[64];
            tmem_ld64(lane_addr + s * BN + TILE, u);
            if (klen1 >= TILE) half_row_p<true>(u, 1, klen1, C2, NM, acc, pk);
            else half_row_p<false>(u, 1, klen1, C2, NM, acc, pk);
#pragma unroll
            for (int w = 0; w < 32; ++w) pk[w] = 0u;
          }
          float lo, hi;
          f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lo, hi);
          return lo + hi;
        };
        float rs = 0.f;
        if (kh0 || kh1) {
          // Only the row's first kept tile is max-reduced. Later tiles reuse
          // its reference: P may exceed 1 when they hold larger logits, which
          // fp32 and bf16 carry at full relative precision, so the reference
          // moves only when a step's P sum nears the top of the range (rare);
          // S_j is still in TMEM then (P is stored below), so the step is
          // recomputed exactly.
          if (!have_ref) {
            m = kept_max() * C;
            have_ref = true;
          }
          rs = make_p(m);
        } else {
#pragma unroll
          for (int w = 0; w < 64; ++w) pk[w] = 0u;
        }
        const bool redo = !(rs <= OVERFLOW_SUM);
        if (__any_sync(0xffffffffu, redo)) {
          const float mx2 = kept_max() * C;  // TMEM loads: the whole warp takes them
          const float m_new = redo ? fmaxf(m, mx2) : m;
          const float alpha = fast_exp2(m - m_new);
          if (j > 0) {
            // O must hold PV_{j-1} before it is rescaled
            if (!__all_sync(0xffffffffu, mbar_wait(pv_done + (j - 1) % NS, ((j - 1) / NS) & 1, abort_flag,
                                                   g.dev_status))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t u[32];
              tmem_ld32(lane_addr + NS * BN + c * 32, u);
#pragma unroll
              for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
              tmem_st32(lane_addr + NS * BN + c * 32, u);
            }
          }
          l *= alpha;
          m = m_new;
          if (kh0 || kh1) rs = make_p(m);
        }
        l += rs;
        tmem_st64(lane_addr + s * BN, pk);  // P_j over the first half of S_j
        tc_fence_before();
        mbar_arrive(p_full + s);
      }
    });
    // epilogue: O / l -> bf16
    if (ok && n_steps > 0 &&
        __all_sync(0xffffffffu, mbar_wait(pv_done + (n_steps - 1) % NS, ((n_steps - 1) / NS) & 1, abort_flag,
                                          g.dev_status))) {
      tc_fence_after();
      const float inv = row_valid && l > 0.f ? 1.0f / l : 0.f;
      const bool in_range = qb * BM + r < g.n_cap;
      // the row's destination: its permuted slot, or its token (padding rows
      // have none)
      __nv_bfloat16* orow = nullptr;
      if (prm.otok) {
        const long long tok = row_valid ? tile_row_token(g, hg, a, r % TILE) : -1;
        if (tok >= 0) orow = prm.otok + (((long long)b * g.T * g.H * g.W + tok) * g.heads + h) * D;
      } else if (in_range) {
        orow = prm.op + (row0 + r) * D;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_addr + NS * BN + c * 32, u);
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          o[e] = pack_bf16x2_rn(__uint_as_float(u[2 * e]) * inv, __uint_as_float(u[2 * e + 1]) * inv);
        if (orow) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
      }
      if (prm.lse && in_range)
        prm.lse[row0 + r] = row_valid && l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D, int TILE, bool TOK>
cudaError_t launch_t(const LayerGeom& g0, const void* qp, const void* kp, const void* vp, const AttnParams& prm0,
                     cudaStream_t s) {
  LayerGeom g = g0;
  std::conditional_t<TOK, TokenMaps, PermMaps> maps;
  if constexpr (TOK) {
    const cudaError_t e = build_token_maps(g, qp, kp, vp, &maps);
    if (e != cudaSuccess) return e;
  } else {
    const uint64_t rows = (uint64_t)g.n_cap, planes = (uint64_t)g.B * g.heads;
    if (encode_tensor_map_3d_bf16(&maps.q, qp, D, rows, planes, 64, BM) != CUDA_SUCCESS ||
        encode_tensor_map_3d_bf16(&maps.k, kp, D, rows, planes, 64, TILE) != CUDA_SUCCESS ||
        encode_tensor_map_3d_bf16(&maps.v, vp, D, rows, planes, 64, TILE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = sparse_attn_kernel<D, TILE, TOK>;
  AttnParams prm = prm0;
  prm.bm_words = (g.nt_cap + 31) / 32;
  int smem = AttnLayout<D>::alloc(prm.bm_words);
  if (smem > 232448) {  // bitmaps do not fit beside the rings: merge the lists
    prm.bm_words = 0;
    smem = AttnLayout<D>::alloc(0);
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int qblocks = (g.nt_cap * TILE + BM - 1) / BM;
  const dim3 grid(qblocks, g.heads, g.B);
  kern<<<grid, NUM_THREADS, smem, s>>>(g, maps, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn_pair(const LayerGeom& g, const void* qp, const void* kp, const void* vp,
                                    const int32_t* idx, int k_cap, float scale, void* op, float* lse,
                                    cudaStream_t s, void* o_tokens, bool tokens_in);

cudaError_t launch_sparse_attn(const LayerGeom& g, const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, int k_cap, float scale, void* op, float* lse, cudaStream_t s,
                               void* o_tokens, bool tokens_in) {
  AttnParams prm;
  prm.k_cap = k_cap;
  prm.bm_words = 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.idx = idx;
  prm.op = o_tokens ? nullptr : reinterpret_cast<__nv_bfloat16*>(op);
  prm.otok = reinterpret_cast<__nv_bfloat16*>(o_tokens);
  prm.lse = lse;
  if (g.tile == 128) return launch_sparse_attn_pair(g, qp, kp, vp, idx, k_cap, scale, op, lse, s, o_tokens, tokens_in);
  if (tokens_in) {
    if (!o_tokens) return cudaErrorInvalidValue;
    if (g.d == 128) return launch_t<128, 64, true>(g, qp, kp, vp, prm, s);
    return launch_t<64, 64, true>(g, qp, kp, vp, prm, s);
  }
  if (g.d == 128) return launch_t<128, 64, false>(g, qp, kp, vp, prm, s);
  return launch_t<64, 64, false>(g, qp, kp, vp, prm, s);
}

}  // namespace veda
