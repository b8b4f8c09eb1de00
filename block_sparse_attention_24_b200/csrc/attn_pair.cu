// Tile-skipping sparse attention for 128-token tiles, two query tiles per CTA
// (Veda summary 2.3, Hardware-Efficient Implementation: only the kept
// key/value tiles are loaded; here each loaded tile also serves both query
// tiles of the CTA when both kept it).
//
// A CTA owns two neighbouring query tiles A and B of one head (pair_stride:
// along time for heads with p_t <= 2 and an even number of time slabs, else
// consecutive). Every tile of the
// union of their kept lists is loaded by TMA exactly once, and S = Q K^T /
// O += P V are issued only for the query tile(s) that kept it. Neighbouring
// query tiles keep mostly the same key tiles (spatio-temporal locality), so
// the union is much shorter than the two lists together and each K/V byte
// from L2 feeds up to twice the tensor work of a one-tile CTA. The union is
// walked over kept-tile bitmaps built in shared memory (AltWalk), taking the
// tiles only A kept and the tiles only B kept alternately where a head has
// no padded tiles; lists that are not ascending and distinct are merged as
// given (UnionWalk).
//
// Roles (384 threads):
//   warps 0-3 / 4-7  softmax of query tile A / B: thread owns one row (TMEM
//                    lane). S_A in TMEM columns [0,128), S_B [128,256); P is
//                    written back as bf16 pairs over the second half of its
//                    S; O_A at [256, 256+D), O_B after it.
//   warp 8           K producer (Q_A, Q_B once; then the union's K tiles)
//   warp 9           MMA issuer (one thread)
//   warp 10          V producer (the union's V tiles)
//   warp 11          idle
// MMA order per union tile e: for each query tile that kept e: its P V of
// the previous union tile (if it kept that one), then S for e; then for a
// query tile that did not keep e, its pending P V. So one query tile's
// softmax runs while the tensor core works for the other. One commit per
// union tile to a ring of step barriers frees the K slot of that tile and the
// V slot of the one before.
//
// Q, K, V come either from the permuted layout [B, heads, n_cap, d] (3D
// tensor maps) or straight from token order [B, N, heads, d] (TOK: 5D maps,
// one per distinct tiling, whose box is a tile). The output goes to the
// permuted layout or to each row's token.
//
// Every mbarrier wait is bounded (VEDA_WAIT_LIMIT_NS); on expiry the CTA
// records VEDA_ERR_TIMEOUT, drains what it issued, frees its TMEM and exits.
#include <climits>
#include <type_traits>

#include "veda_internal.cuh"
#include "walk.cuh"

namespace veda {
namespace {

constexpr int BM = 128;               // rows per query tile
constexpr int BN = 128;               // keys per tile
constexpr int KST = 2, VST = 3;       // K and V ring stages
constexpr int SDR = 4;                // step-done barriers (ring over union positions)
constexpr float OVERFLOW_SUM = 1.8446744e19f;  // 2^64: a tile's P sum above this moves the reference
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_THREADS = 384;
// Registers per thread after the split: softmax warpgroups (2 x 128 threads)
// and the producer/MMA warpgroup (128 threads); 2*128*208 + 128*88 = 64,512
// = the 384*168 the launch reserves.
constexpr int REGS_SOFTMAX = 208, REGS_ROLES = 88;

template <int D>
struct PairLayout {
  static constexpr int QB = BM * D * 2;
  static constexpr int KB = BN * D * 2;
  static constexpr int OFF_Q = 0;  // Q_A, Q_B
  static constexpr int OFF_K = 2 * QB;
  static constexpr int OFF_V = OFF_K + KST * KB;
  static constexpr int OFF_BAR = OFF_V + VST * KB;
  // q_full, k_full[KST], v_full[VST], step_done[SDR], s_full[2], p_full[2], pv_done[2], drain
  static constexpr int NUM_BARS = 1 + KST + VST + SDR + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag, list check
  static constexpr int OFF_BM = (OFF_MISC + 16 + 15) / 16 * 16;  // kept-tile bitmaps of A and B
  // dynamic shared memory for bitmaps of `words` 32-bit words each
  static constexpr int alloc(int words) { return OFF_BM + 8 * words + 1024; }
};

// Which two query tiles share a CTA: tiles a and a + S. For a head whose
// tiles span at most two frames (p_t <= 2) neighbouring time slabs keep the
// most key tiles in common, so S is the tiles per time slab; otherwise S = 1
// (neighbours along W, or the next row). Measured on the benchmark layer's
// kept lists, this cut the mean union of a pair from 1.27k to 1.21k.
// Along time only when the time slabs pair up exactly: with an odd count the
// last slab's tps tiles would run alone, where consecutive pairing leaves at
// most one tile alone.
__host__ __device__ inline int pair_stride(const HeadGeom& hg) {
  return hg.pt <= 2 && (hg.nt / hg.tps) % 2 == 0 ? hg.tps : 1;
}

// CTAs of a head: ceil(n/2)*S pairs (n = nt/S tiles along the paired axis),
// then one CTA per two padding tiles in [nt, nt_cap).
__host__ __device__ inline int pair_ctas(const HeadGeom& hg, int nt_cap) {
  const int S = pair_stride(hg), n = hg.nt / S;
  return (n + 1) / 2 * S + (nt_cap - hg.nt + 1) / 2;
}

struct PairParams {
  int32_t k_cap;
  int32_t bm_words;  // 32-bit words per kept-tile bitmap in shared memory; 0: no bitmaps
  float scale_log2;
  const int32_t* idx;
  __nv_bfloat16* op;    // [B, heads, n_cap, D] (permuted order), or NULL when otok is set
  __nv_bfloat16* otok;  // [B, N, heads, D] (token order) or NULL: rows written straight to their tokens
  float* lse;
};

// A third order over the same bitmaps, for heads whose tiles are all full
// (then the softmax never needs to know which tile it holds, and each query
// tile may take its kept tiles in any order). A union tile only one query
// tile kept runs that query tile's chain alone: the next S can only follow
// its own softmax and P V. So tiles only A kept and tiles only B kept are
// taken alternately while both remain, letting each chain's latency hide
// behind the other's work; otherwise the lowest remaining tile comes next.
// Tiles both kept are steps of their own, as in the other walks.
struct AltWalk {
  struct Cursor {  // lowest remaining tile of one category (A only, B only, both)
    int wi;
    uint32_t w;
  };
  const uint32_t* a;
  const uint32_t* b;
  int nw;
  Cursor ca, cb, cs;
  int last;  // 1: the previous step was a tile only A kept, 2: only B, 0: otherwise
  __device__ uint32_t word(int c, int wi) const {
    const uint32_t x = a[wi], y = b[wi];
    return c == 0 ? (x & ~y) : (c == 1 ? (y & ~x) : (x & y));
  }
  __device__ void init(Cursor& cu, int c) {
    cu.wi = 0;
    cu.w = nw > 0 ? word(c, 0) : 0u;
  }
  // tile index of the lowest remaining bit, INT_MAX when none is left
  __device__ int head(Cursor& cu, int c) {
    while (cu.w == 0u) {
      if (cu.wi + 1 >= nw) return INT_MAX;
      ++cu.wi;
      cu.w = word(c, cu.wi);
    }
    return cu.wi * 32 + __ffs(cu.w) - 1;
  }
  __device__ AltWalk(const uint32_t* a_, const uint32_t* b_, int nw_) : a(a_), b(b_), nw(nw_), last(0) {
    init(ca, 0);
    init(cb, 1);
    init(cs, 2);
  }
  __device__ bool next(int& t, bool& ma, bool& mb) {
    const int ha = head(ca, 0), hb = head(cb, 1), hs = head(cs, 2);
    int c;
    if (last == 1 && hb != INT_MAX) c = 1;
    else if (last == 2 && ha != INT_MAX) c = 0;
    else if (ha == INT_MAX && hb == INT_MAX && hs == INT_MAX) return false;
    else c = (ha < hb && ha < hs) ? 0 : (hb < hs ? 1 : 2);
    // consume the lowest bit of the chosen category (explicit branches keep
    // the cursors in registers)
    if (c == 0) {
      t = ha;
      ca.w &= ca.w - 1u;
    } else if (c == 1) {
      t = hb;
      cb.w &= cb.w - 1u;
    } else {
      t = hs;
      cs.w &= cs.w - 1u;
    }
    ma = c != 1;
    mb = c != 0;
    last = c == 0 ? 1 : (c == 1 ? 2 : 0);
    return true;
  }
};

// Maximum of one 64-key half h of a row of S over the valid keys (all of
// them unless !FULL, then keys below `klen`): eight 3-input max chains.
template <bool FULL>
__device__ __forceinline__ float half_max(const uint32_t (&u)[64], int h, int klen) {
  float pm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k0 = 64 * h + c + i, k1 = k0 + 8;
      const float v0 = (FULL || k0 < klen) ? __uint_as_float(u[c + i]) : -INFINITY;
      const float v1 = (FULL || k1 < klen) ? __uint_as_float(u[c + 8 + i]) : -INFINITY;
      pm[i] = fmax3(pm[i], v0, v1);
    }
  return fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
}

// P = 2^(s*C - m) for one 64-key half h of the row as 32 bf16 pairs (MUFU
// ex2), with four packed partial row sums. Keys at or past `klen` get P = 0
// unless FULL.
template <bool FULL>
__device__ __forceinline__ void half_p(const uint32_t (&u)[64], int h, int klen, uint64_t C2, uint64_t NM,
                                       uint64_t (&acc)[4], uint32_t (&pk)[32]) {
#pragma unroll
  for (int w = 0; w < 32; ++w) {
    const int k0 = 64 * h + 2 * w;
    const uint64_t x = f2_fma(f2(__uint_as_float(u[2 * w]), __uint_as_float(u[2 * w + 1])), C2, NM);
    float x0, x1;
    f2_split(x, x0, x1);
    float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
    if (!FULL) {
      p0 = k0 < klen ? p0 : 0.f;
      p1 = k0 + 1 < klen ? p1 : 0.f;
    }
    acc[w & 3] = f2_add(acc[w & 3], f2(p0, p1));
    pk[w] = pack_bf16x2_rn(p0, p1);
  }
}

// Maximum of a row of S over its valid keys.
template <bool FULL>
__device__ __forceinline__ float row_max(const uint32_t (&u)[BN], int klen) {
  const uint32_t (&u0)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&u[0]);
  const uint32_t (&u1)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&u[64]);
  return fmaxf(half_max<FULL>(u0, 0, klen), half_max<FULL>(u1, 1, klen));
}

// P = 2^(s*C - m) for a whole row as bf16 pairs (keys [0,64) in pk0, [64,128)
// in pk1); returns the row sum of the fp32 values.
template <bool FULL>
__device__ __forceinline__ float row_p(const uint32_t (&u)[BN], int klen, uint64_t C2, float m, uint32_t (&pk0)[32],
                                       uint32_t (&pk1)[32]) {
  const uint32_t (&u0)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&u[0]);
  const uint32_t (&u1)[64] = *reinterpret_cast<const uint32_t(*)[64]>(&u[64]);
  const uint64_t NM = f2(-m, -m);
  uint64_t acc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = f2(0.f, 0.f);
  half_p<FULL>(u0, 0, klen, C2, NM, acc, pk0);
  half_p<FULL>(u1, 1, klen, C2, NM, acc, pk1);
  float lo, hi;
  f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lo, hi);
  return lo + hi;
}

// Tensor maps of the permuted layout [B*heads, n_cap, d]: a tile is rows
// [a*128, a*128+128) of plane b*heads + h.
struct PermMaps {
  CUtensorMap q, k, v;
};

// TOK: Q, K, V in token order through the per-tiling 5D maps (TokenMaps).
template <int D, bool TOK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    sparse_attn_pair_kernel(const __grid_constant__ LayerGeom g,
                            const __grid_constant__ std::conditional_t<TOK, TokenMaps, PermMaps> maps,
                            const PairParams prm) {
  using Lay = PairLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

  const int cp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * g.heads + h;
  const HeadGeom& hg = g.h[h];
  const int nt = hg.nt;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // the two query tiles (qbt >= nt: none), or two padding tiles to zero
  int qa, qbt;
  {
    const int S = pair_stride(hg), n_axis = nt / S, n_pairs = (n_axis + 1) / 2 * S;
    if (cp < n_pairs) {
      const int j = cp / S, rr = cp - j * S;
      qa = 2 * j * S + rr;
      qbt = 2 * j + 1 < n_axis ? qa + S : nt;
    } else {
      qa = nt + 2 * (cp - n_pairs);
      qbt = qa + 1;
    }
  }
  const long long rowA = (long long)bh * g.n_cap + (long long)qa * BM;
  const long long rowB = (long long)bh * g.n_cap + (long long)qbt * BM;

  if (qa >= nt) {  // both query tiles are padding: zero output rows (none in token order)
    for (int i = threadIdx.x; prm.op && i < 2 * BM * D / 8; i += NUM_THREADS) {
      const int r = i / (D / 8);
      if (qa * BM + r < g.n_cap)
        reinterpret_cast<uint4*>(prm.op + (rowA + r) * D)[i % (D / 8)] = make_uint4(0, 0, 0, 0);
    }
    if (prm.lse)
      for (int r = threadIdx.x; r < 2 * BM; r += NUM_THREADS)
        if (qa * BM + r < g.n_cap) prm.lse[rowA + r] = 0.f;
    return;
  }
  const bool has_b = qbt < nt;
  const int n = hg.k;
  const int kA = n, kB = has_b ? n : 0;
  const int32_t* listA = prm.idx ? prm.idx + ((long long)bh * g.nt_cap + qa) * prm.k_cap : nullptr;
  const int32_t* listB = prm.idx ? prm.idx + ((long long)bh * g.nt_cap + (has_b ? qbt : qa)) * prm.k_cap : nullptr;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + KST;
  uint64_t* step_done = v_full + VST;  // [SDR]: all MMAs of union position e issued, and P V of e-1
  uint64_t* s_full = step_done + SDR;  // [2]
  uint64_t* p_full = s_full + 2;     // [2], 128 arrivals each
  uint64_t* pv_done = p_full + 2;    // [2], one phase: the query tile's last P V
  uint64_t* mma_drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);
  volatile int* list_bad = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 8);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(smem + Lay::OFF_BM);
  uint32_t* bmB = bmA + prm.bm_words;
  const bool try_bm = prm.idx != nullptr && prm.bm_words > 0;  // uniform over the CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < Lay::NUM_BARS; ++i) {
      uint64_t* bar = bars + i;
      mbar_init(bar, (bar == p_full || bar == p_full + 1) ? 128 : 1);
    }
    *abort_flag = 0;
    *list_bad = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (try_bm) {
    // kept-tile bitmaps of both lists, built by all threads; an entry out of
    // range or not above its predecessor leaves the CTA on the list merge
    for (int i = threadIdx.x; i < 2 * prm.bm_words; i += NUM_THREADS) bmA[i] = 0u;
    __syncthreads();
    build_kept_bitmaps(listA, kA, listB, kB, nt, bmA, bmB, list_bad, threadIdx.x, NUM_THREADS);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool use_bm = try_bm && *list_bad == 0;
  if (warp >= 8) {
  regs_lower<REGS_ROLES>();
  if (warp == 8 || warp == 10) {
    // ----------------------------------------------------------- producers
    if (lane == 0) {
      const bool is_k = warp == 8;
      const CUtensorMap* map;
      const CUtensorMap* qmap;
      if constexpr (TOK) {
        map = is_k ? &maps.k[hg.tmap] : &maps.v[hg.tmap];
        qmap = &maps.q[hg.tmap];
      } else {
        map = is_k ? &maps.k : &maps.v;
        qmap = &maps.q;
      }
      // columns [bx*64, bx*64+64) of the 128 rows of tile a
      auto load_tile = [&](void* dst, const CUtensorMap* m, uint64_t* bar, int bx, int a) {
        if constexpr (TOK) tma_load_tile_tokens(dst, m, bar, g, hg, bx * 64, h, b, a);
        else tma_load_3d(dst, m, bar, bx * 64, a * BN, bh);
      };
      uint64_t* full = is_k ? k_full : v_full;
      const int ST = is_k ? KST : VST;
      uint8_t* ring = smem + (is_k ? Lay::OFF_K : Lay::OFF_V);
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(qmap);
        mbar_expect_tx(q_full, 2 * Lay::QB);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          load_tile(smem + Lay::OFF_Q + bx * BM * 128, qmap, q_full, bx, qa);
          load_tile(smem + Lay::OFF_Q + Lay::QB + bx * BM * 128, qmap, q_full, bx, qbt);
        }
      }
      int e = 0;
      // one instance per walk type, so only one walk's state is live
      auto produce = [&](auto& uw) {
      int t;
      bool ma, mb;
      while (uw.next(t, ma, mb)) {
        const int st = e % ST;
        // slot reuse: K of position e-KST is free once its S MMAs completed
        // (step e-KST); V of e-VST once its P V completed (issued by the end
        // of step e-VST+1)
        const int sd = e - ST + (is_k ? 0 : 1);
        if (e >= ST && !mbar_wait(step_done + sd % SDR, (sd / SDR) & 1, abort_flag, g.dev_status)) break;
        mbar_expect_tx(full + st, Lay::KB);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          load_tile(ring + st * Lay::KB + bx * BN * 128, map, full + st, bx, t);
        ++e;
      }
      };
      if (use_bm && !hg.padded) {
        AltWalk w(bmA, bmB, prm.bm_words);
        produce(w);
      } else if (use_bm) {
        BitWalk w(bmA, bmB, prm.bm_words);
        produce(w);
      } else {
        UnionWalk w(listA, kA, listB, kB, nt, is_k ? g.dev_status : nullptr);
        produce(w);
      }
      if (*abort_flag) {  // let every copy this warp started land before exiting
        if (is_k) mbar_wait_drain(q_full, 0, VEDA_WAIT_LIMIT_NS);
        for (int x = e - ST < 0 ? 0 : e - ST; x < e; ++x)
          mbar_wait_drain(full + x % ST, (x / ST) & 1, VEDA_WAIT_LIMIT_NS);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(BM, D, false, true);
      // Descriptors are built once; an operand's position inside a ring slot
      // or a tile only adds (byte offset >> 4) to the start-address field,
      // which never carries out of it for addresses below 256 KB.
      const uint64_t dQ = sdesc_sw128(smem_u32(smem + Lay::OFF_Q), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(smem + Lay::OFF_K), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(smem + Lay::OFF_V), BN * 128, 1024);
      // Per query tile state in scalars, and P V / S issue specialised per
      // query tile at compile time: this thread's bookkeeping between MMA
      // batches is on the critical path, and nothing here may live in local
      // memory.
      bool pend0 = false, pend1 = false;  // a P V is pending
      int js0 = 0, js1 = 0;               // S issued
      int prev_e = -1;
      int v_seen = -1;  // V ring entry already waited for
      bool ok = mbar_wait(q_full, 0, abort_flag, g.dev_status);
      if (ok) tc_fence_after();
      using I0 = std::integral_constant<int, 0>;
      using I1 = std::integral_constant<int, 1>;
      // P V for the tile query tile r kept at union position prev_e
      auto issue_pv = [&](auto rc) -> bool {
        constexpr int r = decltype(rc)::value;
        int& js = r ? js1 : js0;
        bool& pend = r ? pend1 : pend0;
        const int vs = prev_e % VST;
        if (!mbar_wait(p_full + r, (js - 1) & 1, abort_flag, g.dev_status)) return false;
        if (v_seen != prev_e) {  // both query tiles' P V of a shared tile read one V entry
          if (!mbar_wait(v_full + vs, (prev_e / VST) & 1, abort_flag, g.dev_status)) return false;
          v_seen = prev_e;
        }
        tc_fence_after();
        const uint32_t o_addr = tmem + 2 * BN + r * D, p_addr = tmem + r * BN + 64;
        const uint64_t dVs = dV + (uint64_t)(vs * (Lay::KB >> 4));
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ts(o_addr, p_addr + kk * 8, dVs + (uint64_t)(kk * (2048 >> 4)), idesc_o,
                       (js > 1 || kk > 0) ? 1u : 0u);
        if (js == (r ? kB : kA)) umma_commit(pv_done + r);  // the query tile's last P V
        pend = false;
        return true;
      };
      // S = Q_r K^T for the K tile in ring slot st
      auto issue_s = [&](auto rc, int st) {
        constexpr int r = decltype(rc)::value;
        const uint64_t dQr = dQ + (uint64_t)(r * (Lay::QB >> 4)), dKs = dK + (uint64_t)(st * (Lay::KB >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4;
          umma_bf16_ss(tmem + r * BN, dQr + off, dKs + off, idesc_s, kk > 0);
        }
        umma_commit(s_full + r);
        (r ? js1 : js0)++;
        (r ? pend1 : pend0) = true;
      };
      // one instance per walk type, so only one walk's state is live
      auto issue_all = [&](auto& uw) {
      int t, e = 0;
      bool mA, mB;
      while (ok && uw.next(t, mA, mB)) {
        const int st = e % KST;
        if (!mbar_wait(k_full + st, (e / KST) & 1, abort_flag, g.dev_status)) break;
        tc_fence_after();
        // query tiles that kept tile e: finish their previous P V (P shares
        // the S columns), then S for tile e
        if (mA) {
          if (pend0 && !(ok = issue_pv(I0{}))) break;
          issue_s(I0{}, st);
        }
        if (mB) {
          if (pend1 && !(ok = issue_pv(I1{}))) break;
          issue_s(I1{}, st);
        }
        // a query tile that did not keep it: release its P V of tile e-1
        // only now, so its softmax overlaps the S just issued
        if (!mA && pend0 && !(ok = issue_pv(I0{}))) break;
        if (!mB && pend1 && !(ok = issue_pv(I1{}))) break;
        umma_commit(step_done + e % SDR);  // frees K of e and V of e-1 for the producers
        prev_e = e;
        ++e;
      }
      };
      if (use_bm && !hg.padded) {
        AltWalk w(bmA, bmB, prm.bm_words);
        issue_all(w);
      } else if (use_bm) {
        BitWalk w(bmA, bmB, prm.bm_words);
        issue_all(w);
      } else {
        UnionWalk w(listA, kA, listB, kB, nt, nullptr);
        issue_all(w);
      }
      if (ok && pend0) ok = issue_pv(I0{});
      if (ok && pend1) ok = issue_pv(I1{});
      umma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0, VEDA_WAIT_LIMIT_NS);
    }
  }
  } else {
    regs_raise<REGS_SOFTMAX>();
    // ------------------------------------------------------------- softmax
    const int r = warp / 4;              // query tile A (0) or B (1)
    const int row = threadIdx.x % BM;    // row in the tile = TMEM lane
    const int a = r ? qbt : qa;
    const int kr = r ? kB : kA;
    const int32_t* my_list = r ? listB : listA;
    const bool row_valid = a < nt && row < tile_len(hg, g.T, a);
    const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t s_col = r * BN, o_col = 2 * BN + r * D;
    const float C = prm.scale_log2;
    const uint64_t C2 = f2(C, C);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // A head whose tiles are all full never needs the kept tile's index here.
    // Otherwise the next list entry is loaded one iteration ahead and
    // range-clamped only when used, so its latency never stalls an iteration.
    const bool padded = hg.padded != 0;
    const int32_t* pad_list = padded ? my_list : nullptr;
    int raw_next = (kr > 0 && pad_list) ? __ldg(pad_list) : 0;
    for (int j = 0; j < kr; ++j) {
      int klen = BN;
      if (padded) {
        const int raw = pad_list ? raw_next : j;
        if (pad_list && j + 1 < kr) raw_next = __ldg(pad_list + j + 1);
        const int kt = (raw >= 0 && raw < nt) ? raw : 0;
        klen = tile_len(hg, g.T, kt);
      }
      const bool full = klen >= BN;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + r, j & 1, abort_flag, g.dev_status))) { ok = false; break; }
      tc_fence_after();
      // the whole S row in registers: one TMEM load
      uint32_t u[BN];
      tmem_ld128(lane_addr + s_col, u);
      if (j == 0) m = (full ? row_max<true>(u, klen) : row_max<false>(u, klen)) * C;
      uint32_t pk0[32], pk1[32];
      float ts = full ? row_p<true>(u, klen, C2, m, pk0, pk1) : row_p<false>(u, klen, C2, m, pk0, pk1);
      // Later tiles are not max-reduced: P = 2^(s*C - m) may exceed 1 when a
      // tile holds larger logits than the first one did, and fp32 / bf16 keep
      // their relative precision at any magnitude, so the reference m only
      // moves when the tile's sum nears the top of the range (rare). P is not
      // stored yet, so S is still intact in TMEM for the exact recomputation.
      const bool redo = !(ts <= OVERFLOW_SUM);
      if (__any_sync(0xffffffffu, redo)) {
        tmem_ld128(lane_addr + s_col, u);
        const float mx2 = (full ? row_max<true>(u, klen) : row_max<false>(u, klen)) * C;
        const float m_new = redo ? fmaxf(m, mx2) : m;
        const float alpha = fast_exp2(m - m_new);
        if (j > 0) {
          // O already holds P V of the previous tile: the MMA thread issues
          // it before this tile's S, and s_full tracks every MMA it issued
          // before its commit
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_addr + o_col + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(lane_addr + o_col + c * 32, o);
          }
        }
        l *= alpha;
        m = m_new;
        ts = full ? row_p<true>(u, klen, C2, m, pk0, pk1) : row_p<false>(u, klen, C2, m, pk0, pk1);
      }
      // P (bf16 pairs) over columns [64,128) of S: keys [0,64) -> [64,96),
      // keys [64,128) -> [96,128)
      tmem_st32_async(lane_addr + s_col + 64, pk0);
      tmem_st32_async(lane_addr + s_col + 96, pk1);
      tmem_wait_st_keep(pk0, pk1);
      l += ts;
      tc_fence_before();
      mbar_arrive(p_full + r);
    }
    // epilogue: O / l -> bf16
    const long long orow_i = (r ? rowB : rowA) + row;
    const bool in_range = a * BM + row < g.n_cap;
    if (kr == 0) {  // query tile beyond this head's tiles: zero rows (none in token order)
      if (in_range) {
        if (prm.op) {
          uint4* dst = reinterpret_cast<uint4*>(prm.op + orow_i * D);
#pragma unroll
          for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0, 0, 0, 0);
        }
        if (prm.lse) prm.lse[orow_i] = 0.f;
      }
    } else if (ok && __all_sync(0xffffffffu, mbar_wait(pv_done + r, 0, abort_flag, g.dev_status))) {
      tc_fence_after();
      const float inv = row_valid ? 1.0f / l : 0.f;
      // the row's destination: its permuted slot, or its token (padding rows
      // have none)
      __nv_bfloat16* orow = nullptr;
      if (prm.otok) {
        const long long n = row_valid ? tile_row_token(g, hg, a, row) : -1;
        if (n >= 0) orow = prm.otok + (((long long)b * g.T * g.H * g.W + n) * g.heads + h) * D;
      } else if (in_range) {
        orow = prm.op + orow_i * D;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(lane_addr + o_col + c * 32, u);
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
      if (prm.lse && in_range) prm.lse[orow_i] = row_valid ? (m + __log2f(l)) * 0.69314718055994531f : 0.f;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D, bool TOK>
cudaError_t launch_pair_t(const LayerGeom& g0, const void* qp, const void* kp, const void* vp, const PairParams& prm,
                          cudaStream_t s) {
  LayerGeom g = g0;
  std::conditional_t<TOK, TokenMaps, PermMaps> maps;
  if constexpr (TOK) {
    const cudaError_t e = build_token_maps(g, qp, kp, vp, &maps);
    if (e != cudaSuccess) return e;
  } else {
    const uint64_t rows = (uint64_t)g.n_cap, planes = (uint64_t)g.B * g.heads;
    if (encode_tensor_map_3d_bf16(&maps.q, qp, D, rows, planes, 64, BM) != CUDA_SUCCESS ||
        encode_tensor_map_3d_bf16(&maps.k, kp, D, rows, planes, 64, BN) != CUDA_SUCCESS ||
        encode_tensor_map_3d_bf16(&maps.v, vp, D, rows, planes, 64, BN) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = sparse_attn_pair_kernel<D, TOK>;
  PairParams p = prm;
  p.bm_words = (g.nt_cap + 31) / 32;
  int smem = PairLayout<D>::alloc(p.bm_words);
  if (smem > 232448) {  // bitmaps do not fit beside the rings: list merge
    p.bm_words = 0;
    smem = PairLayout<D>::alloc(0);
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int ctas = 1;
  for (int h = 0; h < g.heads; ++h) {
    const int c = pair_ctas(g.h[h], g.nt_cap);
    ctas = c > ctas ? c : ctas;
  }
  const dim3 grid(ctas, g.heads, g.B);
  kern<<<grid, NUM_THREADS, smem, s>>>(g, maps, p);
  return cudaGetLastError();
}

}  // namespace

// 128-token tiles: two query tiles per CTA sharing the loads of their union.
// tokens_in: qp, kp, vp are in token order [B, N, heads, d] (then o_tokens is
// the output).
cudaError_t launch_sparse_attn_pair(const LayerGeom& g, const void* qp, const void* kp, const void* vp,
                                    const int32_t* idx, int k_cap, float scale, void* op, float* lse,
                                    cudaStream_t s, void* o_tokens, bool tokens_in) {
  PairParams prm;
  prm.otok = reinterpret_cast<__nv_bfloat16*>(o_tokens);
  prm.k_cap = k_cap;
  prm.bm_words = 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.idx = idx;
  prm.op = o_tokens ? nullptr : reinterpret_cast<__nv_bfloat16*>(op);
  prm.lse = lse;
  if (tokens_in) {
    if (!o_tokens) return cudaErrorInvalidValue;
    if (g.d == 128) return launch_pair_t<128, true>(g, qp, kp, vp, prm, s);
    return launch_pair_t<64, true>(g, qp, kp, vp, prm, s);
  }
  if (g.d == 128) return launch_pair_t<128, false>(g, qp, kp, vp, prm, s);
  return launch_pair_t<64, false>(g, qp, kp, vp, prm, s);
}

}  // namespace veda
