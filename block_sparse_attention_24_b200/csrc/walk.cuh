// Walks over the union of two query tiles' kept key-tile lists, shared by the
// attention kernels (Veda summary 2.3: only kept key tiles are loaded; two
// query tiles that share a CTA load each tile of their union once).
#pragma once

#include <climits>

#include "veda_internal.cuh"

namespace veda {

// Walks the merge of two kept-tile lists: each call yields the next tile and
// which of the two query tiles kept it. Every entry of both lists is visited
// exactly once; equal entries are merged. Each list's entry after the current
// one is loaded one step ahead and range-checked only when it becomes current,
// so a call never waits for a load.
struct UnionWalk {
  const int32_t* la;
  const int32_t* lb;
  int ka, kb, ia, ib, nt;
  int ta, tb;          // current entries (range-checked), INT_MAX past the end
  int ra, rb;          // raw next entries
  int32_t* status;
  __device__ int raw(const int32_t* l, int j, int k) { return j < k ? (l ? __ldg(l + j) : j) : 0; }
  __device__ int checked(int t, bool report_bad) {
    if (t < 0 || t >= nt) {
      if (report_bad && status) report(status, VEDA_ERR_BAD_INDEX);
      t = 0;
    }
    return t;
  }
  __device__ UnionWalk(const int32_t* a, int na, const int32_t* b, int nb, int nt_, int32_t* st)
      : la(a), lb(b), ka(na), kb(nb), ia(0), ib(0), nt(nt_), status(st) {
    ta = ka > 0 ? checked(raw(la, 0, ka), true) : INT_MAX;
    tb = kb > 0 ? checked(raw(lb, 0, kb), true) : INT_MAX;
    ra = raw(la, 1, ka);
    rb = raw(lb, 1, kb);
  }
  __device__ bool next(int& t, bool& ma, bool& mb) {
    if (ia >= ka && ib >= kb) return false;
    t = ta < tb ? ta : tb;
    ma = ta == t;
    mb = tb == t;
    if (ma) {
      ta = ++ia < ka ? checked(ra, true) : INT_MAX;
      ra = raw(la, ia + 1, ka);
    }
    if (mb) {
      tb = ++ib < kb ? checked(rb, true) : INT_MAX;
      rb = raw(lb, ib + 1, kb);
    }
    return true;
  }
};

// The same walk over kept-tile bitmaps in shared memory (valid when both
// lists are ascending, distinct and in range): the next union tile is the
// lowest set bit of the two current words, so a step costs a few integer
// instructions and no load except one shared word per 32 tiles.
struct BitWalk {
  const uint32_t* a;
  const uint32_t* b;
  int nw, wi;
  uint32_t wa, wb;  // current words with the tiles already visited cleared
  __device__ BitWalk(const uint32_t* a_, const uint32_t* b_, int nw_) : a(a_), b(b_), nw(nw_), wi(0), wa(0), wb(0) {
    if (nw > 0) wa = a[0], wb = b[0];
  }
  __device__ bool next(int& t, bool& ma, bool& mb) {
    while ((wa | wb) == 0u) {
      if (++wi >= nw) return false;
      wa = a[wi];
      wb = b[wi];
    }
    const int pos = __ffs(wa | wb) - 1;
    const uint32_t bit = 1u << pos;
    ma = (wa & bit) != 0u;
    mb = (wb & bit) != 0u;
    wa &= ~bit;
    wb &= ~bit;
    t = wi * 32 + pos;
    return true;
  }
};

// Builds the kept-tile bitmaps of two lists (words each) in shared memory
// with every thread of the CTA; sets *bad when an entry is out of range or
// not above its predecessor (then the lists must be merged as given). The
// caller zeroes *bad and synchronises before and after.
__device__ inline void build_kept_bitmaps(const int32_t* la, int ka, const int32_t* lb, int kb, int nt,
                                                   uint32_t* bma, uint32_t* bmb, volatile int* bad, int tid,
                                                   int nthreads) {
  for (int i = tid; i < ka + kb; i += nthreads) {
    const bool in_b = i >= ka;
    const int32_t* l = in_b ? lb : la;
    const int j = in_b ? i - ka : i, kl = in_b ? kb : ka;
    const int t = __ldg(l + j);
    if (t < 0 || t >= nt || (j + 1 < kl && __ldg(l + j + 1) <= t)) *bad = 1;
    else atomicOr((in_b ? bmb : bma) + (t >> 5), 1u << (t & 31));
  }
}

}  // namespace veda
