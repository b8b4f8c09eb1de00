// C ABI entry points of libveda.so: argument validation, layer geometry and
// dispatch to the kernels. Every check here runs before any launch, so a bad
// call returns an error code and leaves the device untouched.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "veda_internal.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(VEDA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Fills `g` from the layer and validates the geometry.
int build_geom(const veda_layer* L, veda::LayerGeom* g) {
  if (!L) return fail(VEDA_ERR_INVALID_ARG, "layer is NULL");
  if (L->B < 1) return fail(VEDA_ERR_INVALID_ARG, "B=%d must be >= 1", L->B);
  if (L->heads < 1 || L->heads > VEDA_MAX_HEADS)
    return fail(VEDA_ERR_INVALID_ARG, "heads=%d outside [1, %d]", L->heads, VEDA_MAX_HEADS);
  if (L->d != 64 && L->d != 128) return fail(VEDA_ERR_UNSUPPORTED, "d=%d: only 64 and 128 are built", L->d);
  if (L->tile != 64 && L->tile != 128)
    return fail(VEDA_ERR_UNSUPPORTED, "tile=%d: only 64 and 128 are built", L->tile);
  if (L->T < 1 || L->H < 1 || L->W < 1) return fail(VEDA_ERR_INVALID_ARG, "empty grid %dx%dx%d", L->T, L->H, L->W);
  if (!L->tilings) return fail(VEDA_ERR_INVALID_ARG, "tilings is NULL");
  const long long N = (long long)L->T * L->H * L->W;
  if (N * L->heads * L->d * (long long)L->B > (1ll << 40)) return fail(VEDA_ERR_UNSUPPORTED, "layer too large");
  std::memset(g, 0, sizeof(*g));
  g->B = L->B;
  g->heads = L->heads;
  g->d = L->d;
  g->T = L->T;
  g->H = L->H;
  g->W = L->W;
  g->tile = L->tile;
  g->dev_status = L->dev_status;
  int n_cap = 0, nt_cap = 0;
  for (int h = 0; h < L->heads; ++h) {
    const veda_tiling t = L->tilings[h];
    if (t.pt < 1 || t.ph < 1 || t.pw < 1)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: tiling (%d,%d,%d) has a non-positive extent", h, t.pt, t.ph, t.pw);
    if ((long long)t.pt * t.ph * t.pw != L->tile)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: tiling (%d,%d,%d) does not factorise tile %d", h, t.pt, t.ph,
                  t.pw, L->tile);
    if (L->H % t.ph || L->W % t.pw)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: p_h=%d, p_w=%d must divide H=%d, W=%d", h, t.ph, t.pw, L->H,
                  L->W);
    veda::HeadGeom& hg = g->h[h];
    hg.pt = t.pt;
    hg.ph = t.ph;
    hg.pw = t.pw;
    hg.nwt = L->W / t.pw;
    hg.tps = (L->H / t.ph) * hg.nwt;
    const long long ntt = (L->T + t.pt - 1) / t.pt;
    const long long nt = ntt * hg.tps;
    if (nt > VEDA_MAX_NT) return fail(VEDA_ERR_UNSUPPORTED, "head %d: %lld tiles exceeds %d", h, nt, VEDA_MAX_NT);
    hg.nt = (int)nt;
    hg.k = 0;
    hg.padded = (L->T % t.pt) != 0;
    hg.tmap = 0;
    if (nt > nt_cap) nt_cap = (int)nt;
    if (nt * L->tile > n_cap) n_cap = (int)(nt * L->tile);
  }
  g->n_cap = n_cap;
  g->nt_cap = nt_cap;
  return VEDA_OK;
}

int check_ptr(const void* p, const char* name) {
  if (!p) return fail(VEDA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(VEDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return VEDA_OK;
}

#define VEDA_TRY(expr)          \
  do {                          \
    int _rc = (expr);           \
    if (_rc != VEDA_OK) return _rc; \
  } while (0)

int after_launch(cudaError_t e, const char* where) {
  if (e != cudaSuccess) return cuda_fail(e, where);
  g_last_error.clear();
  return VEDA_OK;
}

}  // namespace

namespace veda {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

CUresult encode_tensor_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                                   uint32_t box0, uint32_t box1) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return CUDA_ERROR_NOT_FOUND;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};  // bytes, dims 1 and 2
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// One token-layout map (see TokenMaps) for tiling (pt, ph, pw).
CUresult encode_tensor_map_tokens_bf16(CUtensorMap* map, const void* base, const LayerGeom& g, int pt, int ph,
                                       int pw) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return CUDA_ERROR_NOT_FOUND;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  const cuuint64_t d = (cuuint64_t)g.d, hd = d * g.heads;
  cuuint64_t dims[5] = {d, (cuuint64_t)g.heads, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T * g.B};
  cuuint64_t strides[4] = {d * 2, hd * 2, hd * g.W * 2, hd * g.W * g.H * 2};  // bytes, dims 1..4
  cuuint32_t box[5] = {64, 1, (cuuint32_t)pw, (cuuint32_t)ph, (cuuint32_t)pt};
  cuuint32_t estride[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

cudaError_t build_token_maps(LayerGeom& g, const void* q, const void* k, const void* v, TokenMaps* maps) {
  int n = 0, tp[VEDA_MAX_TILINGS][3];
  for (int h = 0; h < g.heads; ++h) {
    HeadGeom& hg = g.h[h];
    int i = 0;
    while (i < n && !(tp[i][0] == hg.pt && tp[i][1] == hg.ph && tp[i][2] == hg.pw)) ++i;
    if (i == n) {
      if (n == VEDA_MAX_TILINGS) return cudaErrorNotSupported;
      tp[n][0] = hg.pt, tp[n][1] = hg.ph, tp[n][2] = hg.pw;
      ++n;
    }
    hg.tmap = i;
  }
  for (int i = 0; i < n; ++i) {
    if (encode_tensor_map_tokens_bf16(&maps->q[i], q, g, tp[i][0], tp[i][1], tp[i][2]) != CUDA_SUCCESS ||
        encode_tensor_map_tokens_bf16(&maps->k[i], k, g, tp[i][0], tp[i][1], tp[i][2]) != CUDA_SUCCESS ||
        (v && encode_tensor_map_tokens_bf16(&maps->v[i], v, g, tp[i][0], tp[i][1], tp[i][2]) != CUDA_SUCCESS))
      return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

}  // namespace veda

extern "C" {

const char* veda_last_error(void) { return g_last_error.c_str(); }

int veda_layout(const veda_layer* L, int32_t* nt, int32_t* n_pad, int32_t* n_cap, int32_t* nt_cap) {
  veda::LayerGeom local;
  VEDA_TRY(build_geom(L, &local));
  for (int h = 0; h < L->heads; ++h) {
    if (nt) nt[h] = local.h[h].nt;
    if (n_pad) n_pad[h] = local.h[h].nt * L->tile;
  }
  if (n_cap) *n_cap = local.n_cap;
  if (nt_cap) *nt_cap = local.nt_cap;
  g_last_error.clear();
  return VEDA_OK;
}

int veda_permute(const veda_layer* L, const void* x, void* xp, int32_t* perm, int inverse, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  VEDA_TRY(check_ptr(x, "x"));
  VEDA_TRY(check_ptr(xp, "xp"));
  if (perm && !inverse) VEDA_TRY(check_ptr(perm, "perm"));
  if (inverse != 0 && inverse != 1) return fail(VEDA_ERR_INVALID_ARG, "inverse must be 0 or 1");
  return after_launch(veda::launch_permute(g, x, xp, inverse ? nullptr : perm, inverse, stream), "veda_permute");
}

int veda_trippool(const veda_layer* L, const void* xp, float* desc, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  VEDA_TRY(check_ptr(xp, "xp"));
  VEDA_TRY(check_ptr(desc, "desc"));
  return after_launch(veda::launch_trippool(g, xp, desc, stream), "veda_trippool");
}

int veda_permute_trippool(const veda_layer* L, const void* x, void* xp, int32_t* perm, float* desc,
                          cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  VEDA_TRY(check_ptr(x, "x"));
  VEDA_TRY(check_ptr(xp, "xp"));
  VEDA_TRY(check_ptr(desc, "desc"));
  if (perm) VEDA_TRY(check_ptr(perm, "perm"));
  return after_launch(veda::launch_permute_pool(g, x, xp, perm, desc, stream), "veda_permute_trippool");
}

size_t veda_tile_scores_ws_bytes(const veda_layer* L, int32_t out_dim) {
  veda::LayerGeom g;
  if (build_geom(L, &g) != VEDA_OK || out_dim < 1) return 0;
  return (size_t)2 * g.B * g.heads * g.nt_cap * out_dim * sizeof(float);
}

int veda_tile_scores(const veda_layer* L, const float* dq, const float* dk, const float* w1q, const float* b1q,
                     const float* w2q, const float* b2q, const float* w1k, const float* b1k, const float* w2k,
                     const float* b2k, int32_t hidden, int32_t out_dim, float scale, float* scores, float* emb_ws,
                     cudaStream_t stream) {
  return veda_tile_scores_heads(L, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden, out_dim, scale, scores,
                                emb_ws, nullptr, stream);
}

int veda_tile_scores_heads(const veda_layer* L, const float* dq, const float* dk, const float* w1q, const float* b1q,
                           const float* w2q, const float* b2q, const float* w1k, const float* b1k, const float* w2k,
                           const float* b2k, int32_t hidden, int32_t out_dim, float scale, float* scores,
                           float* emb_ws, const int32_t* head_on, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  const void* ptrs[] = {dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, scores, emb_ws};
  const char* names[] = {"dq", "dk", "w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k", "scores", "emb_ws"};
  for (int i = 0; i < 12; ++i) VEDA_TRY(check_ptr(ptrs[i], names[i]));
  if (hidden < 4 || hidden > 256 || hidden % 4)
    return fail(VEDA_ERR_UNSUPPORTED, "hidden=%d must be a multiple of 4 in [4, 256]", hidden);
  if (out_dim < 4 || out_dim > 128 || out_dim % 4)
    return fail(VEDA_ERR_UNSUPPORTED, "out_dim=%d must be a multiple of 4 in [4, 128]", out_dim);
  if (head_on) VEDA_TRY(check_ptr(head_on, "head_on"));
  return after_launch(veda::launch_tile_scores(g, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden, out_dim,
                                               scale, scores, emb_ws, stream, head_on),
                      "veda_tile_scores");
}

int veda_topk_mask(const veda_layer* L, const float* scores, const int32_t* k, int32_t k_cap, int32_t* idx,
                   uint8_t* mask, cudaStream_t stream) {
  return veda_topk_mask_heads(L, scores, k, k_cap, idx, mask, nullptr, stream);
}

int veda_topk_mask_heads(const veda_layer* L, const float* scores, const int32_t* k, int32_t k_cap, int32_t* idx,
                         uint8_t* mask, const int32_t* head_on, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  VEDA_TRY(check_ptr(scores, "scores"));
  VEDA_TRY(check_ptr(idx, "idx"));
  if (mask) VEDA_TRY(check_ptr(mask, "mask"));
  if (!k) return fail(VEDA_ERR_INVALID_ARG, "k is NULL");
  if (k_cap < 1) return fail(VEDA_ERR_INVALID_ARG, "k_cap=%d must be >= 1", k_cap);
  for (int h = 0; h < g.heads; ++h) {
    if (k[h] < 1 || k[h] > g.h[h].nt || k[h] > k_cap)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: k=%d outside [1, min(nt=%d, k_cap=%d)]", h, k[h], g.h[h].nt, k_cap);
    g.h[h].k = k[h];
  }
  if (head_on) VEDA_TRY(check_ptr(head_on, "head_on"));
  return after_launch(veda::launch_topk(g, scores, k_cap, idx, mask, stream, head_on), "veda_topk_mask");
}

size_t veda_score_cache_ws_bytes(const veda_layer* L) {
  veda::LayerGeom g;
  if (build_geom(L, &g) != VEDA_OK) return 0;
  return veda::score_cache_ws_bytes(g);
}

int veda_score_cache_step(const veda_layer* L, const float* dq, const float* dk, float* dq_ref, float* dk_ref,
                          float tau, int32_t max_age, int32_t* age, int32_t* refresh, void* ws, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  const void* ptrs[] = {dq, dk, dq_ref, dk_ref, age, refresh, ws};
  const char* names[] = {"dq", "dk", "dq_ref", "dk_ref", "age", "refresh", "ws"};
  for (int i = 0; i < 7; ++i) VEDA_TRY(check_ptr(ptrs[i], names[i]));
  if (!(tau >= 0.f) || tau != tau) return fail(VEDA_ERR_INVALID_ARG, "tau=%g must be >= 0", (double)tau);
  if (max_age < 1) return fail(VEDA_ERR_INVALID_ARG, "max_age=%d must be >= 1", max_age);
  return after_launch(veda::launch_score_cache(g, dq, dk, dq_ref, dk_ref, tau, max_age, age, refresh, ws, stream),
                      "veda_score_cache_step");
}

int veda_tile_scores_topk(const veda_layer* L, const float* dq, const float* dk, const float* w1q, const float* b1q,
                          const float* w2q, const float* b2q, const float* w1k, const float* b1k, const float* w2k,
                          const float* b2k, int32_t hidden, int32_t out_dim, float scale, const int32_t* k,
                          int32_t k_cap, int32_t* idx, uint8_t* mask, float* scores, float* emb_ws,
                          cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  const void* ptrs[] = {dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, idx, emb_ws};
  const char* names[] = {"dq", "dk", "w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k", "idx", "emb_ws"};
  for (int i = 0; i < 12; ++i) VEDA_TRY(check_ptr(ptrs[i], names[i]));
  if (mask) VEDA_TRY(check_ptr(mask, "mask"));
  if (scores) VEDA_TRY(check_ptr(scores, "scores"));
  if (hidden < 4 || hidden > 256 || hidden % 4)
    return fail(VEDA_ERR_UNSUPPORTED, "hidden=%d must be a multiple of 4 in [4, 256]", hidden);
  if (out_dim < 4 || out_dim > 128 || out_dim % 4)
    return fail(VEDA_ERR_UNSUPPORTED, "out_dim=%d must be a multiple of 4 in [4, 128]", out_dim);
  if (!k) return fail(VEDA_ERR_INVALID_ARG, "k is NULL");
  if (k_cap < 1) return fail(VEDA_ERR_INVALID_ARG, "k_cap=%d must be >= 1", k_cap);
  for (int h = 0; h < g.heads; ++h) {
    if (k[h] < 1 || k[h] > g.h[h].nt || k[h] > k_cap)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: k=%d outside [1, min(nt=%d, k_cap=%d)]", h, k[h], g.h[h].nt, k_cap);
    g.h[h].k = k[h];
  }
  if ((size_t)g.nt_cap * 4 + (size_t)out_dim * 4 + 8 * 256 * 4 > 200 * 1024)
    return fail(VEDA_ERR_UNSUPPORTED, "nt_cap=%d: a score row does not fit the fused kernel's shared memory", g.nt_cap);
  cudaError_t e = veda::launch_mlp(g, dq, dk, w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k, hidden, out_dim, emb_ws, stream);
  if (e != cudaSuccess) return after_launch(e, "veda_tile_scores_topk");
  return after_launch(veda::launch_score_topk(g, emb_ws, out_dim, scale, k_cap, idx, mask, scores, stream),
                      "veda_tile_scores_topk");
}

namespace {
// Shared by veda_sparse_attn (permuted output `op`) and
// veda_sparse_attn_unpermute (token-order output `o`).
int sparse_attn_call(const veda_layer* L, const void* qp, const void* kp, const void* vp, const int32_t* idx,
                     const int32_t* k, int32_t k_cap, float scale, void* out, bool to_tokens, float* lse,
                     cudaStream_t stream, const char* name, bool tokens_in = false) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  VEDA_TRY(check_ptr(qp, tokens_in ? "q" : "qp"));
  VEDA_TRY(check_ptr(kp, tokens_in ? "k" : "kp"));
  VEDA_TRY(check_ptr(vp, tokens_in ? "v" : "vp"));
  VEDA_TRY(check_ptr(out, to_tokens ? "o" : "op"));
  if (lse) VEDA_TRY(check_ptr(lse, "lse"));
  if (!(scale > 0.f) || scale != scale) return fail(VEDA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (idx) {
    VEDA_TRY(check_ptr(idx, "idx"));
    if (!k) return fail(VEDA_ERR_INVALID_ARG, "k is NULL");
    if (k_cap < 1) return fail(VEDA_ERR_INVALID_ARG, "k_cap=%d must be >= 1", k_cap);
    for (int h = 0; h < g.heads; ++h) {
      if (k[h] < 1 || k[h] > g.h[h].nt || k[h] > k_cap)
        return fail(VEDA_ERR_INVALID_ARG, "head %d: k=%d outside [1, min(nt=%d, k_cap=%d)]", h, k[h], g.h[h].nt,
                    k_cap);
      g.h[h].k = k[h];
    }
  } else {
    for (int h = 0; h < g.heads; ++h) g.h[h].k = g.h[h].nt;
    k_cap = 0;
  }
  const cudaError_t e = veda::launch_sparse_attn(g, qp, kp, vp, idx, k_cap, scale, to_tokens ? nullptr : out, lse,
                                                stream, to_tokens ? out : nullptr, tokens_in);
  if (e == cudaErrorNotSupported)
    return fail(VEDA_ERR_UNSUPPORTED, "%s: more than %d distinct tilings", name, VEDA_MAX_TILINGS);
  return after_launch(e, name);
}
}  // namespace

int veda_sparse_attn(const veda_layer* L, const void* qp, const void* kp, const void* vp, const int32_t* idx,
                     const int32_t* k, int32_t k_cap, float scale, void* op, float* lse, cudaStream_t stream) {
  return sparse_attn_call(L, qp, kp, vp, idx, k, k_cap, scale, op, false, lse, stream, "veda_sparse_attn");
}

int veda_sparse_attn_tokens(const veda_layer* L, const void* q, const void* k_in, const void* v, const int32_t* idx,
                            const int32_t* k, int32_t k_cap, float scale, void* o, float* lse, cudaStream_t stream) {
  return sparse_attn_call(L, q, k_in, v, idx, k, k_cap, scale, o, true, lse, stream, "veda_sparse_attn_tokens",
                          true);
}

int veda_sparse_attn_unpermute(const veda_layer* L, const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, const int32_t* k, int32_t k_cap, float scale, void* o,
                               float* lse, cudaStream_t stream) {
  return sparse_attn_call(L, qp, kp, vp, idx, k, k_cap, scale, o, true, lse, stream, "veda_sparse_attn_unpermute");
}

size_t veda_full_attn_tilemax_ws_bytes(const veda_layer* L, int32_t n_heads_sel, int32_t n_rows) {
  veda::LayerGeom g;
  if (build_geom(L, &g) != VEDA_OK || n_heads_sel < 1 || n_rows < 1) return 0;
  return veda::tilemax_ws_bytes(n_heads_sel, n_rows, g.tile, g.nt_cap);
}

int veda_full_attn_tilemax(const veda_layer* L, const void* qp, const void* kp, const int32_t* heads_sel,
                           int32_t n_heads_sel, const int32_t* qtile_rows, int32_t n_rows, float scale,
                           float* tilemap, float* lse, const float* scores, float* kl_rows, float* kl_out,
                           float* ws, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  if (g.B != 1) return fail(VEDA_ERR_UNSUPPORTED, "tile map: only B == 1 layers are accepted");
  VEDA_TRY(check_ptr(qp, "qp"));
  VEDA_TRY(check_ptr(kp, "kp"));
  VEDA_TRY(check_ptr(tilemap, "tilemap"));
  if (lse) VEDA_TRY(check_ptr(lse, "lse"));
  if (ws) VEDA_TRY(check_ptr(ws, "ws"));
  if (qtile_rows) VEDA_TRY(check_ptr(qtile_rows, "qtile_rows"));
  if (!heads_sel || n_heads_sel < 1 || n_heads_sel > VEDA_MAX_HEADS)
    return fail(VEDA_ERR_INVALID_ARG, "heads_sel must list 1..%d heads", VEDA_MAX_HEADS);
  if (n_rows < 1) return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d must be >= 1", n_rows);
  if (!(scale > 0.f) || scale != scale) return fail(VEDA_ERR_INVALID_ARG, "scale must be positive and finite");
  for (int s = 0; s < n_heads_sel; ++s) {
    if (heads_sel[s] < 0 || heads_sel[s] >= g.heads)
      return fail(VEDA_ERR_INVALID_ARG, "heads_sel[%d]=%d outside [0, %d)", s, heads_sel[s], g.heads);
    if (!qtile_rows && n_rows > g.h[heads_sel[s]].nt)
      return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d exceeds the %d tiles of head %d", n_rows,
                  g.h[heads_sel[s]].nt, heads_sel[s]);
  }
  if (scores) {
    VEDA_TRY(check_ptr(scores, "scores"));
    VEDA_TRY(check_ptr(kl_rows, "kl_rows"));
    VEDA_TRY(check_ptr(kl_out, "kl_out"));
  }
  return after_launch(veda::launch_tilemax(g, qp, kp, heads_sel, n_heads_sel, qtile_rows, n_rows, scale, tilemap,
                                           lse, scores, scores ? kl_rows : nullptr, scores ? kl_out : nullptr, ws,
                                           stream),
                      "veda_full_attn_tilemax");
}

int veda_tilemap_kl(const veda_layer* L, const int32_t* heads_sel, int32_t n_heads_sel, const int32_t* qtile_rows,
                    int32_t n_rows, const float* tilemap, const float* scores, float* kl_rows, float* kl_out,
                    cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  if (g.B != 1) return fail(VEDA_ERR_UNSUPPORTED, "tile map KL: only B == 1 layers are accepted");
  VEDA_TRY(check_ptr(tilemap, "tilemap"));
  VEDA_TRY(check_ptr(scores, "scores"));
  VEDA_TRY(check_ptr(kl_rows, "kl_rows"));
  VEDA_TRY(check_ptr(kl_out, "kl_out"));
  if (qtile_rows) VEDA_TRY(check_ptr(qtile_rows, "qtile_rows"));
  if (!heads_sel || n_heads_sel < 1 || n_heads_sel > VEDA_MAX_HEADS)
    return fail(VEDA_ERR_INVALID_ARG, "heads_sel must list 1..%d heads", VEDA_MAX_HEADS);
  if (n_rows < 1) return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d must be >= 1", n_rows);
  for (int s = 0; s < n_heads_sel; ++s) {
    if (heads_sel[s] < 0 || heads_sel[s] >= g.heads)
      return fail(VEDA_ERR_INVALID_ARG, "heads_sel[%d]=%d outside [0, %d)", s, heads_sel[s], g.heads);
    if (!qtile_rows && n_rows > g.h[heads_sel[s]].nt)
      return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d exceeds the %d tiles of head %d", n_rows,
                  g.h[heads_sel[s]].nt, heads_sel[s]);
  }
  return after_launch(veda::launch_tilemap_kl(g, heads_sel, n_heads_sel, qtile_rows, n_rows, tilemap, scores,
                                              kl_rows, kl_out, stream),
                      "veda_tilemap_kl");
}

int veda_tilemap_recall(const veda_layer* L, const int32_t* heads_sel, int32_t n_heads_sel,
                        const int32_t* qtile_rows, int32_t n_rows, const float* tilemap, const int32_t* idx,
                        const int32_t* k, int32_t k_cap, int32_t* hits, int32_t* map_idx, float* recall,
                        cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  if (g.B != 1) return fail(VEDA_ERR_UNSUPPORTED, "recall: only B == 1 layers are accepted");
  VEDA_TRY(check_ptr(tilemap, "tilemap"));
  VEDA_TRY(check_ptr(idx, "idx"));
  VEDA_TRY(check_ptr(hits, "hits"));
  VEDA_TRY(check_ptr(recall, "recall"));
  if (map_idx) VEDA_TRY(check_ptr(map_idx, "map_idx"));
  if (qtile_rows) VEDA_TRY(check_ptr(qtile_rows, "qtile_rows"));
  if (!heads_sel || n_heads_sel < 1 || n_heads_sel > VEDA_MAX_HEADS)
    return fail(VEDA_ERR_INVALID_ARG, "heads_sel must list 1..%d heads", VEDA_MAX_HEADS);
  if (n_rows < 1) return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d must be >= 1", n_rows);
  if (!k) return fail(VEDA_ERR_INVALID_ARG, "k is NULL");
  if (k_cap < 1 || k_cap > VEDA_MAX_NT) return fail(VEDA_ERR_INVALID_ARG, "k_cap=%d outside [1, %d]", k_cap, VEDA_MAX_NT);
  for (int h = 0; h < g.heads; ++h) {
    if (k[h] < 1 || k[h] > g.h[h].nt || k[h] > k_cap)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: k=%d outside [1, min(nt=%d, k_cap=%d)]", h, k[h], g.h[h].nt, k_cap);
    g.h[h].k = k[h];
  }
  for (int s = 0; s < n_heads_sel; ++s) {
    if (heads_sel[s] < 0 || heads_sel[s] >= g.heads)
      return fail(VEDA_ERR_INVALID_ARG, "heads_sel[%d]=%d outside [0, %d)", s, heads_sel[s], g.heads);
    if (!qtile_rows && n_rows > g.h[heads_sel[s]].nt)
      return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d exceeds the %d tiles of head %d", n_rows,
                  g.h[heads_sel[s]].nt, heads_sel[s]);
  }
  return after_launch(veda::launch_recall(g, heads_sel, n_heads_sel, qtile_rows, n_rows, tilemap, idx, k_cap, hits,
                                          map_idx, recall, stream),
                      "veda_tilemap_recall");
}

size_t veda_estimator_grad_ws_bytes(const veda_layer* L, int32_t n_heads_sel, int32_t n_rows, int32_t hidden,
                                    int32_t out_dim) {
  veda::LayerGeom g;
  if (build_geom(L, &g) != VEDA_OK || n_heads_sel < 1 || n_rows < 1 || hidden < 1 || out_dim < 1) return 0;
  return (size_t)n_heads_sel * veda::estimator_ws_floats_per_head(g.nt_cap, n_rows, hidden, out_dim, 3 * g.d) *
         sizeof(float);
}

int veda_estimator_grad(const veda_layer* L, const float* dq, const float* dk, const float* w1q, const float* b1q,
                        const float* w2q, const float* b2q, const float* w1k, const float* b1k, const float* w2k,
                        const float* b2k, int32_t hidden, int32_t out_dim, float scale, const int32_t* heads_sel,
                        int32_t n_heads_sel, const int32_t* qtile_rows, int32_t n_rows, const float* tilemap,
                        float* g_w1q, float* g_b1q, float* g_w2q, float* g_b2q, float* g_w1k, float* g_b1k,
                        float* g_w2k, float* g_b2k, float* loss, float* ws, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  if (g.B != 1) return fail(VEDA_ERR_UNSUPPORTED, "estimator gradient: only B == 1 layers are accepted");
  const float* w[8] = {w1q, b1q, w2q, b2q, w1k, b1k, w2k, b2k};
  float* gw[8] = {g_w1q, g_b1q, g_w2q, g_b2q, g_w1k, g_b1k, g_w2k, g_b2k};
  const char* wn[8] = {"w1q", "b1q", "w2q", "b2q", "w1k", "b1k", "w2k", "b2k"};
  const char* gn[8] = {"g_w1q", "g_b1q", "g_w2q", "g_b2q", "g_w1k", "g_b1k", "g_w2k", "g_b2k"};
  VEDA_TRY(check_ptr(dq, "dq"));
  VEDA_TRY(check_ptr(dk, "dk"));
  for (int i = 0; i < 8; ++i) {
    VEDA_TRY(check_ptr(w[i], wn[i]));
    VEDA_TRY(check_ptr(gw[i], gn[i]));
  }
  VEDA_TRY(check_ptr(tilemap, "tilemap"));
  VEDA_TRY(check_ptr(ws, "ws"));
  if (qtile_rows) VEDA_TRY(check_ptr(qtile_rows, "qtile_rows"));
  if (loss) VEDA_TRY(check_ptr(loss, "loss"));
  if (hidden < 4 || hidden > 256 || hidden % 4)
    return fail(VEDA_ERR_UNSUPPORTED, "hidden=%d must be a multiple of 4 in [4, 256]", hidden);
  if (out_dim < 4 || out_dim > 128 || out_dim % 4)
    return fail(VEDA_ERR_UNSUPPORTED, "out_dim=%d must be a multiple of 4 in [4, 128]", out_dim);
  if (!heads_sel || n_heads_sel < 1 || n_heads_sel > VEDA_MAX_HEADS)
    return fail(VEDA_ERR_INVALID_ARG, "heads_sel must list 1..%d heads", VEDA_MAX_HEADS);
  if (n_rows < 1 || n_rows > g.nt_cap) return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d outside [1, nt_cap]", n_rows);
  if (!(scale > 0.f) || scale != scale || scale > 3.0e38f)
    return fail(VEDA_ERR_INVALID_ARG, "scale must be positive and finite");
  for (int s = 0; s < n_heads_sel; ++s) {
    if (heads_sel[s] < 0 || heads_sel[s] >= g.heads)
      return fail(VEDA_ERR_INVALID_ARG, "heads_sel[%d]=%d outside [0, %d)", s, heads_sel[s], g.heads);
    for (int t = 0; t < s; ++t)
      if (heads_sel[t] == heads_sel[s]) return fail(VEDA_ERR_INVALID_ARG, "heads_sel lists head %d twice", heads_sel[s]);
    if (!qtile_rows && n_rows > g.h[heads_sel[s]].nt)
      return fail(VEDA_ERR_INVALID_ARG, "n_rows=%d exceeds the %d tiles of head %d", n_rows,
                  g.h[heads_sel[s]].nt, heads_sel[s]);
  }
  return after_launch(veda::launch_estimator_grad(g, dq, dk, w, gw, hidden, out_dim, scale, heads_sel, n_heads_sel,
                                                  qtile_rows, n_rows, tilemap, loss, ws, stream),
                      "veda_estimator_grad");
}

int veda_output_sq_error(const veda_layer* L, const void* a, const void* b, float* err, cudaStream_t stream) {
  veda::LayerGeom g;
  VEDA_TRY(build_geom(L, &g));
  VEDA_TRY(check_ptr(a, "a"));
  VEDA_TRY(check_ptr(b, "b"));
  VEDA_TRY(check_ptr(err, "err"));
  return after_launch(veda::launch_output_sq_error(g, a, b, err, stream), "veda_output_sq_error");
}

int veda_check_status(const veda_layer* L, cudaStream_t stream) {
  if (!L || !L->dev_status) return fail(VEDA_ERR_INVALID_ARG, "layer or dev_status is NULL");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_check_status: synchronize");
  int32_t v = 0;
  e = cudaMemcpy(&v, L->dev_status, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "veda_check_status: read");
  if (v != 0) {
    const int32_t zero = 0;
    e = cudaMemcpy(L->dev_status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "veda_check_status: clear");
    return fail(v, "device-side status %d (%s)", v,
                v == VEDA_ERR_TIMEOUT ? "a pipeline wait exceeded its limit"
                : v == VEDA_ERR_BAD_INDEX ? "a tile index was outside the head's range"
                                          : "error");
  }
  g_last_error.clear();
  return VEDA_OK;
}

}  // extern "C"

namespace veda {

// Records a message for veda_last_error() from code outside this file.
void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

}  // namespace veda
