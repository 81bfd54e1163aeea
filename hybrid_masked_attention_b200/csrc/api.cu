// extern "C" entry points of libmtfm: host-side argument checks, then launches.
// No allocation, no synchronisation (except mtfm_pack_check / mtfm_meta_read,
// which synchronise on purpose).  See include/mtfm.h for the contract.
#include <math.h>
#include <string.h>

#include "mtfm_internal.cuh"

using namespace mtfm;

namespace {

struct Resolved {
  int B, total_tokens, total_r, total_t, hq, hkv, dh, v2, D, Dkv;
  float alpha, eps;
};

mtfm_status resolve(const mtfm_cfg* c, Resolved* r) {
  if (!c) return MTFM_ERR_INVALID_ARG;
  if (c->batch < 0 || c->total_tokens < 0 || c->total_r < 0 || c->total_t < 0)
    return MTFM_ERR_INVALID_ARG;
  if (c->total_r + c->total_t > c->total_tokens) return MTFM_ERR_INVALID_ARG;
  if (c->hq <= 0 || c->hkv <= 0 || c->head_dim <= 0) return MTFM_ERR_INVALID_ARG;
  if (c->hq % c->hkv != 0) return MTFM_ERR_INVALID_ARG;
  if (c->v2_subtokens != 1 && c->v2_subtokens != 4) return MTFM_ERR_INVALID_ARG;
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256)
    return MTFM_ERR_UNSUPPORTED;
  if (c->hq / c->hkv > 8) return MTFM_ERR_UNSUPPORTED;
  const long long D = (long long)c->hq * c->head_dim;
  if (D > 1024 || D % 32 != 0) return MTFM_ERR_UNSUPPORTED;
  // Row offsets are int32 inside the kernels; element offsets are size_t.
  if ((long long)c->total_tokens * D > (1ll << 40)) return MTFM_ERR_UNSUPPORTED;
  r->B = c->batch;
  r->total_tokens = c->total_tokens;
  r->total_r = c->total_r;
  r->total_t = c->total_t;
  r->hq = c->hq;
  r->hkv = c->hkv;
  r->dh = c->head_dim;
  r->v2 = c->v2_subtokens;
  r->D = (int)D;
  r->Dkv = c->hkv * c->head_dim;
  r->alpha = c->alpha > 0.f ? c->alpha : 1.0f / sqrtf((float)c->head_dim);
  r->eps = c->gln_eps > 0.f ? c->gln_eps : 1e-5f;
  return MTFM_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline mtfm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MTFM_OK : MTFM_ERR_CUDA; }

mtfm_status check_meta(const void* d_meta, const Resolved& r) {
  if (!d_meta) return MTFM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_meta) & 255u) != 0) return MTFM_ERR_INVALID_ARG;
  return MTFM_OK;
}

// tcgen05/TMEM kernels where their TMEM plans fit (head_dim 64, r in {1, 2, 4}: the
// Target layer stacks the r heads of a group as MMA rows; head_dim 256: one head per
// unit, Full and Target layers); the mma.sync kernel covers the other head shapes.  A library compiled with
// -DMTFM_PORTABLE_KERNELS runs the mma.sync kernels for every shape (a test build
// for comparing the two; the shipped library has no run-time switch).
#ifdef MTFM_PORTABLE_KERNELS
constexpr bool kPortableOnly = true;
#else
constexpr bool kPortableOnly = false;
#endif
cudaError_t launch_attn(const Resolved& r, const MetaView& m, const MetaLayout& L, bool target,
                        const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                        float* a, cudaStream_t st) {
  AttnShape shape{r.hq, r.hkv, r.dh, r.v2, r.alpha, target};
  const int max_items = target ? L.max_items_target : L.max_items_full;
  const int rows = target ? r.total_t : r.total_tokens;
  if (!kPortableOnly && target && attn_fwd_tgt_supported(shape))
    return launch_attn_fwd_tgt(shape, m, max_items, rows, r.total_tokens, q, k, v, a, st);
  if (!kPortableOnly && !target && attn_fwd_tc_supported(shape))
    return launch_attn_fwd_tc(shape, m, max_items, rows, r.total_tokens, q, k, v, a, st);
  if (!kPortableOnly && attn_fwd_tc256_supported(shape))
    return launch_attn_fwd_tc256(shape, m, max_items, rows, r.total_tokens, q, k, v, a, st);
  return launch_attn_fwd_mma(shape, m, max_items, q, k, v, a, st);
}

// Attention only: A (fp32) for the Full or Target layout.
mtfm_status attn_only(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                      const uint16_t* d_k, const uint16_t* d_v, float* d_a, void* stream,
                      bool target) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  const int rows = target ? r.total_t : r.total_tokens;
  if (r.total_tokens == 0) return MTFM_OK;
  if (!d_k || !d_v) return MTFM_ERR_INVALID_ARG;
  if (rows > 0 && (!d_q || !d_a)) return MTFM_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_k) || !aligned16(d_v) || !aligned16(d_a))
    return MTFM_ERR_INVALID_ARG;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  const MetaView m = meta_view(const_cast<void*>(d_meta), L);
  return cuda_status(launch_attn(r, m, L, target, reinterpret_cast<const __nv_bfloat16*>(d_q),
                                 reinterpret_cast<const __nv_bfloat16*>(d_k),
                                 reinterpret_cast<const __nv_bfloat16*>(d_v), d_a,
                                 static_cast<cudaStream_t>(stream)));
}

// d_y: fp32, or bf16 (round to nearest) when y_bf16.
mtfm_status gate_fwd(const mtfm_cfg* cfg, const void* d_meta, bool target, const float* d_a,
                     const uint16_t* d_u, const float* d_gamma, const float* d_beta, void* d_y,
                     float* d_stats, void* stream, bool y_bf16 = false) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  const int rows = target ? r.total_t : r.total_tokens;
  if (rows == 0) return MTFM_OK;
  if (!d_a || !d_u || !d_y) return MTFM_ERR_INVALID_ARG;
  if ((d_gamma == nullptr) != (d_beta == nullptr)) return MTFM_ERR_INVALID_ARG;
  if (d_gamma && !d_stats) return MTFM_ERR_INVALID_ARG;
  if (!aligned16(d_a) || !aligned16(d_u) || !aligned16(d_y) ||
      (d_gamma && (!aligned16(d_gamma) || !aligned16(d_beta))) ||
      (d_stats && (reinterpret_cast<uintptr_t>(d_stats) & 7u)))
    return MTFM_ERR_INVALID_ARG;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  const MetaView m = meta_view(const_cast<void*>(d_meta), L);
  const __nv_bfloat16* u = reinterpret_cast<const __nv_bfloat16*>(d_u);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (y_bf16)
    return cuda_status(launch_gate_fwd_bf16(m, target, rows, r.D, r.eps, d_a, u, d_gamma, d_beta,
                                            static_cast<__nv_bfloat16*>(d_y), d_stats, st));
  return cuda_status(launch_gate_fwd(m, target, rows, r.D, r.eps, d_a, u, d_gamma, d_beta,
                                     static_cast<float*>(d_y), d_stats, st));
}

mtfm_status attn_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                     const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                     const float* d_gamma, const float* d_beta, void* d_y, float* d_a,
                     float* d_stats, void* stream, bool target, bool y_bf16 = false) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  const int rows = target ? r.total_t : r.total_tokens;
  // validate both halves before launching either
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  if (r.total_tokens == 0) return MTFM_OK;
  if (rows > 0 && (!d_u || !d_y)) return MTFM_ERR_INVALID_ARG;
  if ((d_gamma == nullptr) != (d_beta == nullptr)) return MTFM_ERR_INVALID_ARG;
  if (d_gamma && rows > 0 && !d_stats) return MTFM_ERR_INVALID_ARG;
  if (!aligned16(d_u) || !aligned16(d_y) || (d_gamma && (!aligned16(d_gamma) || !aligned16(d_beta))) ||
      (d_stats && (reinterpret_cast<uintptr_t>(d_stats) & 7u)))
    return MTFM_ERR_INVALID_ARG;
  s = attn_only(cfg, d_meta, d_q, d_k, d_v, d_a, stream, target);
  if (s != MTFM_OK) return s;
  return gate_fwd(cfg, d_meta, target, d_a, d_u, d_gamma, d_beta, d_y, d_stats, stream, y_bf16);
}

// Target attention over a cached K/V prefix (attention only): the tensor-core Target
// kernel with the prefix rows from the cache and the T rows' keys/values apart.
mtfm_status attn_target_cached(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                               const uint16_t* d_kp, const uint16_t* d_vp, const uint16_t* d_kc,
                               const uint16_t* d_vc, float* d_a, void* stream) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  AttnShape shape{r.hq, r.hkv, r.dh, r.v2, r.alpha, true};
  if (!attn_fwd_tgt_supported(shape) || kPortableOnly) return MTFM_ERR_UNSUPPORTED;
  if (r.total_t == 0 || r.total_tokens == 0) return MTFM_OK;
  const int prefix_rows = r.total_tokens - r.total_t;
  if (!d_q || !d_kc || !d_vc || !d_a) return MTFM_ERR_INVALID_ARG;
  if (prefix_rows > 0 && (!d_kp || !d_vp)) return MTFM_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_kc) || !aligned16(d_vc) || !aligned16(d_a) ||
      (prefix_rows > 0 && (!aligned16(d_kp) || !aligned16(d_vp))))
    return MTFM_ERR_INVALID_ARG;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  const MetaView m = meta_view(const_cast<void*>(d_meta), L);
  auto bf = [](const uint16_t* p) { return reinterpret_cast<const __nv_bfloat16*>(p); };
  return cuda_status(launch_attn_fwd_tgt(shape, m, L.max_items_target, r.total_t, r.total_tokens, bf(d_q),
                                         bf(d_kp), bf(d_vp), d_a, static_cast<cudaStream_t>(stream), bf(d_kc),
                                         bf(d_vc)));
}

// Scratch of the backward: dA as bf16 hi and lo parts [rows, D] each, then the
// per-block dgamma/dbeta partials.
struct BwdWs {
  size_t da_hi, da_lo, partials, total;
};
BwdWs bwd_ws(const Resolved& r, bool target) {
  BwdWs w;
  const int rows = target ? r.total_t : r.total_tokens;
  w.da_hi = 0;
  w.da_lo = align256(sizeof(uint16_t) * (size_t)rows * r.D);
  w.partials = w.da_lo + align256(sizeof(uint16_t) * (size_t)rows * r.D);
  w.total = align256(w.partials + sizeof(float) * 6 * (size_t)r.D * kGateBwdBlocks);
  return w;
}

mtfm_status attn_bwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                     const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                     const float* d_gamma, const float* d_beta, const float* d_a,
                     const float* d_stats, const uint16_t* d_dy, float* d_dq, float* d_dk,
                     float* d_dv, float* d_du, float* d_dgamma, float* d_dbeta, void* d_ws,
                     size_t ws_bytes, void* stream, bool target) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  if (r.total_tokens == 0) return MTFM_OK;
  const int rows = target ? r.total_t : r.total_tokens;
  if (!d_k || !d_v || !d_dk || !d_dv || !d_ws) return MTFM_ERR_INVALID_ARG;
  if (rows > 0 && (!d_q || !d_u || !d_a || !d_dy || !d_dq || !d_du)) return MTFM_ERR_INVALID_ARG;
  const bool gln = d_gamma != nullptr;
  if ((d_beta != nullptr) != gln || (d_dgamma != nullptr) != gln || (d_dbeta != nullptr) != gln)
    return MTFM_ERR_INVALID_ARG;
  if (gln && rows > 0 && !d_stats) return MTFM_ERR_INVALID_ARG;
  const void* ptrs[] = {d_q, d_k, d_v, d_u, d_a, d_dy, d_dq, d_dk, d_dv, d_du, d_ws};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MTFM_ERR_INVALID_ARG;
  const BwdWs w = bwd_ws(r, target);
  if (ws_bytes < w.total) return MTFM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  const MetaView m = meta_view(const_cast<void*>(d_meta), L);
  char* ws = static_cast<char*>(d_ws);
  __nv_bfloat16* da_hi = reinterpret_cast<__nv_bfloat16*>(ws + w.da_hi);
  __nv_bfloat16* da_lo = reinterpret_cast<__nv_bfloat16*>(ws + w.da_lo);
  float* partials = reinterpret_cast<float*>(ws + w.partials);
  cudaError_t e = cudaSuccess;
  if (rows > 0) {
    e = cudaMemsetAsync(d_dq, 0, sizeof(float) * (size_t)rows * r.D, st);
    if (e != cudaSuccess) return MTFM_ERR_CUDA;
  }
  e = launch_gate_bwd(m, target, rows, r.D, r.eps, d_a, d_stats,
                      reinterpret_cast<const __nv_bfloat16*>(d_u),
                      reinterpret_cast<const __nv_bfloat16*>(d_dy), d_gamma, d_beta, d_du, da_hi,
                      da_lo, partials, kGateBwdBlocks, d_dgamma, d_dbeta, st);
  if (e != cudaSuccess) return MTFM_ERR_CUDA;
  AttnShape shape{r.hq, r.hkv, r.dh, r.v2, r.alpha, target};
  // tcgen05 kernel for head_dim 64; the mma.sync kernel for the other head sizes
  // (and for every shape in a -DMTFM_PORTABLE_KERNELS test build).
  if (!kPortableOnly && attn_bwd_tc_supported(shape)) {
    e = launch_attn_bwd_tc(shape, m, L.max_items_full, rows, r.total_tokens,
                           reinterpret_cast<const __nv_bfloat16*>(d_q), reinterpret_cast<const __nv_bfloat16*>(d_k),
                           reinterpret_cast<const __nv_bfloat16*>(d_v), da_hi, da_lo, d_dq, d_dk, d_dv, st);
    return cuda_status(e);
  }
  e = launch_attn_bwd_mma(shape, m, L.max_items_full, reinterpret_cast<const __nv_bfloat16*>(d_q),
                          reinterpret_cast<const __nv_bfloat16*>(d_k),
                          reinterpret_cast<const __nv_bfloat16*>(d_v), da_hi, da_lo, d_dq, d_dk,
                          d_dv, st);
  return cuda_status(e);
}


// ------------------------------------------------------------------ backbone stack
// Scratch of one layer, reused by every layer of a stack: X~ (all rows) and
// X~_T (T rows) in bf16; U, Q (rows of the layer's queries), K, V in bf16; A in
// fp32; Y in bf16; GLN row statistics.
struct StackWs {
  size_t xn, xnt, u, q, k, v, a, y, stats, total;
};
StackWs stack_ws(const Resolved& r, int d) {
  StackWs w;
  const size_t N = (size_t)r.total_tokens, T = (size_t)r.total_t;
  size_t o = 0;
  w.xn = o;    o = align256(o + N * d * 2);
  w.xnt = o;   o = align256(o + T * d * 2);
  w.u = o;     o = align256(o + N * r.D * 2);
  w.q = o;     o = align256(o + N * r.D * 2);
  w.k = o;     o = align256(o + N * r.Dkv * 2);
  w.v = o;     o = align256(o + N * r.Dkv * 2);
  w.a = o;     o = align256(o + N * r.D * 4);
  w.y = o;     o = align256(o + N * r.D * 2);
  w.stats = o; o = align256(o + N * 2 * 4);
  w.total = o;
  return w;
}

// Shapes the stack kernels take: d_model and hq*head_dim multiples of 64
// (GEMM tiles), d_model <= 1024 (RMSNorm keeps a row in registers).
mtfm_status check_stack_cfg(const Resolved& r, int d) {
  if (d <= 0 || d % 64 != 0) return MTFM_ERR_INVALID_ARG;
  if (d > 1024 || r.D % 64 != 0) return MTFM_ERR_UNSUPPORTED;
  return MTFM_OK;
}

mtfm_status check_layer_weights(const Resolved& r, const mtfm_layer_weights* w, bool target) {
  if (!w || !w->rms_w || !w->w_in || !w->w_o) return MTFM_ERR_INVALID_ARG;
  if (target != (w->w_kv != nullptr)) return MTFM_ERR_INVALID_ARG;
  if ((w->gamma == nullptr) != (w->beta == nullptr)) return MTFM_ERR_INVALID_ARG;
  if (!aligned16(w->rms_w) || !aligned16(w->w_in) || !aligned16(w->w_o) ||
      (w->w_kv && !aligned16(w->w_kv)) || (w->gamma && (!aligned16(w->gamma) || !aligned16(w->beta))))
    return MTFM_ERR_INVALID_ARG;
  return MTFM_OK;
}

// One layer, all launches on `st`; arguments already checked.
cudaError_t layer_fwd(const Resolved& r, const MetaView& m, const MetaLayout& L, int d, bool target,
                      const mtfm_layer_weights& w, float* x, char* ws, const StackWs& W,
                      cudaStream_t st) {
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  auto wt = [](const uint16_t* p) { return reinterpret_cast<const __nv_bfloat16*>(p); };
  const int N = r.total_tokens, T = r.total_t, D = r.D, Dkv = r.Dkv;
  const int rows_q = target ? T : N;
  cudaError_t e;
  // X~ = RMSNorm(X) for every row (K, V read all rows); X~_T gathered for a Target layer
  if ((e = launch_rmsnorm(m.hdr, x, N, d, nullptr, w.rms_w, kRmsEps, bf(W.xn), st)) != cudaSuccess) return e;
  if (target && (e = launch_rmsnorm(m.hdr, x, T, d, m.t_rows, w.rms_w, kRmsEps, bf(W.xnt), st)) != cudaSuccess)
    return e;
  if (!target) {
    // [U Q K V] = SiLU(X~ W_uqkv^T)
    GemmEpi g{kEpiSiluSplit, 4, {0, D, 2 * D, 2 * D + Dkv, 2 * D + 2 * Dkv},
              {bf(W.u), bf(W.q), bf(W.k), bf(W.v)}, {D, D, Dkv, Dkv}, nullptr, 0, nullptr};
    if ((e = launch_gemm_tc(m.hdr, bf(W.xn), d, wt(w.w_in), N, 2 * D + 2 * Dkv, d, g, st)) != cudaSuccess)
      return e;
  } else {
    // [U Q]_T = SiLU(X~_T W_uq^T), [K V] = SiLU(X~ W_kv^T)
    GemmEpi guq{kEpiSiluSplit, 2, {0, D, 2 * D, 0, 0}, {bf(W.u), bf(W.q), nullptr, nullptr}, {D, D, 0, 0},
                nullptr, 0, nullptr};
    if ((e = launch_gemm_tc(m.hdr, bf(W.xnt), d, wt(w.w_in), T, 2 * D, d, guq, st)) != cudaSuccess) return e;
    GemmEpi gkv{kEpiSiluSplit, 2, {0, Dkv, 2 * Dkv, 0, 0}, {bf(W.k), bf(W.v), nullptr, nullptr},
                {Dkv, Dkv, 0, 0}, nullptr, 0, nullptr};
    if ((e = launch_gemm_tc(m.hdr, bf(W.xn), d, wt(w.w_kv), N, 2 * Dkv, d, gkv, st)) != cudaSuccess) return e;
  }
  float* a = reinterpret_cast<float*>(ws + W.a);
  if ((e = launch_attn(r, m, L, target, bf(W.q), bf(W.k), bf(W.v), a, st)) != cudaSuccess) return e;
  if ((e = launch_gate_fwd_bf16(m, target, rows_q, D, r.eps, a, bf(W.u), w.gamma, w.beta, bf(W.y),
                                reinterpret_cast<float*>(ws + W.stats), st)) != cudaSuccess)
    return e;
  // X (+)= Y W_o^T, scattered back to the T rows for a Target layer
  GemmEpi go{kEpiResidual, 0, {0, 0, 0, 0, 0}, {nullptr, nullptr, nullptr, nullptr}, {0, 0, 0, 0}, x, d,
             target ? m.t_rows : nullptr};
  return launch_gemm_tc(m.hdr, bf(W.y), D, wt(w.w_o), rows_q, d, D, go, st);
}

mtfm_status stack_fwd(const mtfm_cfg* cfg, const void* d_meta, int d, int n_layers, const char* kinds,
                      const mtfm_layer_weights* layers, float* d_x, void* d_ws, size_t ws_bytes,
                      void* stream) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  if ((s = check_stack_cfg(r, d)) != MTFM_OK) return s;
  if (n_layers < 0 || (n_layers > 0 && (!kinds || !layers))) return MTFM_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    if (kinds[l] != 'F' && kinds[l] != 'T') return MTFM_ERR_INVALID_ARG;
    if ((s = check_layer_weights(r, &layers[l], kinds[l] == 'T')) != MTFM_OK) return s;
  }
  if (n_layers == 0 || r.total_tokens == 0) return MTFM_OK;
  const StackWs W = stack_ws(r, d);
  if (!d_x || !aligned16(d_x)) return MTFM_ERR_INVALID_ARG;
  if (!d_ws || (reinterpret_cast<uintptr_t>(d_ws) & 255u)) return MTFM_ERR_INVALID_ARG;
  if (ws_bytes < W.total) return MTFM_ERR_WORKSPACE_TOO_SMALL;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  const MetaView m = meta_view(const_cast<void*>(d_meta), L);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int l = 0; l < n_layers; ++l) {
    cudaError_t e = layer_fwd(r, m, L, d, kinds[l] == 'T', layers[l], d_x, static_cast<char*>(d_ws), W, st);
    if (e != cudaSuccess) return MTFM_ERR_CUDA;
  }
  return MTFM_OK;
}

// ------------------------------------------------------------------ V2 Target layer
// Scratch: the stack's layer scratch, then the FFN's pre-normed input X~2_T (bf16
// [T, d]) and hidden layer H (bf16 [T, d_ff]).
struct V2Ws {
  StackWs base;
  size_t xn2, hid, total;
};
V2Ws v2_ws(const Resolved& r, int d, int dff) {
  V2Ws w;
  w.base = stack_ws(r, d);
  const size_t T = (size_t)r.total_t;
  size_t o = w.base.total;
  w.xn2 = o; o = align256(o + T * d * 2);
  w.hid = o; o = align256(o + T * dff * 2);
  w.total = o;
  return w;
}

mtfm_status check_v2(const Resolved& r, int d, int dff) {
  mtfm_status s = check_stack_cfg(r, d);
  if (s != MTFM_OK) return s;
  if (r.v2 != 4) return MTFM_ERR_INVALID_ARG;
  if (dff <= 0 || dff % 64 != 0) return MTFM_ERR_INVALID_ARG;
  if (r.total_t % 4 != 0) return MTFM_ERR_INVALID_ARG;
  return MTFM_OK;
}

mtfm_status v2_layer_fwd(const mtfm_cfg* cfg, const void* d_meta, int d, int dff, const mtfm_v2_layer_weights* w,
                         float* x, void* d_ws, size_t ws_bytes, void* stream) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  if ((s = check_v2(r, d, dff)) != MTFM_OK) return s;
  if (!w || !w->rms_w || !w->w_kv || !w->w_o || !w->rms_w2) return MTFM_ERR_INVALID_ARG;
  if ((w->gamma == nullptr) != (w->beta == nullptr)) return MTFM_ERR_INVALID_ARG;
  const void* ptrs[] = {w->rms_w, w->w_kv, w->w_o, w->rms_w2};
  for (const void* q : ptrs)
    if (!aligned16(q)) return MTFM_ERR_INVALID_ARG;
  if (w->gamma && (!aligned16(w->gamma) || !aligned16(w->beta))) return MTFM_ERR_INVALID_ARG;
  for (int k = 0; k < 4; ++k)
    if (!w->w_uq[k] || !w->w_gate[k] || !w->w_up[k] || !w->w_down[k] || !aligned16(w->w_uq[k]) ||
        !aligned16(w->w_gate[k]) || !aligned16(w->w_up[k]) || !aligned16(w->w_down[k]))
      return MTFM_ERR_INVALID_ARG;
  if (r.total_tokens == 0 || r.total_t == 0) return MTFM_OK;  // no target: X unchanged
  if (!x || !aligned16(x)) return MTFM_ERR_INVALID_ARG;
  if (!d_ws || (reinterpret_cast<uintptr_t>(d_ws) & 255u)) return MTFM_ERR_INVALID_ARG;
  const V2Ws V = v2_ws(r, d, dff);
  const StackWs& W = V.base;
  if (ws_bytes < V.total) return MTFM_ERR_WORKSPACE_TOO_SMALL;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  const MetaView m = meta_view(const_cast<void*>(d_meta), L);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(d_ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  auto wt = [](const uint16_t* q) { return reinterpret_cast<const __nv_bfloat16*>(q); };
  const int N = r.total_tokens, T = r.total_t, D = r.D, Dkv = r.Dkv, T4 = T / 4;
  cudaError_t e;
  // attention block: X~ on all rows (K, V) and on the T rows (the sub-tokens' [U Q])
  if ((e = launch_rmsnorm(m.hdr, x, N, d, nullptr, w->rms_w, kRmsEps, bf(W.xn), st)) != cudaSuccess) return MTFM_ERR_CUDA;
  if ((e = launch_rmsnorm(m.hdr, x, T, d, m.t_rows, w->rms_w, kRmsEps, bf(W.xnt), st)) != cudaSuccess)
    return MTFM_ERR_CUDA;
  GemmEpi gkv{kEpiSiluSplit, 2, {0, Dkv, 2 * Dkv, 0, 0}, {bf(W.k), bf(W.v), nullptr, nullptr}, {Dkv, Dkv, 0, 0},
              nullptr, 0, nullptr, 0, nullptr};
  if ((e = launch_gemm_tc(m.hdr, bf(W.xn), d, wt(w->w_kv), N, 2 * Dkv, d, gkv, st)) != cudaSuccess)
    return MTFM_ERR_CUDA;
  // sub-token position s of every target is T row 4 i + s (L_T is a multiple of 4 per user,
  // so targets start at multiples of 4): strided operands select the rows of one position
  for (int k = 0; k < 4; ++k) {
    GemmEpi guq{kEpiSiluSplit, 2, {0, D, 2 * D, 0, 0}, {bf(W.u) + (size_t)k * D, bf(W.q) + (size_t)k * D, nullptr, nullptr},
                {4 * D, 4 * D, 0, 0}, nullptr, 0, nullptr, 0, nullptr};
    if ((e = launch_gemm_tc(m.hdr, bf(W.xnt) + (size_t)k * d, 4 * d, wt(w->w_uq[k]), T4, 2 * D, d, guq, st)) !=
        cudaSuccess)
      return MTFM_ERR_CUDA;
  }
  float* a = reinterpret_cast<float*>(ws + W.a);
  if ((e = launch_attn(r, m, L, true, bf(W.q), bf(W.k), bf(W.v), a, st)) != cudaSuccess) return MTFM_ERR_CUDA;
  if ((e = launch_gate_fwd_bf16(m, true, T, D, r.eps, a, bf(W.u), w->gamma, w->beta, bf(W.y),
                                reinterpret_cast<float*>(ws + W.stats), st)) != cudaSuccess)
    return MTFM_ERR_CUDA;
  GemmEpi go{kEpiResidual, 0, {0, 0, 0, 0, 0}, {nullptr, nullptr, nullptr, nullptr}, {0, 0, 0, 0}, x, d, m.t_rows,
             1, nullptr};
  if ((e = launch_gemm_tc(m.hdr, bf(W.y), D, wt(w->w_o), T, d, D, go, st)) != cudaSuccess) return MTFM_ERR_CUDA;
  // mixing of each target's sub-tokens (in place on X), then the FFN's pre-norm
  if ((e = launch_mix_rmsnorm(m.hdr, x, T4, d, m.t_rows, w->rms_w2, kRmsEps, bf(V.xn2), st)) != cudaSuccess)
    return MTFM_ERR_CUDA;
  // per-sub-token SwiGLU FFN with the residual
  for (int k = 0; k < 4; ++k) {
    GemmEpi gup{kEpiSwiGLU, 1, {0, 2 * dff, 0, 0, 0}, {bf(V.hid) + (size_t)k * dff, nullptr, nullptr, nullptr},
                {4 * dff, 0, 0, 0}, nullptr, 0, nullptr, 0, wt(w->w_up[k])};
    if ((e = launch_gemm_tc(m.hdr, bf(V.xn2) + (size_t)k * d, 4 * d, wt(w->w_gate[k]), T4, 2 * dff, d, gup, st)) !=
        cudaSuccess)
      return MTFM_ERR_CUDA;
    GemmEpi gdn{kEpiResidual, 0, {0, 0, 0, 0, 0}, {nullptr, nullptr, nullptr, nullptr}, {0, 0, 0, 0}, x, d,
                m.t_rows + k, 4, nullptr};
    if ((e = launch_gemm_tc(m.hdr, bf(V.hid) + (size_t)k * dff, 4 * dff, wt(w->w_down[k]), T4, d, dff, gdn, st)) !=
        cudaSuccess)
      return MTFM_ERR_CUDA;
  }
  return MTFM_OK;
}

}  // namespace

extern "C" {

const char* mtfm_status_string(mtfm_status s) {
  switch (s) {
    case MTFM_OK: return "ok";
    case MTFM_ERR_INVALID_ARG: return "invalid argument";
    case MTFM_ERR_UNSORTED_TS: return "R timestamps not ascending within a user";
    case MTFM_ERR_UNSUPPORTED: return "unsupported shape";
    case MTFM_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MTFM_ERR_CUDA: return "CUDA runtime error";
    case MTFM_ERR_TIMEOUT: return "device wait timed out";
    case MTFM_ERR_BAD_LENGTHS: return "lengths negative, inconsistent with totals, or L_T not a multiple of v2_subtokens";
    case MTFM_ERR_BOUNDS: return "a bounds check of the bounds-checked build failed";
  }
  return "unknown status";
}

size_t mtfm_meta_bytes(const mtfm_cfg* cfg) {
  Resolved r;
  if (resolve(cfg, &r) != MTFM_OK) return 0;
  return meta_layout(r.B, r.total_tokens, r.total_t).total;
}

mtfm_status mtfm_pack(const mtfm_cfg* cfg, const int32_t* d_lh, const int32_t* d_lr,
                      const int32_t* d_lt, const int64_t* d_r_ts, const int64_t* d_t_exp,
                      void* d_meta, size_t meta_bytes, void* stream) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  if (meta_bytes < L.total) return MTFM_ERR_WORKSPACE_TOO_SMALL;
  if (r.B > 0 && (!d_lh || !d_lr || !d_lt)) return MTFM_ERR_INVALID_ARG;
  if (r.total_r > 0 && !d_r_ts) return MTFM_ERR_INVALID_ARG;
  if (r.total_t > 0 && !d_t_exp) return MTFM_ERR_INVALID_ARG;
  const MetaView m = meta_view(d_meta, L);
  return cuda_status(launch_pack(*cfg, m, d_lh, d_lr, d_lt, d_r_ts, d_t_exp,
                                 static_cast<cudaStream_t>(stream)));
}

mtfm_status mtfm_pack_check(const void* d_meta, void* stream) {
  if (!d_meta) return MTFM_ERR_INVALID_ARG;
  MetaHeader h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, d_meta, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MTFM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MTFM_ERR_CUDA;
  if (h.magic != kMetaMagic) return MTFM_ERR_INVALID_ARG;
  if (h.error & kErrBadLengths) return MTFM_ERR_BAD_LENGTHS;
  if (h.error & kErrUnsorted) return MTFM_ERR_UNSORTED_TS;
  if (h.error & kErrBounds) return MTFM_ERR_BOUNDS;
  if (h.error & kErrTimeout) return MTFM_ERR_TIMEOUT;
  if (h.error & kErrConfig) return MTFM_ERR_UNSUPPORTED;
  return MTFM_OK;
}

int32_t mtfm_debug_bounds_build(void) {
#ifdef MTFM_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

mtfm_status mtfm_debug_site(const void* d_meta, int32_t* site, void* stream) {
  if (!d_meta || !site) return MTFM_ERR_INVALID_ARG;
  MetaHeader h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, d_meta, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MTFM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MTFM_ERR_CUDA;
  if (h.magic != kMetaMagic) return MTFM_ERR_INVALID_ARG;
  *site = h.dbg_site;
  return MTFM_OK;
}

mtfm_status mtfm_meta_read(const mtfm_cfg* cfg, const void* d_meta, int32_t* seq_off,
                           int32_t* r_off, int32_t* t_off, int32_t* kv_end, uint8_t* row_type,
                           int32_t* n_items_full, int32_t* n_items_target, int32_t* items_full,
                           int32_t* items_target, void* stream) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  if ((s = check_meta(d_meta, r)) != MTFM_OK) return s;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const char* b = static_cast<const char*>(d_meta);
  MetaHeader h;
  struct Cp { void* dst; size_t off, bytes; } cps[] = {
      {&h, 0, sizeof(h)},
      {seq_off, L.seq_off, sizeof(int32_t) * (size_t)(r.B + 1)},
      {r_off, L.r_off, sizeof(int32_t) * (size_t)(r.B + 1)},
      {t_off, L.t_off, sizeof(int32_t) * (size_t)(r.B + 1)},
      {kv_end, L.kv_end, sizeof(int32_t) * (size_t)r.total_tokens},
      {row_type, L.row_type, (size_t)r.total_tokens},
      {items_full, L.items_full, sizeof(WorkItem) * (size_t)L.max_items_full},
      {items_target, L.items_target, sizeof(WorkItem) * (size_t)L.max_items_target},
  };
  for (const Cp& c : cps) {
    if (!c.dst || c.bytes == 0) continue;
    if (cudaMemcpyAsync(c.dst, b + c.off, c.bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return MTFM_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return MTFM_ERR_CUDA;
  if (n_items_full) *n_items_full = h.n_items_full;
  if (n_items_target) *n_items_target = h.n_items_target;
  return MTFM_OK;
}

mtfm_status mtfm_attn_full_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                               const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                               const float* d_gamma, const float* d_beta, float* d_y, float* d_a,
                               float* d_stats, void* stream) {
  return attn_fwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_y, d_a, d_stats, stream,
                  false);
}

mtfm_status mtfm_attn_target_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                 const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                 const float* d_gamma, const float* d_beta, float* d_y,
                                 float* d_a, float* d_stats, void* stream) {
  return attn_fwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_y, d_a, d_stats, stream,
                  true);
}

mtfm_status mtfm_attn_full_fwd_bf16y(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                     const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                     const float* d_gamma, const float* d_beta, uint16_t* d_y, float* d_a,
                                     float* d_stats, void* stream) {
  return attn_fwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_y, d_a, d_stats, stream,
                  false, true);
}

mtfm_status mtfm_attn_target_fwd_bf16y(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                       const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                       const float* d_gamma, const float* d_beta, uint16_t* d_y,
                                       float* d_a, float* d_stats, void* stream) {
  return attn_fwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_y, d_a, d_stats, stream,
                  true, true);
}

mtfm_status mtfm_attn_target_cached_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                        const uint16_t* d_k_prefix, const uint16_t* d_v_prefix,
                                        const uint16_t* d_k_cand, const uint16_t* d_v_cand,
                                        const uint16_t* d_u, const float* d_gamma, const float* d_beta,
                                        float* d_y, float* d_a, float* d_stats, void* stream) {
  Resolved r;
  mtfm_status s = resolve(cfg, &r);
  if (s != MTFM_OK) return s;
  // the gate's arguments are checked before the attention launches
  if (r.total_t > 0) {
    if (!d_u || !d_y) return MTFM_ERR_INVALID_ARG;
    if ((d_gamma == nullptr) != (d_beta == nullptr)) return MTFM_ERR_INVALID_ARG;
    if (d_gamma && !d_stats) return MTFM_ERR_INVALID_ARG;
    if (!aligned16(d_u) || !aligned16(d_y) || (d_gamma && (!aligned16(d_gamma) || !aligned16(d_beta))) ||
        (d_stats && (reinterpret_cast<uintptr_t>(d_stats) & 7u)))
      return MTFM_ERR_INVALID_ARG;
  }
  s = attn_target_cached(cfg, d_meta, d_q, d_k_prefix, d_v_prefix, d_k_cand, d_v_cand, d_a, stream);
  if (s != MTFM_OK || r.total_t == 0 || r.total_tokens == 0) return s;
  return gate_fwd(cfg, d_meta, true, d_a, d_u, d_gamma, d_beta, d_y, d_stats, stream);
}

mtfm_status mtfm_attn_target_cached(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                    const uint16_t* d_k_prefix, const uint16_t* d_v_prefix,
                                    const uint16_t* d_k_cand, const uint16_t* d_v_cand, float* d_a,
                                    void* stream) {
  return attn_target_cached(cfg, d_meta, d_q, d_k_prefix, d_v_prefix, d_k_cand, d_v_cand, d_a, stream);
}

int32_t mtfm_max_items(const mtfm_cfg* cfg, int is_target) {
  Resolved r;
  if (resolve(cfg, &r) != MTFM_OK) return -1;
  const MetaLayout L = meta_layout(r.B, r.total_tokens, r.total_t);
  return is_target ? L.max_items_target : L.max_items_full;
}

mtfm_status mtfm_attn_full(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                           const uint16_t* d_k, const uint16_t* d_v, float* d_a, void* stream) {
  return attn_only(cfg, d_meta, d_q, d_k, d_v, d_a, stream, false);
}

mtfm_status mtfm_attn_target(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                             const uint16_t* d_k, const uint16_t* d_v, float* d_a, void* stream) {
  return attn_only(cfg, d_meta, d_q, d_k, d_v, d_a, stream, true);
}

mtfm_status mtfm_gate_fwd(const mtfm_cfg* cfg, const void* d_meta, int is_target, const float* d_a,
                          const uint16_t* d_u, const float* d_gamma, const float* d_beta,
                          float* d_y, float* d_stats, void* stream) {
  return gate_fwd(cfg, d_meta, is_target != 0, d_a, d_u, d_gamma, d_beta, d_y, d_stats, stream);
}

size_t mtfm_bwd_workspace_bytes(const mtfm_cfg* cfg, int is_target) {
  Resolved r;
  if (resolve(cfg, &r) != MTFM_OK) return 0;
  return bwd_ws(r, is_target != 0).total;
}

mtfm_status mtfm_attn_full_bwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                               const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                               const float* d_gamma, const float* d_beta, const float* d_a,
                               const float* d_stats, const uint16_t* d_dy, float* d_dq,
                               float* d_dk, float* d_dv, float* d_du, float* d_dgamma,
                               float* d_dbeta, void* d_ws, size_t ws_bytes, void* stream) {
  return attn_bwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_a, d_stats, d_dy, d_dq,
                  d_dk, d_dv, d_du, d_dgamma, d_dbeta, d_ws, ws_bytes, stream, false);
}

mtfm_status mtfm_attn_target_bwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                 const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                 const float* d_gamma, const float* d_beta, const float* d_a,
                                 const float* d_stats, const uint16_t* d_dy, float* d_dq,
                                 float* d_dk, float* d_dv, float* d_du, float* d_dgamma,
                                 float* d_dbeta, void* d_ws, size_t ws_bytes, void* stream) {
  return attn_bwd(cfg, d_meta, d_q, d_k, d_v, d_u, d_gamma, d_beta, d_a, d_stats, d_dy, d_dq,
                  d_dk, d_dv, d_du, d_dgamma, d_dbeta, d_ws, ws_bytes, stream, true);
}

size_t mtfm_stack_workspace_bytes(const mtfm_cfg* cfg, int32_t d_model) {
  Resolved r;
  if (resolve(cfg, &r) != MTFM_OK || check_stack_cfg(r, d_model) != MTFM_OK) return 0;
  return stack_ws(r, d_model).total;
}

mtfm_status mtfm_layer_fwd(const mtfm_cfg* cfg, const void* d_meta, int32_t d_model, int is_target,
                           const mtfm_layer_weights* weights, float* d_x, void* d_ws, size_t ws_bytes,
                           void* stream) {
  const char kind = is_target ? 'T' : 'F';
  return stack_fwd(cfg, d_meta, d_model, 1, &kind, weights, d_x, d_ws, ws_bytes, stream);
}

mtfm_status mtfm_stack_fwd(const mtfm_cfg* cfg, const void* d_meta, int32_t d_model, int32_t n_layers,
                           const char* kinds, const mtfm_layer_weights* layers, float* d_x, void* d_ws,
                           size_t ws_bytes, void* stream) {
  return stack_fwd(cfg, d_meta, d_model, n_layers, kinds, layers, d_x, d_ws, ws_bytes, stream);
}

size_t mtfm_v2_workspace_bytes(const mtfm_cfg* cfg, int32_t d_model, int32_t d_ff) {
  Resolved r;
  if (resolve(cfg, &r) != MTFM_OK || check_v2(r, d_model, d_ff) != MTFM_OK) return 0;
  return v2_ws(r, d_model, d_ff).total;
}

mtfm_status mtfm_v2_target_layer_fwd(const mtfm_cfg* cfg, const void* d_meta, int32_t d_model, int32_t d_ff,
                                     const mtfm_v2_layer_weights* weights, float* d_x, void* d_ws, size_t ws_bytes,
                                     void* stream) {
  return v2_layer_fwd(cfg, d_meta, d_model, d_ff, weights, d_x, d_ws, ws_bytes, stream);
}

mtfm_status mtfm_selftest_wait_timeout(void* d_meta, int64_t limit_cycles, void* stream) {
  if (!d_meta || (reinterpret_cast<uintptr_t>(d_meta) & 255u) != 0) return MTFM_ERR_INVALID_ARG;
  if (limit_cycles <= 0 || limit_cycles > 4000000000ll) return MTFM_ERR_INVALID_ARG;
  return cuda_status(launch_wait_timeout(static_cast<MetaHeader*>(d_meta), (long long)limit_cycles,
                                         static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
