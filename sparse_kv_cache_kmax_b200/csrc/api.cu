// Host side of the C ABI declared in include/ekv.h: argument validation
// (before any launch), workspace sizing and carving, and kernel dispatch.
#include <math.h>

#include "kernels.cuh"

namespace ekv {

__device__ unsigned int g_error_flags = 0u;

namespace {

inline size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Carver {
  char* base;
  size_t used = 0;
  template <typename V>
  V* take(size_t count) {
    V* p = reinterpret_cast<V*>(base + used);
    used += a256(count * sizeof(V));
    return p;
  }
};

bool pow2_group(int G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }

ekv_status check_cache(const ekv_cache* c, bool need_v, bool need_meta) {
  if (c == nullptr) return EKV_ERR_INVALID_ARG;
  if (c->dtype != EKV_F32 && c->dtype != EKV_BF16) return EKV_ERR_UNSUPPORTED;
  if (c->num_kv_heads < 1 || c->num_phys_pages < 1 || c->head_dim < 1 || c->page_size < 1)
    return EKV_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return EKV_ERR_UNSUPPORTED;
  if (c->page_size != 16 && c->page_size != 32) return EKV_ERR_UNSUPPORTED;
  if (c->k_pool == nullptr) return EKV_ERR_INVALID_ARG;
  if (need_v && c->v_pool == nullptr) return EKV_ERR_INVALID_ARG;
  if (need_meta && (c->box == nullptr || c->mom == nullptr)) return EKV_ERR_INVALID_ARG;
  return EKV_OK;
}

ekv_status check_seqs(const ekv_seqs* s) {
  if (s == nullptr || s->page_table == nullptr || s->seq_lens == nullptr) return EKV_ERR_INVALID_ARG;
  if (s->batch < 1 || s->max_pages < 1) return EKV_ERR_INVALID_ARG;
  return EKV_OK;
}

ekv_status check_heads(const ekv_cache* c, int Hq) {
  if (Hq < 1 || Hq % c->num_kv_heads != 0) return EKV_ERR_INVALID_ARG;
  const int G = Hq / c->num_kv_heads;
  if (!pow2_group(G)) return EKV_ERR_UNSUPPORTED;
  return EKV_OK;
}

bool finite_pos(float x) { return isfinite(x) && x > 0.0f; }

ekv_status check_alpha(float alpha) {
  if (!isfinite(alpha) || !(alpha > 1.0f)) return EKV_ERR_INVALID_ARG;
  return EKV_OK;
}

int gauss_beta(float alpha) {
  const double b = 1.0 / (static_cast<double>(alpha) - 1.0);
  const double r = nearbyint(b);
  if (fabs(b - r) > 1e-6 || r < 1.0 || r > 4.0) return 0;
  return static_cast<int>(r);
}

size_t gauss_ws_bytes(const ekv_cache* c, const ekv_seqs* s, int Hq) {
  const size_t U = static_cast<size_t>(s->batch) * c->num_kv_heads;
  const size_t G = static_cast<size_t>(Hq / c->num_kv_heads);
  const size_t rows = U * G * static_cast<size_t>(s->max_pages);
  const size_t nch = U * static_cast<size_t>(filter_chunks(s->max_pages));
  return 3 * a256(rows * sizeof(float)) + a256(U * G * sizeof(double)) + a256(nch * sizeof(int)) +
         a256(nch * sizeof(double)) + a256(nch * sizeof(int));
}

GaussWs carve_gauss(Carver& cv, const ekv_cache* c, const ekv_seqs* s, int Hq) {
  const size_t U = static_cast<size_t>(s->batch) * c->num_kv_heads;
  const size_t G = static_cast<size_t>(Hq / c->num_kv_heads);
  const size_t rows = U * G * static_cast<size_t>(s->max_pages);
  GaussWs w;
  w.mu = cv.take<float>(rows);
  w.sig = cv.take<float>(rows);
  w.hat = cv.take<float>(rows);
  w.tau_hat = cv.take<double>(U * G);
  w.nchunk = filter_chunks(s->max_pages);
  w.fcount = cv.take<int>(U * static_cast<size_t>(w.nchunk));
  w.fbest = cv.take<double>(U * static_cast<size_t>(w.nchunk));
  w.fbest_at = cv.take<int>(U * static_cast<size_t>(w.nchunk));
  return w;
}

size_t decode_ws_bytes(const ekv_cache* c, const ekv_seqs* s, int Hq, int cap) {
  const size_t U = static_cast<size_t>(s->batch) * c->num_kv_heads;
  const size_t G = static_cast<size_t>(Hq / c->num_kv_heads);
  const size_t nqk = static_cast<size_t>(qk_splits(cap, c->page_size));
  const size_t npv = static_cast<size_t>(pv_splits(static_cast<int>(U), cap));
  const size_t S = static_cast<size_t>(c->page_size), D = static_cast<size_t>(c->head_dim);
  return a256(U * G * cap * S * sizeof(float)) + a256(U * G * cap * sizeof(float)) +
         a256(U * G * nqk * sizeof(float)) + a256(U * G * sizeof(float)) +
         a256(U * npv * G * D * sizeof(float)) + a256(U * sizeof(int)) + a256(U * cap * sizeof(int));
}

DecodeWs carve_decode(Carver& cv, const ekv_cache* c, const ekv_seqs* s, int Hq, int cap) {
  const size_t U = static_cast<size_t>(s->batch) * c->num_kv_heads;
  const size_t G = static_cast<size_t>(Hq / c->num_kv_heads);
  const int nqk = qk_splits(cap, c->page_size);
  const int npv = pv_splits(static_cast<int>(U), cap);
  const size_t S = static_cast<size_t>(c->page_size), D = static_cast<size_t>(c->head_dim);
  DecodeWs w;
  w.zbuf = cv.take<float>(U * G * cap * S);
  w.pmax = cv.take<float>(U * G * cap);
  w.cmax = cv.take<float>(U * G * static_cast<size_t>(nqk));
  w.taus = cv.take<float>(U * G);
  w.part = cv.take<float>(U * static_cast<size_t>(npv) * G * D);
  w.counter = cv.take<int>(U);
  w.sphys = cv.take<int>(U * static_cast<size_t>(cap));
  w.nqk = nqk;
  w.npv = npv;
  return w;
}

// Scratch of ekv_decode_adaptive: page scores, a count, the decode's scratch
// for every page, and the top-k scratch for any budget.
size_t adaptive_ws_bytes(const ekv_cache* c, const ekv_seqs* s, int Hq) {
  const size_t U = static_cast<size_t>(s->batch) * c->num_kv_heads;
  return a256(U * static_cast<size_t>(s->max_pages) * sizeof(float)) + a256(sizeof(int32_t)) +
         decode_ws_bytes(c, s, Hq, s->max_pages) +
         a256(topk_ws_bytes_upto(static_cast<int>(U), s->max_pages, s->max_pages));
}

size_t step_ws_bytes(const ekv_cache* c, const ekv_seqs* s, int Hq, int cap) {
  const size_t U = static_cast<size_t>(s->batch) * c->num_kv_heads;
  return a256(U * static_cast<size_t>(s->max_pages) * sizeof(float)) + gauss_ws_bytes(c, s, Hq) +
         decode_ws_bytes(c, s, Hq, cap) + a256(topk_ws_bytes_upto(static_cast<int>(U), s->max_pages, cap));
}

ekv_status check_ws(void* ws, size_t have, size_t need) {
  if (need > 0 && ws == nullptr) return EKV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return EKV_ERR_WORKSPACE;
  if (have < need) return EKV_ERR_WORKSPACE;
  return EKV_OK;
}

inline ekv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? EKV_OK : EKV_ERR_CUDA; }

#define EKV_TRY(expr)                   \
  do {                                  \
    const ekv_status st_ = (expr);      \
    if (st_ != EKV_OK) return st_;      \
  } while (0)

ekv_status validate_decode(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                           int32_t Hq, float scale, float alpha, const int32_t* sel,
                           const int32_t* n_sel, int32_t cap, const float* out) {
  EKV_TRY(check_cache(cache, true, false));
  EKV_TRY(check_seqs(seqs));
  EKV_TRY(check_heads(cache, Hq));
  EKV_TRY(check_alpha(alpha));
  if (q == nullptr || out == nullptr || !finite_pos(scale) || cap < 1) return EKV_ERR_INVALID_ARG;
  if ((sel == nullptr) != (n_sel == nullptr)) return EKV_ERR_INVALID_ARG;
  if (sel == nullptr && cap < seqs->max_pages) return EKV_ERR_INVALID_ARG;
  return EKV_OK;
}

}  // namespace
}  // namespace ekv

using namespace ekv;

extern "C" {

EKV_API ekv_status ekv_build_page_meta(const ekv_cache* cache, const ekv_seqs* seqs, void* stream) {
  EKV_TRY(check_cache(cache, false, true));
  EKV_TRY(check_seqs(seqs));
  return cuda_status(launch_build_meta(*cache, *seqs, static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_append(const ekv_cache* cache, const ekv_seqs* seqs, const void* k_new,
                              const void* v_new, void* stream) {
  EKV_TRY(check_cache(cache, true, true));
  EKV_TRY(check_seqs(seqs));
  if (k_new == nullptr || v_new == nullptr) return EKV_ERR_INVALID_ARG;
  return cuda_status(launch_append(*cache, *seqs, k_new, v_new, static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_score_pages(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                   int32_t num_q_heads, float scale, float* ub, void* stream) {
  EKV_TRY(check_cache(cache, false, true));
  EKV_TRY(check_seqs(seqs));
  EKV_TRY(check_heads(cache, num_q_heads));
  if (q == nullptr || ub == nullptr || !finite_pos(scale)) return EKV_ERR_INVALID_ARG;
  return cuda_status(
      launch_score(*cache, *seqs, q, num_q_heads, scale, ub, static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_select_topk(const ekv_seqs* seqs, int32_t num_kv_heads, int32_t page_size,
                                   const float* ub, int32_t k, int32_t* sel, int32_t* n_sel,
                                   void* ws, size_t ws_bytes, void* stream) {
  EKV_TRY(check_seqs(seqs));
  if (num_kv_heads < 1 || ub == nullptr || sel == nullptr || n_sel == nullptr || k < 1)
    return EKV_ERR_INVALID_ARG;
  if (page_size != 16 && page_size != 32) return EKV_ERR_UNSUPPORTED;
  const size_t need = topk_ws_bytes(seqs->batch * num_kv_heads, seqs->max_pages, k);
  if (ws != nullptr) EKV_TRY(check_ws(ws, ws_bytes, need));
  return cuda_status(launch_topk(*seqs, num_kv_heads, page_size, ub, k, k, sel, n_sel,
                                 ws != nullptr && need > 0 ? ws : nullptr,
                                 static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_select_gauss(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                    int32_t num_q_heads, float scale, float alpha, float delta,
                                    int32_t cap, int32_t* sel, int32_t* n_sel, float* tau_hat,
                                    void* ws, size_t ws_bytes, void* stream) {
  EKV_TRY(check_cache(cache, false, true));
  EKV_TRY(check_seqs(seqs));
  EKV_TRY(check_heads(cache, num_q_heads));
  EKV_TRY(check_alpha(alpha));
  if (q == nullptr || sel == nullptr || n_sel == nullptr || cap < 1 || !finite_pos(scale) ||
      isnan(delta))
    return EKV_ERR_INVALID_ARG;
  if (gauss_beta(alpha) == 0) return EKV_ERR_UNSUPPORTED;
  if (cache->head_dim == 64 && num_q_heads / cache->num_kv_heads > 8) return EKV_ERR_UNSUPPORTED;
  EKV_TRY(check_ws(ws, ws_bytes, gauss_ws_bytes(cache, seqs, num_q_heads)));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver cv{static_cast<char*>(ws)};
  const GaussWs gw = carve_gauss(cv, cache, seqs, num_q_heads);
  EKV_TRY(cuda_status(launch_gauss_stats(*cache, *seqs, q, num_q_heads, scale, alpha, gw, st)));
  return cuda_status(launch_gauss_select(*cache, *seqs, num_q_heads, alpha, delta, cap, gw, sel,
                                         n_sel, tau_hat, st));
}

EKV_API ekv_status ekv_entmax_decode(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                     int32_t num_q_heads, float scale, float alpha,
                                     const int32_t* sel, const int32_t* n_sel, int32_t cap,
                                     int32_t dense_v, float* out, float* tau,
                                     int32_t* support_count, uint32_t* support_bits, void* ws,
                                     size_t ws_bytes, void* stream) {
  EKV_TRY(validate_decode(cache, seqs, q, num_q_heads, scale, alpha, sel, n_sel, cap, out));
  EKV_TRY(check_ws(ws, ws_bytes, decode_ws_bytes(cache, seqs, num_q_heads, cap)));
  Carver cv{static_cast<char*>(ws)};
  const DecodeWs dw = carve_decode(cv, cache, seqs, num_q_heads, cap);
  return cuda_status(launch_decode(*cache, *seqs, q, num_q_heads, scale, alpha, sel, n_sel, cap,
                                   dense_v, out, tau, support_count, support_bits, dw,
                                   static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_exactness_certificate(const ekv_seqs* seqs, int32_t num_kv_heads,
                                             int32_t page_size, int32_t num_q_heads, float alpha,
                                             const float* ub, const int32_t* sel,
                                             const int32_t* n_sel, int32_t cap, const float* tau,
                                             int32_t* certified, void* stream) {
  EKV_TRY(check_seqs(seqs));
  EKV_TRY(check_alpha(alpha));
  if (num_kv_heads < 1 || page_size < 1 || num_q_heads < num_kv_heads || num_q_heads % num_kv_heads != 0)
    return EKV_ERR_INVALID_ARG;
  if (ub == nullptr || sel == nullptr || n_sel == nullptr || tau == nullptr || certified == nullptr || cap < 1)
    return EKV_ERR_INVALID_ARG;
  if (!certificate_smem_ok(seqs->max_pages)) return EKV_ERR_UNSUPPORTED;
  return cuda_status(launch_certificate(*seqs, num_kv_heads, page_size, num_q_heads, alpha, ub, sel, n_sel,
                                        cap, tau, certified, static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_decode_adaptive(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                       int32_t num_q_heads, float scale, float alpha, int32_t k0,
                                       int32_t* sel, int32_t* n_sel, float* out, float* tau,
                                       int32_t* certified, int32_t* k_used, void* ws, size_t ws_bytes,
                                       void* stream) {
  EKV_TRY(validate_decode(cache, seqs, q, num_q_heads, 1.0f, alpha, sel, n_sel, seqs ? seqs->max_pages : 1, out));
  EKV_TRY(check_cache(cache, true, true));
  if (!finite_pos(scale) || sel == nullptr || tau == nullptr || certified == nullptr || k_used == nullptr || k0 < 1)
    return EKV_ERR_INVALID_ARG;
  if (!certificate_smem_ok(seqs->max_pages)) return EKV_ERR_UNSUPPORTED;
  EKV_TRY(check_ws(ws, ws_bytes, adaptive_ws_bytes(cache, seqs, num_q_heads)));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t U = static_cast<size_t>(seqs->batch) * cache->num_kv_heads;
  const int P = seqs->max_pages;
  Carver cv{static_cast<char*>(ws)};
  float* ub = cv.take<float>(U * static_cast<size_t>(P));
  int32_t* count = cv.take<int32_t>(1);
  const DecodeWs dw = carve_decode(cv, cache, seqs, num_q_heads, P);
  void* tws = cv.base + cv.used;
  EKV_TRY(cuda_status(launch_score(*cache, *seqs, q, num_q_heads, scale, ub, st)));
  int k = k0 < P ? k0 : P;
  for (;;) {
    // sel holds [batch, Hkv, k] for the current budget k
    const size_t tk = topk_ws_bytes(static_cast<int>(U), P, k);
    EKV_TRY(cuda_status(launch_topk(*seqs, cache->num_kv_heads, cache->page_size, ub, k, k, sel, n_sel,
                                    tk > 0 ? tws : nullptr, st)));
    Carver cv2{static_cast<char*>(ws)};
    cv2.take<float>(U * static_cast<size_t>(P));
    cv2.take<int32_t>(1);
    const DecodeWs dk = carve_decode(cv2, cache, seqs, num_q_heads, k);
    EKV_TRY(cuda_status(launch_decode(*cache, *seqs, q, num_q_heads, scale, alpha, sel, n_sel, k, 0, out, tau,
                                      nullptr, nullptr, dk, st)));
    EKV_TRY(cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), st)));
    EKV_TRY(cuda_status(launch_certificate(*seqs, cache->num_kv_heads, cache->page_size, num_q_heads, alpha, ub,
                                           sel, n_sel, k, tau, certified, st, count)));
    int32_t left = 0;
    EKV_TRY(cuda_status(cudaMemcpyAsync(&left, count, sizeof(int32_t), cudaMemcpyDeviceToHost, st)));
    EKV_TRY(cuda_status(cudaStreamSynchronize(st)));
    if (left == 0 || k >= P) break;
    k = 2 * k < P ? 2 * k : P;
  }
  (void)dw;
  *k_used = k;
  return EKV_OK;
}

EKV_API ekv_status ekv_softmax_decode(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                      int32_t num_q_heads, float scale, const int32_t* sel,
                                      const int32_t* n_sel, int32_t cap, float* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream) {
  EKV_TRY(validate_decode(cache, seqs, q, num_q_heads, scale, 1.5f, sel, n_sel, cap, out));
  if (cache->dtype != EKV_BF16 || cache->page_size % 16 != 0) return EKV_ERR_UNSUPPORTED;
  const int U = seqs->batch * cache->num_kv_heads;
  EKV_TRY(check_ws(ws, ws_bytes, softmax_ws_bytes(U, num_q_heads, cache->num_kv_heads,
                                                  cache->head_dim, cap)));
  return cuda_status(launch_softmax_decode(*cache, *seqs, q, num_q_heads, scale, sel, n_sel, cap, out,
                                           lse, ws, static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_decode_step(const ekv_cache* cache, const ekv_seqs* seqs,
                                   const ekv_step_params* p, const void* q, int32_t num_q_heads,
                                   const void* k_new, const void* v_new, int32_t* sel,
                                   int32_t* n_sel, float* out, float* tau, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (p == nullptr) return EKV_ERR_INVALID_ARG;
  const bool full = p->policy == EKV_POLICY_FULL;
  if (p->policy != EKV_POLICY_TOPK && p->policy != EKV_POLICY_GAUSS && !full)
    return EKV_ERR_INVALID_ARG;
  EKV_TRY(check_cache(cache, true, true));
  const int cap = full ? seqs->max_pages : p->cap;
  EKV_TRY(validate_decode(cache, seqs, q, num_q_heads, p->scale, p->alpha, full ? nullptr : sel,
                          full ? nullptr : n_sel, cap, out));
  if (!full && (sel == nullptr || n_sel == nullptr)) return EKV_ERR_INVALID_ARG;
  if (p->policy == EKV_POLICY_TOPK && (p->k < 1 || p->k > cap)) return EKV_ERR_INVALID_ARG;
  if (p->policy == EKV_POLICY_GAUSS) {
    if (gauss_beta(p->alpha) == 0) return EKV_ERR_UNSUPPORTED;
    if (cache->head_dim == 64 && num_q_heads / cache->num_kv_heads > 8) return EKV_ERR_UNSUPPORTED;
    if (isnan(p->delta)) return EKV_ERR_INVALID_ARG;
  }
  if (p->append && (k_new == nullptr || v_new == nullptr)) return EKV_ERR_INVALID_ARG;
  EKV_TRY(check_ws(ws, ws_bytes, step_ws_bytes(cache, seqs, num_q_heads, cap)));

  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver cv{static_cast<char*>(ws)};
  const size_t U = static_cast<size_t>(seqs->batch) * cache->num_kv_heads;
  float* ub = cv.take<float>(U * static_cast<size_t>(seqs->max_pages));
  const GaussWs gw = carve_gauss(cv, cache, seqs, num_q_heads);
  const DecodeWs dw = carve_decode(cv, cache, seqs, num_q_heads, cap);
  void* tws = cv.base + cv.used;  // top-k scratch (sized for any k ≤ cap)

  if (p->append) EKV_TRY(cuda_status(launch_append(*cache, *seqs, k_new, v_new, st)));
  const int32_t* use_sel = sel;
  const int32_t* use_n = n_sel;
  if (p->policy == EKV_POLICY_TOPK) {
    EKV_TRY(cuda_status(launch_score(*cache, *seqs, q, num_q_heads, p->scale, ub, st, p->append ? 1 : 0)));
    EKV_TRY(cuda_status(launch_topk(*seqs, cache->num_kv_heads, cache->page_size, ub, p->k, cap,
                                    sel, n_sel,
                                    topk_ws_bytes(static_cast<int>(U), seqs->max_pages, p->k) > 0 ? tws : nullptr,
                                    st)));
  } else if (p->policy == EKV_POLICY_GAUSS) {
    EKV_TRY(cuda_status(launch_gauss_stats(*cache, *seqs, q, num_q_heads, p->scale, p->alpha, gw, st,
                                           p->append ? 1 : 0)));
    EKV_TRY(cuda_status(launch_gauss_select(*cache, *seqs, num_q_heads, p->alpha, p->delta, cap, gw,
                                            sel, n_sel, nullptr, st)));
  } else {
    use_sel = nullptr;
    use_n = nullptr;
  }
  return cuda_status(launch_decode(*cache, *seqs, q, num_q_heads, p->scale, p->alpha, use_sel,
                                   use_n, cap, p->dense_v, out, tau, nullptr, nullptr, dw, st));
}

EKV_API size_t ekv_workspace_bytes(int32_t op, const ekv_cache* cache, const ekv_seqs* seqs,
                                   int32_t num_q_heads, int32_t cap) {
  if (check_cache(cache, false, false) != EKV_OK || seqs == nullptr || seqs->batch < 1 ||
      seqs->max_pages < 1 || check_heads(cache, num_q_heads) != EKV_OK)
    return 0;
  switch (op) {
    case EKV_OP_SELECT_GAUSS:
      return gauss_ws_bytes(cache, seqs, num_q_heads);
    case EKV_OP_ENTMAX_DECODE:
      return cap < 1 ? 0 : decode_ws_bytes(cache, seqs, num_q_heads, cap);
    case EKV_OP_DECODE_STEP:
      return cap < 1 ? 0 : step_ws_bytes(cache, seqs, num_q_heads, cap);
    case EKV_OP_SELECT_TOPK:
      return cap < 1 ? 0 : topk_ws_bytes(seqs->batch * cache->num_kv_heads, seqs->max_pages, cap);
    case EKV_OP_DECODE_ADAPTIVE:
      return adaptive_ws_bytes(cache, seqs, num_q_heads);
    case EKV_OP_SOFTMAX_DECODE:
      return cap < 1 ? 0 : softmax_ws_bytes(seqs->batch * cache->num_kv_heads, num_q_heads,
                                            cache->num_kv_heads, cache->head_dim, cap);
    default:
      return 0;
  }
}

EKV_API int32_t ekv_step_kernel_count(const ekv_cache* cache, const ekv_seqs* seqs,
                                      const ekv_step_params* p, int32_t num_q_heads) {
  if (p == nullptr || check_cache(cache, false, false) != EKV_OK || seqs == nullptr ||
      seqs->batch < 1 || seqs->max_pages < 1 || check_heads(cache, num_q_heads) != EKV_OK)
    return 0;
  const bool full = p->policy == EKV_POLICY_FULL;
  const int cap = full ? seqs->max_pages : p->cap;
  if (cap < 1) return 0;
  int n = p->append ? 1 : 0;
  if (p->policy == EKV_POLICY_TOPK)
    n += 1 + (topk_ws_bytes(seqs->batch * cache->num_kv_heads, seqs->max_pages, p->k) > 0 ? 2 : 1);
  else if (p->policy == EKV_POLICY_GAUSS) n += 4;
  else if (!full) return 0;
  return n + decode_kernel_count(*cache, *seqs, num_q_heads, cap, p->dense_v);
}

EKV_API ekv_status ekv_selftest_wait_timeout(uint32_t polls, void* stream) {
  if (polls < 1 || polls > (1u << 20)) return EKV_ERR_INVALID_ARG;
  return cuda_status(launch_wait_timeout_selftest(polls, static_cast<cudaStream_t>(stream)));
}

EKV_API ekv_status ekv_get_error(uint32_t* flags) {
  if (flags == nullptr) return EKV_ERR_INVALID_ARG;
  unsigned int v = 0u, zero = 0u;
  if (cudaDeviceSynchronize() != cudaSuccess) return EKV_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_error_flags, sizeof(v)) != cudaSuccess) return EKV_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(zero)) != cudaSuccess) return EKV_ERR_CUDA;
  *flags = v;
  return EKV_OK;
}

EKV_API const char* ekv_status_string(ekv_status status) {
  switch (status) {
    case EKV_OK: return "ok";
    case EKV_ERR_INVALID_ARG: return "invalid argument";
    case EKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case EKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case EKV_ERR_CUDA: return "CUDA error";
    case EKV_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
