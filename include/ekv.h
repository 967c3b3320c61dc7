/*
 * ekv.h — C ABI of the EntmaxKV support-aware paged α-entmax decode library
 * (libekv.so, hand-written CUDA for sm_100a).
 *
 * Source of the method: "Résumé Technique : EntmaxKV – Décodage Conscient du
 * Support pour l'Attention Entmax" (gist.science/fr/paper/2605.21649), cited
 * below as [EntmaxKV] with the section that defines each operation.  The page
 * states the problem (a paged KV cache, a decode query, per-page metadata, a
 * top-k budget k or a margin Δ, α) and prints no formula and no API; the
 * formulas used are stated beside each call.
 *
 * Conventions shared by every call
 * --------------------------------
 * Ownership   The caller owns every buffer.  All pointers named "device" point
 *             to CUDA device memory; the library never allocates and keeps no
 *             state between calls except the sticky device error word read by
 *             ekv_get_error().
 * Streams     `stream` is a cudaStream_t passed as void* (NULL = legacy
 *             default stream).  Every call only enqueues work on it and never
 *             synchronises, except ekv_get_error().
 * Errors      Host-side validation runs before any launch and returns
 *             EKV_ERR_INVALID_ARG / EKV_ERR_UNSUPPORTED / EKV_ERR_WORKSPACE
 *             without touching the device.  A failed launch returns
 *             EKV_ERR_CUDA.  Data-dependent faults found on the device (a page
 *             id outside the pool, a sequence length outside 1..max_pages·S, a
 *             Gaussian selection larger than `cap`) never trap: the kernel skips
 *             the access, clamps, and ORs a bit into the device error word.
 * Dtypes      EKV_BF16 or EKV_F32 for the K/V pools, the metadata pools and
 *             the query.  Scores, bounds, thresholds and outputs are fp32.
 * Indices     Pages named in `sel` are *logical* page indices of the
 *             sequence; page_table maps them to physical pages.
 * Units       A unit is one (sequence b, KV head h) pair, u = b·Hkv + h.
 *             Query head hq belongs to KV head hq / G with G = Hq / Hkv.
 *
 * Memory layouts (row-major, dense)
 * ---------------------------------
 *   k_pool, v_pool [num_phys_pages, Hkv, S, d]
 *   box            [Hkv, num_phys_pages, 2, d]   row 0 = k_max, row 1 = k_min
 *   mom            [Hkv, num_phys_pages, 2, d]   row 0 = mean,  row 1 = variance
 *                  (head-major: one head's rows of consecutive physical pages
 *                  are adjacent, so scoring a sequence reads them in order)
 *   page_table     [batch, max_pages] int32, seq_lens [batch] int32
 *   q              [batch, Hq, d]
 *   ub             [batch, Hkv, max_pages] fp32
 *   sel            [batch, Hkv, cap] int32 (ascending), n_sel [batch, Hkv]
 *   out            [batch, Hq, d] fp32
 */
#ifndef EKV_H
#define EKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EKV_API __attribute__((visibility("default")))

typedef enum {
  EKV_OK = 0,
  EKV_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, α ≤ 1, k < 1, ... */
  EKV_ERR_UNSUPPORTED = 2, /* d ∉ {64,128}, S ∉ {16,32}, G ∉ {1,2,4,8,16}, β not integer */
  EKV_ERR_WORKSPACE = 3,   /* ws too small or not 256-byte aligned */
  EKV_ERR_CUDA = 4,        /* a kernel launch or CUDA runtime call failed */
  EKV_ERR_TIMEOUT = 5      /* reserved: a bounded device wait gave up */
} ekv_status;

typedef enum { EKV_F32 = 0, EKV_BF16 = 1 } ekv_dtype;

/* Bits of the sticky device error word (ekv_get_error). */
#define EKV_EFLAG_BAD_PAGE 1u      /* page_table entry outside [0, num_phys_pages) */
#define EKV_EFLAG_BAD_LEN 2u       /* seq_lens entry outside [1, max_pages·S] */
#define EKV_EFLAG_SEL_OVERFLOW 4u  /* Gaussian policy kept more than cap pages */
#define EKV_EFLAG_BAD_SEL 8u       /* sel entry outside [0, pages of the sequence) */
#define EKV_EFLAG_TIMEOUT 16u      /* a bounded wait on an asynchronous copy gave up */

/* The paged KV cache and its per-page metadata pools (all device memory). */
typedef struct {
  int32_t dtype;          /* ekv_dtype of k_pool, v_pool, box, mom and q */
  int32_t head_dim;       /* d ∈ {64, 128} */
  int32_t page_size;      /* S ∈ {16, 32} tokens per page */
  int32_t num_kv_heads;   /* Hkv ≥ 1 */
  int32_t num_phys_pages; /* pages in each pool */
  void* k_pool;
  void* v_pool;
  void* box;
  void* mom;
} ekv_cache;

/* The batch of sequences: page tables and lengths (device memory). */
typedef struct {
  const int32_t* page_table; /* [batch, max_pages] physical page of each logical page */
  const int32_t* seq_lens;   /* [batch] tokens, including the one being decoded */
  int32_t batch;
  int32_t max_pages;
} ekv_seqs;

/*
 * ekv_build_page_meta — [EntmaxKV] §2.A, "Bornes de Boîte Englobante" and
 * "Statistiques Gaussiennes".  For every page p < ⌈L_b/S⌉ of every sequence
 * and every KV head, over the n_p = min(S, L_b − p·S) valid tokens, writes
 *   box: k_max_j, k_min_j (exact);
 *   mom: μ_j = (1/n_p)Σ_t k_tj and the population variance
 *        σ²_j = (1/n_p)Σ_t (k_tj − μ_j)²,
 * both accumulated in float64 in token order and rounded once (nearest-even)
 * to the cache dtype.  Used after prefill; reads all of K.
 */
EKV_API ekv_status ekv_build_page_meta(const ekv_cache* cache, const ekv_seqs* seqs, void* stream);

/*
 * ekv_append — the cache append of a decode step, fused with the metadata
 * update of [EntmaxKV] §2.A.  k_new, v_new: device [batch, Hkv, d] in the cache
 * dtype.  Writes token L_b − 1 of every sequence (seq_lens already counts it)
 * into its page, then recomputes box/mom of that page over its valid tokens
 * exactly as ekv_build_page_meta does.
 */
EKV_API ekv_status ekv_append(const ekv_cache* cache, const ekv_seqs* seqs, const void* k_new,
                              const void* v_new, void* stream);

/*
 * ekv_score_pages — [EntmaxKV] §2.A, the bounding-box upper bound.  For query
 * head h and page p: ub_{p,h} = scale·Σ_j max(q_hj·kmin_pj, q_hj·kmax_pj),
 * an upper bound of every token score scale·q_h·k of the page.  The page
 * score of a KV head is the max over the G query heads of its group:
 * ub[b, kvh, p] for p < ⌈L_b/S⌉ (entries past that are not written).
 * q: device [batch, Hq, d]; ub: device fp32 [batch, Hkv, max_pages].
 */
EKV_API ekv_status ekv_score_pages(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                   int32_t num_q_heads, float scale, float* ub, void* stream);

/*
 * ekv_select_topk — [EntmaxKV] §2.B.1, "Sélection de Pages Top-k": per unit,
 * the k pages with the largest ub (ties to the lower logical index; all pages
 * when ⌈L_b/S⌉ ≤ k), written ascending to sel[b, kvh, 0..n_sel) with
 * n_sel = min(k, ⌈L_b/S⌉).  page_size S turns seq_lens into page counts.
 * ub: device [batch, Hkv, max_pages] (ekv_score_pages); sel: device
 * [batch, Hkv, k]; n_sel: [batch, Hkv].  ws: ekv_workspace_bytes(
 * EKV_OP_SELECT_TOPK, ..., cap = k) bytes, which is 0 (ws may be NULL) up to
 * 16384 pages per sequence; longer sequences with that scratch are selected
 * in two stages (chunks of 8192 pages keep their k best, then k among those),
 * without it in one slower stage.
 */
EKV_API ekv_status ekv_select_topk(const ekv_seqs* seqs, int32_t num_kv_heads, int32_t page_size,
                                   const float* ub, int32_t k, int32_t* sel, int32_t* n_sel,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * ekv_select_gauss — [EntmaxKV] §2.A "Statistiques Gaussiennes" + §2.B.2,
 * "Sélection Entmax Consciente de Gaussienne".  Per query head h: token scores
 * of page p are modelled as N(m, s²) with m = scale·q_h·μ_p and
 * s² = scale²·Σ_j q_hj² σ²_pj.  τ̂_h solves Σ_p n_p·E[(u − τ̂)_+^β] = 1 with
 * u ~ N((α−1)m, (α−1)²s²), β = 1/(α−1) ∈ {1,2,3,4} (else EKV_ERR_UNSUPPORTED).
 * Page p is kept when (α−1)·(m + s·√(2 ln n_p)) > τ̂_h − Δ for any head of the
 * group; if none is, the single page with the largest margin.  sel (ascending)
 * holds at most cap pages: a larger selection keeps its first cap pages and
 * sets EKV_EFLAG_SEL_OVERFLOW.  tau_hat: device fp32 [batch, Hq] (nullable).
 * ws: device scratch of ekv_workspace_bytes(EKV_OP_SELECT_GAUSS, ...) bytes.
 */
EKV_API ekv_status ekv_select_gauss(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                    int32_t num_q_heads, float scale, float alpha, float delta,
                                    int32_t cap, int32_t* sel, int32_t* n_sel, float* tau_hat,
                                    void* ws, size_t ws_bytes, void* stream);

/*
 * ekv_entmax_decode — [EntmaxKV] §2.C, "Attention Entmax Parcimonieuse".  Over
 * the valid tokens T of the selected pages (sel == NULL: every page of the
 * sequence, the full-cache decode), for every query head of the unit:
 *   z_i = scale·q·k_i,  u_i = (α−1)·z_i,
 *   τ solves Σ_{i∈T} [u_i − τ]_+^{1/(α−1)} = 1,  p_i = [u_i − τ]_+^{1/(α−1)},
 *   out = Σ_i p_i·v_i,
 * reading V only for pages that hold a token with p_i > 0 for some head of
 * the group (dense_v ≠ 0 reads every selected V page instead).
 * sel: device [batch, Hkv, cap] with n_sel entries per unit (ascending), or
 * NULL with n_sel NULL; cap bounds n_sel (max_pages when sel is NULL).
 * Outputs (device): out fp32 [batch, Hq, d]; nullable tau [batch, Hq],
 * support_count [batch, Hq] int32, support_bits uint32
 * [batch, Hq, ⌈cap·S/32⌉] (bit i of a row: token i of the selected-token list,
 * page-major, is in the support).
 * ws: ekv_workspace_bytes(EKV_OP_ENTMAX_DECODE, ...) bytes.
 */
EKV_API ekv_status ekv_entmax_decode(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                     int32_t num_q_heads, float scale, float alpha,
                                     const int32_t* sel, const int32_t* n_sel, int32_t cap,
                                     int32_t dense_v, float* out, float* tau,
                                     int32_t* support_count, uint32_t* support_bits, void* ws,
                                     size_t ws_bytes, void* stream);

/*
 * ekv_softmax_decode — softmax attention decode over the paged cache: the
 * full-cache baseline of [EKV] §4 (reading the whole cache is what sparse
 * decoding avoids), split over pages.  For every query head h, o_h = Σ_i e^{z_i − m}·v_i / Σ_i e^{z_i − m}
 * with z_i = scale·q_h·k_i over every valid token of the selected pages
 * (sel = NULL with n_sel NULL: every page of the sequence; cap ≥ max_pages).
 * sel: device [batch, Hkv, cap] logical page indices with n_sel entries per
 * unit (as ekv_entmax_decode).  Outputs (device): out fp32 [batch, Hq, d];
 * lse (nullable) fp32 [batch, Hq] = m + ln Σ_i e^{z_i − m} (−inf for a
 * sequence without tokens, whose output row is 0).  bf16 caches with a page
 * size that is a multiple of 16; any other returns EKV_ERR_UNSUPPORTED.
 * ws: ekv_workspace_bytes(EKV_OP_SOFTMAX_DECODE, ...) bytes; the call clears
 * the part it needs.
 */
EKV_API ekv_status ekv_softmax_decode(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                      int32_t num_q_heads, float scale, const int32_t* sel,
                                      const int32_t* n_sel, int32_t cap, float* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream);

/*
 * ekv_exactness_certificate — [EKV] §3 "Récupération du Support": the sparse
 * output equals the full-cache output when the selection holds the α-entmax
 * support.  certified[b, hq] = 1 when (α−1)·max_{p ∉ sel} ub[b, kvh, p] ≤
 * tau[b, hq] over the valid unselected pages p of unit (b, kvh = hq / G), or
 * when no valid page is left unselected; else 0.  A head whose τ is +inf (no
 * finite score among the selected tokens) is certified only in the latter
 * case.  ub: device [batch, Hkv, max_pages] unit scores from ekv_score_pages;
 * sel / n_sel / cap as for ekv_entmax_decode (non-NULL); tau: device
 * [batch, Hq] from the decode of that selection; certified: device int32
 * [batch, Hq].  max_pages above 393216 returns EKV_ERR_UNSUPPORTED.
 */
EKV_API ekv_status ekv_exactness_certificate(const ekv_seqs* seqs, int32_t num_kv_heads,
                                             int32_t page_size, int32_t num_q_heads, float alpha,
                                             const float* ub, const int32_t* sel,
                                             const int32_t* n_sel, int32_t cap, const float* tau,
                                             int32_t* certified, void* stream);

/*
 * ekv_decode_adaptive — the top-k decode with a budget that grows until the
 * output is provably the full-cache one ([EKV] §3 "Récupération du Support",
 * through ekv_exactness_certificate): page scores once, then for
 * k = k0, 2·k0, 4·k0, … (at most max_pages) the top-k selection, the sparse
 * decode and the certificate of every query head; the first k at which every
 * head of every unit is certified (or every page is selected) ends it.  The
 * count of uncertified heads is kept on the device and read back once per
 * round, so the call synchronises `stream` once per round.  Outputs are those
 * of the last round: sel device [batch, Hkv, k] (row stride k = *k_used; the
 * buffer must hold batch·Hkv·max_pages entries), n_sel [batch, Hkv], out
 * fp32 [batch, Hq, d], tau fp32 [batch, Hq], certified int32 [batch, Hq]
 * (all 1: a selection of every page is certified too); k_used: host int.  scale and
 * alpha as ekv_entmax_decode.  ws: ekv_workspace_bytes(
 * EKV_OP_DECODE_ADAPTIVE, ...) bytes (cap ignored).
 */
EKV_API ekv_status ekv_decode_adaptive(const ekv_cache* cache, const ekv_seqs* seqs, const void* q,
                                       int32_t num_q_heads, float scale, float alpha, int32_t k0,
                                       int32_t* sel, int32_t* n_sel, float* out, float* tau,
                                       int32_t* certified, int32_t* k_used, void* ws, size_t ws_bytes,
                                       void* stream);

/* Bytes of the library-owned scratch array of ekv_entmax_decode_static_ws. */
#define EKV_STATIC_WS_BYTES (16u << 20)

/*
 * ekv_entmax_decode_static_ws — ekv_entmax_decode without a caller workspace.
 * The source page has no counterpart to this call: it exists for callers
 * that cannot allocate device memory, such as a plugin inside a framework
 * that owns the device memory pool and offers no scratch buffer, or a serving
 * loop that must not call cudaMalloc once running.  Arguments and outputs are
 * those of ekv_entmax_decode; the scratch comes from one static device array
 * of EKV_STATIC_WS_BYTES bytes that every GPU loading the library holds until
 * the process exits.  A configuration whose scratch
 * (ekv_workspace_bytes(EKV_OP_ENTMAX_DECODE, ...)) exceeds that size returns
 * EKV_ERR_WORKSPACE before any device work (the limit is checked against
 * the scratch of every decode path, although the one-cluster-per-unit path,
 * taken for few units, keeps its scratch in shared memory and reads none of
 * the array; the many-unit and fp32 paths keep their scores, maxima, page
 * ids and split counters there).  All calls on a device share the array:
 * calls that overlap on the GPU race, so serialise them.  The array keeps
 * the previous call's contents; the only part that must start at zero (the
 * split counters) is reset by the call itself.  The call looks up the
 * array's device address with the device current: on the first call on a
 * device, and again on every call made outside a stream capture (so a
 * cudaDeviceReset, after which the address may change, is followed); a call
 * inside a capture uses the address found before, so make one call on each
 * device before capturing.  Allocates nothing.
 */
EKV_API ekv_status ekv_entmax_decode_static_ws(const ekv_cache* cache, const ekv_seqs* seqs,
                                               const void* q, int32_t num_q_heads, float scale,
                                               float alpha, const int32_t* sel,
                                               const int32_t* n_sel, int32_t cap, int32_t dense_v,
                                               float* out, float* tau, int32_t* support_count,
                                               uint32_t* support_bits, void* stream);

/* Selection policies of a whole decode step. */
typedef enum { EKV_POLICY_TOPK = 0, EKV_POLICY_GAUSS = 1, EKV_POLICY_FULL = 2 } ekv_policy;

typedef struct {
  int32_t policy;  /* ekv_policy */
  int32_t k;       /* top-k budget (EKV_POLICY_TOPK) */
  float delta;     /* margin Δ (EKV_POLICY_GAUSS) */
  int32_t cap;     /* pages a unit may select: k for top-k, ≤ max_pages otherwise */
  float alpha;     /* α > 1 */
  float scale;     /* score scale, usually 1/√d */
  int32_t dense_v; /* 1: read V of every selected page */
  int32_t append;  /* 1: run ekv_append(k_new, v_new) first */
} ekv_step_params;

/*
 * ekv_decode_step — one whole decode step of [EntmaxKV] §2 in stream order:
 * append (if params->append) → page scores + top-k, or the Gaussian policy,
 * or every page → sparse α-entmax attention.  sel / n_sel receive the
 * selection (device [batch, Hkv, cap] / [batch, Hkv]); out [batch, Hq, d].
 * tau (nullable) receives [batch, Hq] thresholds.  ws: ekv_workspace_bytes(
 * EKV_OP_DECODE_STEP, ...) bytes.
 */
EKV_API ekv_status ekv_decode_step(const ekv_cache* cache, const ekv_seqs* seqs,
                                   const ekv_step_params* params, const void* q,
                                   int32_t num_q_heads, const void* k_new, const void* v_new,
                                   int32_t* sel, int32_t* n_sel, float* out, float* tau, void* ws,
                                   size_t ws_bytes, void* stream);

typedef enum {
  EKV_OP_SELECT_GAUSS = 1,
  EKV_OP_ENTMAX_DECODE = 2,
  EKV_OP_DECODE_STEP = 3,
  EKV_OP_SOFTMAX_DECODE = 4,
  EKV_OP_SELECT_TOPK = 5,
  EKV_OP_DECODE_ADAPTIVE = 6
} ekv_op;

/*
 * ekv_workspace_bytes — device scratch an op needs, from the host-side sizes
 * only (cache dims, batch, max_pages, Hq, cap; for EKV_OP_DECODE_STEP `cap` is
 * params->cap).  Returns 0 when the sizes are invalid.
 */
EKV_API size_t ekv_workspace_bytes(int32_t op, const ekv_cache* cache, const ekv_seqs* seqs,
                                   int32_t num_q_heads, int32_t cap);

/*
 * ekv_step_kernel_count — how many kernels one ekv_decode_step call with these
 * arguments enqueues: the append (if params->append), the selection (2 for
 * top-k, 3 when it runs in two stages (more than 16384 pages per sequence),
 * 3 for the Gaussian policy, 0 for every page) and the decode (1 when
 * a bf16 selection fits the one-cluster-per-unit kernel, else 3).  Host-side
 * only; returns 0 when the sizes are invalid.
 */
EKV_API int32_t ekv_step_kernel_count(const ekv_cache* cache, const ekv_seqs* seqs,
                                      const ekv_step_params* params, int32_t num_q_heads);

/*
 * ekv_selftest_wait_timeout — exercises the failure path every bounded wait
 * of the library shares: one GPU thread waits, for `polls` polls (1 to
 * 1048576), on an mbarrier that nothing ever completes; the wait gives up,
 * ORs EKV_EFLAG_TIMEOUT into the device error word and the kernel returns, so
 * the context stays usable.  No source-page counterpart: a diagnostic for
 * failure detection.
 */
EKV_API ekv_status ekv_selftest_wait_timeout(uint32_t polls, void* stream);

/* Reads the sticky device error word into *flags (EKV_EFLAG_* bits) and clears
 * it.  Synchronises the device. */
EKV_API ekv_status ekv_get_error(uint32_t* flags);

/* Static description of a status code. */
EKV_API const char* ekv_status_string(ekv_status status);

#ifdef __cplusplus
}
#endif
#endif /* EKV_H */
