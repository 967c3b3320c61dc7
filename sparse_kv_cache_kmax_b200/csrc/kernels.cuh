// Launchers of libekv's kernels (internal to the library; the public C ABI is
// include/ekv.h, implemented in api.cu).
#pragma once

#include "common.cuh"

namespace ekv {

// Decode work split.  The score pass over the selected K takes 256 tokens per
// CTA (8 warps × 32 tokens); the V pass aims for eight CTAs per SM of a B200
// (two resident at a time), so that a dense V read keeps enough rows in flight.
constexpr int kQkTokensPerCta = 256;
constexpr int kPvTargetCtas = 1184;
constexpr int kPvMaxSplits = 64;

struct DecodeWs {
  float* zbuf;      // [U, G, cap·S] scores z of the selected tokens (−inf: no token)
  float* pmax;      // [U, G, cap]   page maxima of z
  float* cmax;      // [U, G, nqk]   maxima of z per score-pass CTA
  float* taus;      // [U, G]        thresholds τ (fp32)
  float* part;      // [U, npv, G, d] partial outputs of the V pass
  int* counter;     // [U]           finished V-pass CTAs
  int* sphys;       // [U, cap]      physical page of each selected slot (−1: bad)
  int nqk, npv;     // score-pass and V-pass CTAs per unit
};


// Pages per CTA of the Gaussian filter.
constexpr int kFilterChunk = 1024;
inline int filter_chunks(int max_pages) { return (max_pages + kFilterChunk - 1) / kFilterChunk; }

struct GaussWs {
  float* mu;        // [U, G, max_pages] (α−1)·m
  float* sig;       // [U, G, max_pages] (α−1)·s
  float* hat;       // [U, G, max_pages] (α−1)·ŝ
  double* tau_hat;  // [U, G]
  int* fcount;      // [U, nchunk] pages kept per filter chunk
  double* fbest;    // [U, nchunk] the chunk's largest margin
  int* fbest_at;    // [U, nchunk] its page (lowest on ties)
  int nchunk;
};

cudaError_t launch_build_meta(const ekv_cache& c, const ekv_seqs& s, cudaStream_t st);
cudaError_t launch_append(const ekv_cache& c, const ekv_seqs& s, const void* k_new,
                          const void* v_new, cudaStream_t st);
// after_append = 1: the previous kernel on the stream is launch_append, and
// the bf16 kernels overlap it (only tiles holding a sequence's last page wait).
cudaError_t launch_score(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq, float scale,
                         float* ub, cudaStream_t st, int after_append = 0);
cudaError_t launch_gauss_stats(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                               float scale, float alpha, const GaussWs& ws, cudaStream_t st,
                               int after_append = 0);
// ws: topk_ws_bytes(U, max_pages, k) bytes (NULL when that is 0, or for the
// one-stage path).
size_t topk_ws_bytes(int units, int max_pages, int k);
size_t topk_ws_bytes_upto(int units, int max_pages, int cap);  // the most any k ≤ cap needs
cudaError_t launch_topk(const ekv_seqs& s, int Hkv, int S, const float* ub, int k, int stride,
                        int32_t* sel, int32_t* n_sel, void* ws, cudaStream_t st);
cudaError_t launch_gauss_select(const ekv_cache& c, const ekv_seqs& s, int Hq, float alpha,
                                float delta, int cap, const GaussWs& ws, int32_t* sel,
                                int32_t* n_sel, float* tau_hat, cudaStream_t st);
cudaError_t launch_decode(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                          float scale, float alpha, const int32_t* sel, const int32_t* n_sel,
                          int cap, int dense_v, float* out, float* tau, int32_t* support_count,
                          uint32_t* support_bits, const DecodeWs& ws, cudaStream_t st);

// One bounded wait that nothing satisfies (certify.cu): raises EKV_EFLAG_TIMEOUT.
cudaError_t launch_wait_timeout_selftest(unsigned int polls, cudaStream_t st);

// Streaming multiprocessors of the current device (score.cu).
int sm_count();

// Exactness certificate per query head (certify.cu).
int certificate_smem_ok(int max_pages);
// uncertified (nullable): a device int the kernel adds the uncertified heads to.
cudaError_t launch_certificate(const ekv_seqs& s, int Hkv, int S, int Hq, float alpha, const float* ub,
                               const int32_t* sel, const int32_t* n_sel, int cap, const float* tau,
                               int32_t* cert, cudaStream_t st, int32_t* uncertified = nullptr);

// Softmax decode split over pages (softmax.cu).
int softmax_splits(int units, int cap);
size_t softmax_ws_bytes(int units, int Hq, int Hkv, int d, int cap);
cudaError_t launch_softmax_decode(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                                  float scale, const int32_t* sel, const int32_t* n_sel, int cap,
                                  float* out, float* lse, void* ws, cudaStream_t st);

// Kernels one launch_decode enqueues for these sizes (2: split decode, 1: cluster decode, 3: three-kernel decode).
int decode_kernel_count(const ekv_cache& c, const ekv_seqs& s, int Hq, int cap, int dense_v);

// Score-pass CTAs per unit: cap pages of S tokens, 256 tokens per CTA.
inline int qk_splits(int cap, int S) {
  const int pages = kQkTokensPerCta / S;
  return (cap + pages - 1) / pages;
}
// V-pass CTAs per unit (each scans an equal run of the selected pages).
inline int pv_splits(int units, int cap) {
  int ns = (kPvTargetCtas + units - 1) / units;
  if (ns > kPvMaxSplits) ns = kPvMaxSplits;
  if (ns > cap) ns = cap;
  if (ns < 1) ns = 1;
  const int per = (cap + ns - 1) / ns;
  return (cap + per - 1) / per;
}

}  // namespace ekv
