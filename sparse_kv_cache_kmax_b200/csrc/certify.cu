// Exactness certificate — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §3 "Récupération du Support": the sparse output equals the
// full-cache output when the selected tokens contain the α-entmax support.
// Every token score of page p is at most the page's unit score ub_p (the
// bound, maximised over the group's heads), so if (α−1)·max_{p ∉ sel} ub_p ≤
// τ_h, no unselected token can enter head h's support: τ_h then also solves
// the full-cache equation and the outputs agree.
//
// One CTA per unit: the selected pages are marked in a shared-memory bitmask,
// the unselected pages' scores are reduced to their maximum, and each query
// head of the group compares it with its τ.
#include "kernels.cuh"

namespace ekv {

namespace {

constexpr int kCertThreads = 256;

__global__ void __launch_bounds__(kCertThreads)
    certificate_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                       int max_pages, int Hkv, int G, int Hq, const int32_t* __restrict__ sel,
                       const int32_t* __restrict__ n_sel, int cap, const float* __restrict__ tau,
                       float am1, int32_t* __restrict__ cert, int32_t* __restrict__ uncertified) {
  grid_dep_enter();
  extern __shared__ unsigned int selmask[];  // [⌈max_pages/32⌉]
  __shared__ float scratch[32];
  const int unit = blockIdx.x, b = unit / Hkv, kvh = unit % Hkv, tid = threadIdx.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  const int words = (P + 31) / 32;
  for (int w = tid; w < words; w += kCertThreads) selmask[w] = 0u;
  __syncthreads();
  const int n = max(0, min(n_sel[unit], cap));
  for (int i = tid; i < n; i += kCertThreads) {
    const int p = sel[static_cast<size_t>(unit) * cap + i];
    if (p >= 0 && p < P) atomicOr(&selmask[p >> 5], 1u << (p & 31));
  }
  __syncthreads();
  float m = -INFINITY;
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  for (int p = tid; p < P; p += kCertThreads)
    if (!((selmask[p >> 5] >> (p & 31)) & 1u)) m = fmaxf(m, row[p]);
  m = block_reduce(m, scratch, [](float x, float y) { return fmaxf(x, y); });
  for (int h = tid; h < G; h += kCertThreads) {
    const size_t orow = static_cast<size_t>(b) * Hq + static_cast<size_t>(kvh) * G + h;
    const float t = tau[orow];
    // nothing unselected can hold support; a head with no support in the
    // selection (τ = +inf) is exact only if nothing is left unselected
    const int ok = (m == -INFINITY || (t < INFINITY && am1 * m <= t)) ? 1 : 0;
    cert[orow] = ok;
    if (!ok && uncertified) atomicAdd(uncertified, 1);
  }
}

}  // namespace

// Self-test of the bounded-wait path: one thread waits on an mbarrier that
// nothing ever arrives at, for `polls` polls; the wait gives up, raises
// EKV_EFLAG_TIMEOUT and the kernel returns normally.
__global__ void wait_timeout_selftest_kernel(unsigned int polls) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0u, polls);
}

cudaError_t launch_wait_timeout_selftest(unsigned int polls, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 1, 0, st>>>(polls);
  return cudaGetLastError();
}

int certificate_smem_ok(int max_pages) { return (max_pages + 31) / 32 * 4 <= 48 * 1024; }

cudaError_t launch_certificate(const ekv_seqs& s, int Hkv, int S, int Hq, float alpha, const float* ub,
                               const int32_t* sel, const int32_t* n_sel, int cap, const float* tau,
                               int32_t* cert, cudaStream_t st, int32_t* uncertified) {
  const size_t smem = static_cast<size_t>((s.max_pages + 31) / 32) * sizeof(unsigned int);
  const cudaError_t e = launch_k(certificate_kernel, dim3(s.batch * Hkv), dim3(kCertThreads), smem, st, ub,
                                 s.seq_lens, S, s.max_pages, Hkv, Hq / Hkv, Hq, sel, n_sel, cap, tau,
                                 alpha - 1.0f, cert, uncertified);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ekv
