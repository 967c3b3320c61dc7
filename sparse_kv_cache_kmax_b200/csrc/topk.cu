// Top-k page selection — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.B, "Sélection de Pages Top-k": per (sequence, KV head), the k
// pages with the largest bounding-box score, ties to the lower logical page.
//
// One CTA per unit.  Scores become order-preserving uint32 keys, cached in
// shared memory when the unit has at most kSmemKeys pages.  The k-th largest
// key K* is found by a most-significant-digit radix select over 12, 12 and 8
// bits (a histogram of the keys that share the prefix found so far, built
// with warp-aggregated atomics, then a suffix count from the top).  Wide
// first digits keep the exponent-heavy top bits of fp32 scores from piling
// into a handful of bins.  The output pass gives each thread a contiguous
// run of pages, so one block scan of "taken" counts writes every key > K*
// and the lowest-index (k − #{key > K*}) keys equal to K* in ascending page
// order.  All arithmetic on keys is integer.
#include "kernels.cuh"

namespace ekv {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kSmemKeys = 16384;
constexpr int kMaxBins = 4096;

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                int max_pages, int Hkv, int k, int stride, int32_t* __restrict__ sel,
                int32_t* __restrict__ n_sel) {
  extern __shared__ uint32_t keys_s[];  // [min(max_pages, kSmemKeys)]
  __shared__ unsigned int hist[kMaxBins];
  __shared__ unsigned int s_digit, s_above;
  __shared__ int scan_scratch[32];

  const int unit = blockIdx.x, b = unit / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, nt = blockDim.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  int32_t* out = sel + static_cast<size_t>(unit) * stride;
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  if (P <= k) {
    for (int i = tid; i < P; i += nt) out[i] = i;
    if (tid == 0) n_sel[unit] = P;
    return;
  }
  const bool cached = P <= kSmemKeys;
  if (cached)
    for (int i = tid; i < P; i += nt) keys_s[i] = float_key(row[i]);
  __syncthreads();
  auto key_at = [&](int i) -> uint32_t { return cached ? keys_s[i] : float_key(row[i]); };

  unsigned int prefix = 0u, mask = 0u, krem = static_cast<unsigned int>(k);
  const int shifts[3] = {20, 8, 0}, widths[3] = {12, 12, 8};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass], nbins = 1 << widths[pass];
    for (int i = tid; i < nbins; i += nt) hist[i] = 0u;
    __syncthreads();
    for (int base = 0; base < P; base += nt) {
      const int i = base + tid;
      unsigned int bin = 0xffffffffu;  // no bin: outside the surviving prefix
      if (i < P) {
        const uint32_t key = key_at(i);
        if ((key & mask) == prefix) bin = (key >> shift) & static_cast<unsigned int>(nbins - 1);
      }
      const unsigned int same = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xffffffffu && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
    }
    __syncthreads();
    // thread t owns `per` consecutive bins counted from the top
    const int per = nbins >= nt ? nbins / nt : 1;
    unsigned int c[kMaxBins / kTopkThreads], local = 0u;
#pragma unroll
    for (int r = 0; r < kMaxBins / kTopkThreads; ++r) {
      const int bin = nbins - 1 - per * tid - r;
      c[r] = (r < per && bin >= 0) ? hist[bin] : 0u;
      local += c[r];
    }
    int total;
    const unsigned int before =
        static_cast<unsigned int>(block_exclusive_scan(static_cast<int>(local), scan_scratch, &total));
    if (before < krem && before + local >= krem) {
      unsigned int acc = before;
      int r = 0;
      while (r < per - 1 && acc + c[r] < krem) acc += c[r++];
      s_digit = static_cast<unsigned int>(nbins - 1 - per * tid - r);
      s_above = acc;
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= static_cast<unsigned int>(nbins - 1) << shift;
    krem -= s_above;
    __syncthreads();
  }

  // output: contiguous runs per thread keep the ascending page order
  const uint32_t kth = prefix;
  const int run = (P + nt - 1) / nt;
  const int i0 = min(P, tid * run), i1 = min(P, i0 + run);
  int n_gt = 0, n_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    n_gt += key > kth ? 1 : 0;
    n_eq += key == kth ? 1 : 0;
  }
  int eq_total, take_total;
  const int eq_before = block_exclusive_scan(n_eq, scan_scratch, &eq_total);
  const int ties_here = max(0, min(n_eq, static_cast<int>(krem) - eq_before));
  int pos = block_exclusive_scan(n_gt + ties_here, scan_scratch, &take_total);
  int ties_left = ties_here;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    bool take = key > kth;
    if (key == kth && ties_left > 0) {
      take = true;
      --ties_left;
    }
    if (take && pos < k) out[pos++] = i;
  }
  if (tid == 0) n_sel[unit] = k;
}

}  // namespace

cudaError_t launch_topk(const ekv_seqs& s, int Hkv, int S, const float* ub, int k, int stride,
                        int32_t* sel, int32_t* n_sel, cudaStream_t st) {
  const int keys = s.max_pages < kSmemKeys ? s.max_pages : kSmemKeys;
  const size_t smem = static_cast<size_t>(keys) * sizeof(uint32_t);
  const size_t static_smem = kMaxBins * sizeof(unsigned int) + 64 * sizeof(int);
  if (smem + static_smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  topk_kernel<<<s.batch * Hkv, kTopkThreads, smem, st>>>(ub, s.seq_lens, S, s.max_pages, Hkv, k,
                                                          stride, sel, n_sel);
  return cudaGetLastError();
}

}  // namespace ekv
