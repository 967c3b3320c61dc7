// Top-k page selection — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.B, "Sélection de Pages Top-k": per (sequence, KV head), the k
// pages with the largest bounding-box score, ties to the lower logical page.
//
// One CTA per unit.  Scores become order-preserving uint32 keys, cached in
// shared memory when the unit has at most kSmemKeys pages.  The k-th largest
// key K* is found by a radix select whose digits adapt to the keys: each
// pass bins the keys of the current interval [lo, hi] into at most 4096
// equal bins that span exactly that interval (bin = (key − lo) >> shift), so
// scores spread over all bins instead of piling into the few bins their
// exponent bits would give.  The bin holding the k-th largest key becomes the
// next interval; a pass with shift 0 leaves a single key value, K*, after at
// most three passes (often two).  The output pass gives each thread a
// contiguous run of pages, so one block scan of "taken" counts writes every
// key > K* and the lowest-index (k − #{key > K*}) keys equal to K* in
// ascending page order.  All arithmetic on keys is integer.
#include "kernels.cuh"

namespace ekv {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kSmemKeys = 16384;
constexpr int kBins = 4096;
constexpr int kDigitBits = 12;
constexpr int kBinsPerThread = kBins / kTopkThreads;

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                int max_pages, int Hkv, int k, int stride, int32_t* __restrict__ sel,
                int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  extern __shared__ uint32_t keys_s[];  // [min(max_pages, kSmemKeys)]
  __shared__ unsigned int hist[2][kBins];
  __shared__ unsigned int w_a[kTopkWarps], w_b[kTopkWarps];
  __shared__ unsigned int s_lo, s_hi, s_above;

  const int unit = blockIdx.x, b = unit / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  int32_t* out = sel + static_cast<size_t>(unit) * stride;
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  if (P <= k) {
    for (int i = tid; i < P; i += kTopkThreads) out[i] = i;
    if (tid == 0) n_sel[unit] = P;
    return;
  }
  const bool cached = P <= kSmemKeys;
  unsigned int kmin = 0xffffffffu, kmax = 0u;
  for (int i = tid; i < P; i += kTopkThreads) {
    const uint32_t key = float_key(row[i]);
    if (cached) keys_s[i] = key;
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  }
  for (int i = tid; i < kBins; i += kTopkThreads) hist[0][i] = 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    w_a[warp] = kmin;
    w_b[warp] = kmax;
  }
  __syncthreads();
  kmin = w_a[lane];
  kmax = w_b[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  auto key_at = [&](int i) -> uint32_t { return cached ? keys_s[i] : float_key(row[i]); };

  // The interval [lo, hi] holds the k-th largest key; krem of its keys are
  // still to be taken.  Each pass splits it into ≤ 4096 equal bins.
  unsigned int lo = kmin, hi = kmax, krem = static_cast<unsigned int>(k);
  int cur = 0;
  for (int pass = 0; pass < 4 && lo < hi; ++pass) {
    const unsigned int range = hi - lo;
    const int width = 32 - __clz(range);
    const int shift = width > kDigitBits ? width - kDigitBits : 0;
    const int nbins = static_cast<int>(range >> shift) + 1;
    unsigned int* hc = hist[cur];
    for (int base = 0; base < P; base += kTopkThreads) {
      const int i = base + tid;
      unsigned int bin = 0xffffffffu;  // outside the interval
      if (i < P) {
        const uint32_t key = key_at(i);
        if (key >= lo && key <= hi) bin = (key - lo) >> shift;
      }
      const unsigned int b0 = __shfl_sync(0xffffffffu, bin, 0);
      if (__all_sync(0xffffffffu, bin == b0)) {  // one bin for the whole warp
        if (lane == 0 && b0 != 0xffffffffu) atomicAdd(&hc[b0], 32u);
      } else if (bin != 0xffffffffu) {
        atomicAdd(&hc[bin], 1u);
      }
    }
    for (int i = tid; i < kBins; i += kTopkThreads) hist[cur ^ 1][i] = 0u;  // next pass's bins
    __syncthreads();
    // thread t owns `per` consecutive bins counted from the top
    const int per = (nbins + kTopkThreads - 1) / kTopkThreads;
    unsigned int c[kBinsPerThread], local = 0u;
#pragma unroll
    for (int r = 0; r < kBinsPerThread; ++r) {
      const int bin = nbins - 1 - per * tid - r;
      c[r] = (r < per && bin >= 0) ? hc[bin] : 0u;
      local += c[r];
    }
    unsigned int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) w_a[warp] = incl;
    __syncthreads();
    unsigned int wt = w_a[lane], wincl = wt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += y;
    }
    const unsigned int warp_before = __shfl_sync(0xffffffffu, wincl - wt, warp);
    const unsigned int before = warp_before + incl - local;
    if (local > 0 && before < krem && before + local >= krem) {
      unsigned int acc = before;
      int r = 0;
      while (r < per - 1 && acc + c[r] < krem) acc += c[r++];
      const unsigned int bin = static_cast<unsigned int>(nbins - 1 - per * tid - r);
      s_above = acc;
      const unsigned long long base = static_cast<unsigned long long>(lo) + (static_cast<unsigned long long>(bin) << shift);
      s_lo = static_cast<unsigned int>(base);
      s_hi = static_cast<unsigned int>(min(static_cast<unsigned long long>(hi), base + ((1ull << shift) - 1ull)));
    }
    __syncthreads();
    krem -= s_above;
    lo = s_lo;
    hi = s_hi;
    cur ^= 1;
  }

  // Output: contiguous runs per thread keep the ascending page order.  The
  // selected pages are every key > K* and the first krem keys equal to K*;
  // an element's position = #greater before it + min(#equal before it, krem).
  const uint32_t kth = lo;
  const int run = (P + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(P, tid * run), i1 = min(P, i0 + run);
  unsigned int n_gt = 0, n_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    n_gt += key > kth ? 1u : 0u;
    n_eq += key == kth ? 1u : 0u;
  }
  unsigned int g_incl = n_gt, e_incl = n_eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int yg = __shfl_up_sync(0xffffffffu, g_incl, o);
    const unsigned int ye = __shfl_up_sync(0xffffffffu, e_incl, o);
    if (lane >= o) {
      g_incl += yg;
      e_incl += ye;
    }
  }
  __syncthreads();  // w_a / w_b were read above
  if (lane == 31) {
    w_a[warp] = g_incl;
    w_b[warp] = e_incl;
  }
  __syncthreads();
  unsigned int wg = w_a[lane], we = w_b[lane], wg_incl = wg, we_incl = we;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int yg = __shfl_up_sync(0xffffffffu, wg_incl, o);
    const unsigned int ye = __shfl_up_sync(0xffffffffu, we_incl, o);
    if (lane >= o) {
      wg_incl += yg;
      we_incl += ye;
    }
  }
  unsigned int gt_before = __shfl_sync(0xffffffffu, wg_incl - wg, warp) + g_incl - n_gt;
  unsigned int eq_before = __shfl_sync(0xffffffffu, we_incl - we, warp) + e_incl - n_eq;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    if (key > kth) {
      const unsigned int pos = gt_before + min(eq_before, krem);
      if (pos < static_cast<unsigned int>(k)) out[pos] = i;
      ++gt_before;
    } else if (key == kth) {
      if (eq_before < krem) {
        const unsigned int pos = gt_before + eq_before;
        if (pos < static_cast<unsigned int>(k)) out[pos] = i;
      }
      ++eq_before;
    }
  }
  if (tid == 0) n_sel[unit] = k;
}

}  // namespace

cudaError_t launch_topk(const ekv_seqs& s, int Hkv, int S, const float* ub, int k, int stride,
                        int32_t* sel, int32_t* n_sel, cudaStream_t st) {
  const int keys = s.max_pages < kSmemKeys ? s.max_pages : kSmemKeys;
  const size_t smem = static_cast<size_t>(keys) * sizeof(uint32_t);
  const size_t static_smem = 2 * kBins * sizeof(unsigned int) + 256;
  if (smem + static_smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t le = launch_k(topk_kernel, dim3(s.batch * Hkv), dim3(kTopkThreads), smem, st, ub,
                                  s.seq_lens, S, s.max_pages, Hkv, k, stride, sel, n_sel);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

}  // namespace ekv
