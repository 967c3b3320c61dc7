// Top-k page selection — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.B, "Sélection de Pages Top-k": per (sequence, KV head), the k
// pages with the largest bounding-box score, ties to the lower logical page.
//
// One CTA per list.  Scores become order-preserving uint32 keys, cached in
// shared memory when the list has at most kSmemKeys entries.  A unit with
// more pages than that is done in two stages: chunks of pages each keep their own k best (any page of
// the unit's k best is among its chunk's k best under the same order), then
// one CTA selects k among those winners, read through their page indices, so
// ties and order are unchanged.  The k-th largest
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
constexpr int kChunk = 8192;    // pages per first-stage chunk of a long unit
constexpr int kBins = 4096;
constexpr int kDigitBits = 12;
constexpr int kRankMax = 256;  // keys of the k-th key's bin ranked directly

// The k largest of n > k entries (key_of(i): order-preserving key of entry
// i), ties to the lower position; writes idx_of(position) of each, in
// ascending position order, to out[0..k) and k to *n_out.  The whole CTA
// calls it.  keys_s: shared scratch of n keys when cache_keys.
template <class KeyOf, class IdxOf>
__device__ void select_k(int P, int k, KeyOf key_of, IdxOf idx_of, uint32_t* keys_s, bool cache_keys,
                         int32_t* __restrict__ out, int32_t* __restrict__ n_out) {
  __shared__ unsigned int hist[2][kBins];
  __shared__ unsigned int w_a[kTopkWarps], w_b[kTopkWarps];
  __shared__ uint32_t rk_key[kRankMax];
  __shared__ int rk_idx[kRankMax];
  __shared__ unsigned int s_lo, s_hi, s_above, s_count, s_fill;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool cached = cache_keys;
  unsigned int kmin = 0xffffffffu, kmax = 0u;
  for (int i = tid; i < P; i += kTopkThreads) {
    const uint32_t key = key_of(i);
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
  auto key_at = [&](int i) -> uint32_t { return cached ? keys_s[i] : key_of(i); };

  // The interval [lo, hi] holds the k-th largest key; krem of its keys are
  // still to be taken.  Each pass splits it into ≤ 4096 equal bins; once the
  // bin of the k-th key holds few keys, they are ranked directly.
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
    // warp w covers bins top − 128w − 32r − lane (r = 0..3), counted from the top
    const int top = nbins - 1;
    unsigned int wsum = 0u;
#pragma unroll
    for (int r = 0; r < kBins / kTopkThreads; ++r) {
      const int bin = top - 128 * warp - 32 * r - lane;
      wsum += bin >= 0 ? hc[bin] : 0u;
    }
    wsum = __reduce_add_sync(0xffffffffu, wsum);
    if (lane == 0) w_a[warp] = wsum;
    __syncthreads();
    const unsigned int wt = w_a[lane];
    unsigned int wincl = wt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += y;
    }
    unsigned int before = __shfl_sync(0xffffffffu, wincl - wt, warp);
    const unsigned int mine = __shfl_sync(0xffffffffu, wt, warp);
    if (before < krem && before + mine >= krem) {  // this warp holds the k-th key's bin
#pragma unroll 1
      for (int r = 0; r < kBins / kTopkThreads; ++r) {
        const int bin = top - 128 * warp - 32 * r - lane;
        const unsigned int c = bin >= 0 ? hc[bin] : 0u;
        unsigned int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (c > 0 && before + incl - c < krem && before + incl >= krem) {
          s_above = before + incl - c;
          s_count = c;
          s_fill = 0u;
          const unsigned long long base = static_cast<unsigned long long>(lo) + (static_cast<unsigned long long>(bin) << shift);
          s_lo = static_cast<unsigned int>(base);
          s_hi = static_cast<unsigned int>(min(static_cast<unsigned long long>(hi), base + ((1ull << shift) - 1ull)));
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
        if (before >= krem) break;
      }
    }
    __syncthreads();
    krem -= s_above;
    lo = s_lo;
    hi = s_hi;
    cur ^= 1;
    const unsigned int cnt = s_count;
    if (lo < hi && cnt <= kRankMax) {
      // rank the bin's keys by (key descending, page ascending): the one of
      // rank krem − 1 is K*; of the keys equal to K*, krem − #{key > K*} go
      for (int base = 0; base < P; base += kTopkThreads) {
        const int i = base + tid;
        if (i < P) {
          const uint32_t key = key_at(i);
          if (key >= lo && key <= hi) {
            const unsigned int pos = atomicAdd(&s_fill, 1u);
            rk_key[pos] = key;
            rk_idx[pos] = i;
          }
        }
      }
      __syncthreads();
      if (tid < static_cast<int>(cnt)) {
        const uint32_t key = rk_key[tid];
        const int idx = rk_idx[tid];
        unsigned int rank = 0u, greater = 0u;
        for (unsigned int c = 0; c < cnt; ++c) {
          const uint32_t kc = rk_key[c];
          greater += kc > key ? 1u : 0u;
          rank += (kc > key || (kc == key && rk_idx[c] < idx)) ? 1u : 0u;
        }
        if (rank == krem - 1u) {
          s_lo = key;
          s_above = greater;
        }
      }
      __syncthreads();
      lo = hi = s_lo;
      krem -= s_above;
      break;
    }
  }

  // Output in ascending page order: warp w walks its chunk of pages with
  // ballots; a taken page's slot = #{greater before} + min(#{equal before}, krem).
  const uint32_t kth = lo;
  const int cw = (((P + kTopkWarps - 1) / kTopkWarps) + 31) & ~31;
  const int c0 = warp * cw, c1 = min(P, c0 + cw);
  unsigned int ng = 0u, ne = 0u;
  for (int i0 = c0; i0 < c1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < c1 ? key_at(i) : 0u;
    ng += __popc(__ballot_sync(0xffffffffu, i < c1 && key > kth));
    ne += __popc(__ballot_sync(0xffffffffu, i < c1 && key == kth));
  }
  __syncthreads();  // w_a / w_b were read above
  if (lane == 0) {
    w_a[warp] = ng;
    w_b[warp] = ne;
  }
  __syncthreads();
  unsigned int xg = w_a[lane], xe = w_b[lane], ig = xg, ie = xe;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int yg = __shfl_up_sync(0xffffffffu, ig, o);
    const unsigned int ye = __shfl_up_sync(0xffffffffu, ie, o);
    if (lane >= o) {
      ig += yg;
      ie += ye;
    }
  }
  unsigned int gt_before = __shfl_sync(0xffffffffu, ig - xg, warp);
  unsigned int eq_before = __shfl_sync(0xffffffffu, ie - xe, warp);
  const unsigned int lower = (1u << lane) - 1u;
  for (int i0 = c0; i0 < c1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < c1 ? key_at(i) : 0u;
    const bool gt = i < c1 && key > kth, eq = i < c1 && key == kth;
    const unsigned int bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const unsigned int my_g = gt_before + __popc(bg & lower), my_e = eq_before + __popc(be & lower);
    if (gt) {
      const unsigned int pos = my_g + min(my_e, krem);
      if (pos < static_cast<unsigned int>(k)) out[pos] = idx_of(i);
    } else if (eq && my_e < krem) {
      const unsigned int pos = my_g + my_e;
      if (pos < static_cast<unsigned int>(k)) out[pos] = idx_of(i);
    }
    gt_before += __popc(bg);
    eq_before += __popc(be);
  }
  if (tid == 0) *n_out = k;
}

// One unit per CTA (units of at most kSmemKeys pages).
__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                int max_pages, int Hkv, int k, int stride, int32_t* __restrict__ sel,
                int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  extern __shared__ uint32_t keys_s[];  // [min(max_pages, kSmemKeys)]
  const int unit = blockIdx.x, b = unit / Hkv, tid = threadIdx.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  int32_t* out = sel + static_cast<size_t>(unit) * stride;
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  if (P <= k) {
    for (int i = tid; i < P; i += kTopkThreads) out[i] = i;
    if (tid == 0) n_sel[unit] = P;
    return;
  }
  select_k(P, k, [&](int i) { return float_key(row[i]); }, [](int i) { return i; }, keys_s,
           P <= kSmemKeys, out, n_sel + unit);
}

// First stage of a long unit: chunk c keeps its k best pages.
__global__ void __launch_bounds__(kTopkThreads)
    topk_chunk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                      int max_pages, int Hkv, int k, int chunk, int nchunk, int32_t* __restrict__ cand,
                      int32_t* __restrict__ ccount) {
  grid_dep_enter();
  extern __shared__ uint32_t keys_s[];  // [chunk]
  const int c = blockIdx.x, unit = blockIdx.y, b = unit / Hkv, tid = threadIdx.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  const int base = c * chunk, n = max(0, min(chunk, P - base));
  int32_t* out = cand + (static_cast<size_t>(unit) * nchunk + c) * k;
  int32_t* cnt = ccount + static_cast<size_t>(unit) * nchunk + c;
  if (n <= k) {
    for (int i = tid; i < n; i += kTopkThreads) out[i] = base + i;
    if (tid == 0) *cnt = n;
    return;
  }
  const float* row = ub + static_cast<size_t>(unit) * max_pages + base;
  select_k(n, k, [&](int i) { return float_key(row[i]); }, [&](int i) { return base + i; }, keys_s, true,
           out, cnt);
}

// Second stage: the unit's k best among its chunks' winners (in page order).
__global__ void __launch_bounds__(kTopkThreads)
    topk_merge_kernel(const float* __restrict__ ub, int max_pages, int k, int nchunk,
                      const int32_t* __restrict__ cand, const int32_t* __restrict__ ccount, int stride,
                      int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  extern __shared__ uint32_t dyn_m[];  // [nchunk·k] page indices, then [nchunk·k] keys
  __shared__ int s_off[65];
  const int unit = blockIdx.x, tid = threadIdx.x;
  int* cl = reinterpret_cast<int*>(dyn_m);
  uint32_t* keys_s = dyn_m + static_cast<size_t>(nchunk) * k;
  if (tid == 0) {
    int o = 0;
    for (int c = 0; c < nchunk; ++c) {
      s_off[c] = o;
      o += max(0, min(k, ccount[static_cast<size_t>(unit) * nchunk + c]));
    }
    s_off[nchunk] = o;
  }
  __syncthreads();
  for (int c = 0; c < nchunk; ++c) {
    const int n = s_off[c + 1] - s_off[c];
    const int32_t* src = cand + (static_cast<size_t>(unit) * nchunk + c) * k;
    for (int i = tid; i < n; i += kTopkThreads) cl[s_off[c] + i] = src[i];
  }
  __syncthreads();
  const int n2 = s_off[nchunk];
  int32_t* out = sel + static_cast<size_t>(unit) * stride;
  if (n2 <= k) {
    for (int i = tid; i < n2; i += kTopkThreads) out[i] = cl[i];
    if (tid == 0) n_sel[unit] = n2;
    return;
  }
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  select_k(n2, k, [&](int i) { return float_key(row[cl[i]]); }, [&](int i) { return cl[i]; }, keys_s, true,
           out, n_sel + unit);
}

}  // namespace

// Two-stage plan: chunk pages per first-stage CTA (0: one stage).  Only
// units whose keys exceed one CTA's cache split (measured: splitting shorter
// units to fill the GPU costs more in the second launch and its barriers
// than it saves).
struct TopkPlan {
  int chunk, nchunk;
};

TopkPlan topk_plan(int units, int max_pages, int k) {
  (void)units;
  TopkPlan pl{0, 1};
  if (max_pages <= kSmemKeys) return pl;
  const int nchunk = (max_pages + kChunk - 1) / kChunk;
  if (nchunk > 64 || static_cast<size_t>(nchunk) * k > static_cast<size_t>(kSmemKeys)) return pl;
  const int chunk = ((max_pages + nchunk - 1) / nchunk + 31) / 32 * 32;
  pl.chunk = chunk;
  pl.nchunk = (max_pages + chunk - 1) / chunk;
  return pl;
}

size_t topk_ws_bytes(int units, int max_pages, int k) {
  const TopkPlan pl = topk_plan(units, max_pages, k);
  if (pl.chunk == 0) return 0;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return al(static_cast<size_t>(units) * pl.nchunk * k * sizeof(int32_t)) +
         al(static_cast<size_t>(units) * pl.nchunk * sizeof(int32_t));
}

size_t topk_ws_bytes_upto(int units, int max_pages, int cap) {
  size_t most = 0;
  for (int k = 1; k <= cap && k <= max_pages; ++k) {
    const size_t b = topk_ws_bytes(units, max_pages, k);
    if (b > most) most = b;
  }
  return most;
}

cudaError_t launch_topk(const ekv_seqs& s, int Hkv, int S, const float* ub, int k, int stride,
                        int32_t* sel, int32_t* n_sel, void* ws, cudaStream_t st) {
  const int U = s.batch * Hkv;
  const size_t static_smem = 2 * kBins * sizeof(unsigned int) + kRankMax * 8 + 1024;
  const TopkPlan pl = topk_plan(U, s.max_pages, k);
  if (ws != nullptr && pl.chunk > 0) {
    const int nchunk = pl.nchunk;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    int32_t* cand = static_cast<int32_t*>(ws);
    int32_t* ccount = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + al(static_cast<size_t>(U) * nchunk * k * sizeof(int32_t)));
    const size_t smem1 = static_cast<size_t>(pl.chunk) * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem1));
    if (e != cudaSuccess) return e;
    e = launch_k(topk_chunk_kernel, dim3(nchunk, U), dim3(kTopkThreads), smem1, st, ub, s.seq_lens, S,
                 s.max_pages, Hkv, k, pl.chunk, nchunk, cand, ccount);
    if (e != cudaSuccess) return e;
    const size_t smem2 = 2 * static_cast<size_t>(nchunk) * k * sizeof(uint32_t);
    if (smem2 + static_smem > 48 * 1024) {
      e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem2));
      if (e != cudaSuccess) return e;
    }
    e = launch_k(topk_merge_kernel, dim3(U), dim3(kTopkThreads), smem2, st, ub, s.max_pages, k, nchunk,
                 cand, ccount, stride, sel, n_sel);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const int keys = s.max_pages < kSmemKeys ? s.max_pages : kSmemKeys;
  const size_t smem = static_cast<size_t>(keys) * sizeof(uint32_t);
  if (smem + static_smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t le = launch_k(topk_kernel, dim3(U), dim3(kTopkThreads), smem, st, ub,
                                  s.seq_lens, S, s.max_pages, Hkv, k, stride, sel, n_sel);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

}  // namespace ekv
