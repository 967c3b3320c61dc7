// Radix selection of the k largest keys of a list by one CTA of THREADS
// threads with BINS histogram bins, used by the top-k kernels (topk.cu) —
// EntmaxKV summary page
// (gist.science/fr/paper/2605.21649) §2.B "Sélection de Pages Top-k": the k
// pages with the largest bound, ties to the lower page, ascending.
//
// Scores become order-preserving uint32 keys.  The k-th largest key K* is
// found by a radix select whose digits adapt to the keys: each pass bins the
// keys of the current interval [lo, hi] into at most BINS equal bins that
// span exactly that interval (bin = (key − lo) >> shift), so scores spread
// over all bins instead of piling into the few bins their exponent bits
// would give.  The bin holding the k-th largest key becomes the next
// interval; once it holds few keys they are ranked directly, and a pass with
// shift 0 leaves a single key value, K*.  The output gives each thread its
// run of positions: one block scan of (#key > K*, #key = K*) places every key
// > K* and the lowest-position (k − #{key > K*}) keys equal to K* in
// ascending position order.  All arithmetic on keys is integer.
#pragma once

#include "kernels.cuh"

namespace ekv {

// Keys of a contiguous row of scores.
struct RowKeys {
  const float* row;
  __device__ uint32_t operator()(int i) const { return float_key(row[i]); }
  template <int KPT>
  __device__ void load(int i0, int n, uint32_t (&key)[KPT]) const {
    const float* src = row + i0;
    if (i0 + KPT <= n && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
#pragma unroll
      for (int v = 0; v < KPT / 4; ++v) {
        const float4 f = reinterpret_cast<const float4*>(src)[v];
        key[4 * v] = float_key(f.x);
        key[4 * v + 1] = float_key(f.y);
        key[4 * v + 2] = float_key(f.z);
        key[4 * v + 3] = float_key(f.w);
      }
    } else {
#pragma unroll
      for (int j = 0; j < KPT; ++j) key[j] = i0 + j < n ? float_key(src[j]) : 0u;
    }
  }
};

// Keys of scattered entries of a row, read through a list of page indices.
struct ListKeys {
  const float* row;
  const int* list;
  __device__ uint32_t operator()(int i) const { return float_key(row[list[i]]); }
  template <int KPT>
  __device__ void load(int i0, int n, uint32_t (&key)[KPT]) const {
#pragma unroll
    for (int j = 0; j < KPT; ++j) key[j] = i0 + j < n ? float_key(row[list[i0 + j]]) : 0u;
  }
};


template <int THREADS, int BINS, int LIST = 8192>
struct Select {
  static constexpr int kTopkThreads = THREADS;
  static constexpr int kTopkWarps = THREADS / 32;
  static constexpr int kKeysPerThread = LIST / THREADS;            // registers per thread for lists ≤ LIST
  static constexpr int kRegKeys = 2 * kKeysPerThread * THREADS;    // longest list held in registers
  static constexpr int kBins = BINS;
  static constexpr int kDigitBits = BINS == 4096 ? 12 : (BINS == 2048 ? 11 : 10);
  static constexpr int kRankMax = 256;  // keys of the k-th key's bin ranked directly
  static_assert(THREADS >= kRankMax && THREADS <= 1024 && THREADS % 32 == 0, "block size");
  static_assert(BINS % THREADS == 0 && LIST % THREADS == 0 && (1 << kDigitBits) == BINS, "bins and keys per thread");

struct SelectShared {
  unsigned int hist[2][kBins];
  unsigned int w_a[kTopkWarps], w_b[kTopkWarps];
  uint32_t rk_key[kRankMax];
  int rk_idx[kRankMax];
  unsigned int rk_rank[kRankMax];
  unsigned int s_lo, s_hi, s_above, s_count, s_fill;
};

// The interval [lo, hi] holds the k-th largest key with krem keys of it
// still to take: bins its keys (count_bins(hc, lo, shift) adds every key of
// the interval to hc), then moves [lo, hi] to the bin of the k-th key.  The
// whole CTA calls it; returns the bin's key count.
template <class CountBins>
static __device__ unsigned int narrow(SelectShared& sh, int cur, unsigned int& lo, unsigned int& hi,
                               unsigned int& krem, CountBins count_bins) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned int range = hi - lo;
  const int width = 32 - __clz(range);
  const int shift = width > kDigitBits ? width - kDigitBits : 0;
  const int top = static_cast<int>(range >> shift);
  unsigned int* hc = sh.hist[cur];
  count_bins(hc, lo, hi, shift);
  for (int i = tid; i < kBins; i += kTopkThreads) sh.hist[cur ^ 1][i] = 0u;  // next pass's bins
  __syncthreads();
  // thread t covers bins top − 4t − r (r = 0..3), counted from the top
  unsigned int c[kBins / kTopkThreads], mine = 0u;
#pragma unroll
  for (int r = 0; r < kBins / kTopkThreads; ++r) {
    const int bin = top - (kBins / kTopkThreads) * tid - r;
    c[r] = bin >= 0 ? hc[bin] : 0u;
    mine += c[r];
  }
  unsigned int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.w_a[warp] = incl;
  __syncthreads();
  const unsigned int wt = lane < kTopkWarps ? sh.w_a[lane] : 0u;
  unsigned int wincl = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, wincl, o);
    if (lane >= o) wincl += y;
  }
  unsigned int before = __shfl_sync(0xffffffffu, wincl - wt, warp) + incl - mine;
  if (before < krem && before + mine >= krem) {  // this thread holds the k-th key's bin
#pragma unroll
    for (int r = 0; r < kBins / kTopkThreads; ++r) {
      if (before < krem && before + c[r] >= krem) {
        const int bin = top - (kBins / kTopkThreads) * tid - r;
        sh.s_above = before;
        sh.s_count = c[r];
        const unsigned long long base =
            static_cast<unsigned long long>(lo) + (static_cast<unsigned long long>(bin) << shift);
        sh.s_lo = static_cast<unsigned int>(base);
        sh.s_hi = static_cast<unsigned int>(min(static_cast<unsigned long long>(hi), base + ((1ull << shift) - 1ull)));
      }
      before += c[r];
    }
  }
  if (tid == 0) sh.s_fill = 0u;
  __syncthreads();
  krem -= sh.s_above;
  lo = sh.s_lo;
  hi = sh.s_hi;
  return sh.s_count;
}

// K* from the cnt ≤ kRankMax keys in [lo, hi] gathered into rk_key/rk_idx:
// ranked by (key descending, position ascending), the one of rank krem − 1.
// The threads split into as many slices of the list as fit; each key's rank
// is the sum over the slices.
static __device__ void rank_bin(SelectShared& sh, unsigned int cnt, unsigned int& lo, unsigned int& hi,
                         unsigned int& krem) {
  const int tid = threadIdx.x;
  const int per = cnt <= 64u ? 64 : cnt <= 128u ? 128 : kRankMax;
  const int nslice = kTopkThreads / per;
  const int e = tid % per, slice = tid / per;
  if (e < static_cast<int>(cnt) && slice < nslice) {
    const uint32_t key = sh.rk_key[e];
    const int idx = sh.rk_idx[e];
    const unsigned int c0 = cnt * slice / nslice, c1 = cnt * (slice + 1) / nslice;
    unsigned int rank = 0u, greater = 0u;
    for (unsigned int c = c0; c < c1; ++c) {
      const uint32_t kc = sh.rk_key[c];
      greater += kc > key ? 1u : 0u;
      rank += (kc > key || (kc == key && sh.rk_idx[c] < idx)) ? 1u : 0u;
    }
    if (c1 > c0) atomicAdd(&sh.rk_rank[e], rank | (greater << 16));
  }
  __syncthreads();
  for (int i = tid; i < static_cast<int>(cnt); i += kTopkThreads) {
    const unsigned int rg = sh.rk_rank[i];
    if ((rg & 0xffffu) == krem - 1u) {
      sh.s_lo = sh.rk_key[i];
      sh.s_above = rg >> 16;
    }
  }
  __syncthreads();
  lo = hi = sh.s_lo;
  krem -= sh.s_above;
}

// The k largest of n entries (kRegKeys ≥ n > k; keys.load fills a thread's
// run of KPT positions), ties to the lower position; writes idx_of(position)
// of each, in ascending position order, to out[0..k) and k to *n_out.  The
// whole CTA calls it.
template <int KPT, class Keys, class IdxOf>
static __device__ void select_k_reg(SelectShared& sh, int n, int k, const Keys& keys, IdxOf idx_of,
                             int32_t* __restrict__ out, int32_t* __restrict__ n_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = tid * KPT;
  uint32_t key[KPT];
  keys.template load<KPT>(i0, n, key);
  const int nv = max(0, min(KPT, n - i0));  // valid positions of this thread
  unsigned int kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (j < nv) {
      kmin = min(kmin, key[j]);
      kmax = max(kmax, key[j]);
    }
  }
  for (int i = tid; i < kBins; i += kTopkThreads) sh.hist[0][i] = 0u;
  for (int i = tid; i < kRankMax; i += kTopkThreads) sh.rk_rank[i] = 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    sh.w_a[warp] = kmin;
    sh.w_b[warp] = kmax;
  }
  __syncthreads();
  kmin = lane < kTopkWarps ? sh.w_a[lane] : 0xffffffffu;
  kmax = lane < kTopkWarps ? sh.w_b[lane] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  __syncthreads();  // w_a / w_b are reused below

  unsigned int lo = kmin, hi = kmax, krem = static_cast<unsigned int>(k);
  int cur = 0;
#pragma unroll 1
  for (int pass = 0; pass < 4 && lo < hi; ++pass) {
    // neighbouring positions often share a bin: one atomic per run of them
    const unsigned int cnt = narrow(sh, cur, lo, hi, krem, [&](unsigned int* hc, unsigned int l, unsigned int h, int shift) {
      unsigned int prev = 0xffffffffu, run = 0u;
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        const bool in = j < nv && key[j] >= l && key[j] <= h;
        const unsigned int bin = in ? (key[j] - l) >> shift : 0xffffffffu;
        if (bin != prev) {
          if (prev != 0xffffffffu) atomicAdd(&hc[prev], run);
          prev = bin;
          run = 0u;
        }
        run += in ? 1u : 0u;
      }
      if (prev != 0xffffffffu) atomicAdd(&hc[prev], run);
    });
    cur ^= 1;
    if (lo < hi && cnt <= kRankMax) {
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        if (j < nv && key[j] >= lo && key[j] <= hi) {
          const unsigned int pos = atomicAdd(&sh.s_fill, 1u);
          sh.rk_key[pos] = key[j];
          sh.rk_idx[pos] = i0 + j;
        }
      }
      __syncthreads();
      rank_bin(sh, cnt, lo, hi, krem);
      break;
    }
  }

  // Output: this thread's run of positions, after a block scan of its counts
  // of keys > K* (low half) and = K* (high half); both stay below 2^16.
  const uint32_t kth = lo;
  unsigned int gt = 0u, eq = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    gt += (j < nv && key[j] > kth) ? 1u : 0u;
    eq += (j < nv && key[j] == kth) ? 1u : 0u;
  }
  const unsigned int mine = gt | (eq << 16);
  unsigned int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.w_b[warp] = incl;
  __syncthreads();
  const unsigned int wt = lane < kTopkWarps ? sh.w_b[lane] : 0u;
  unsigned int wincl = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, wincl, o);
    if (lane >= o) wincl += y;
  }
  const unsigned int before = __shfl_sync(0xffffffffu, wincl - wt, warp) + incl - mine;
  unsigned int g = before & 0xffffu, e = before >> 16;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (j < nv) {
      if (key[j] > kth) {
        const unsigned int pos = g + min(e, krem);
        if (pos < static_cast<unsigned int>(k)) out[pos] = idx_of(i0 + j);
        ++g;
      } else if (key[j] == kth) {
        if (e < krem) {
          const unsigned int pos = g + e;
          if (pos < static_cast<unsigned int>(k)) out[pos] = idx_of(i0 + j);
        }
        ++e;
      }
    }
  }
  if (tid == 0) *n_out = k;
}

// The same selection for lists longer than kRegKeys (no key cache: each pass
// re-reads the keys through key_of).  Positions are visited in strides of
// the block; the output walks each warp's contiguous chunk with ballots.
template <class KeyOf, class IdxOf>
static __device__ void select_k_long(SelectShared& sh, int P, int k, KeyOf key_of, IdxOf idx_of,
                              int32_t* __restrict__ out, int32_t* __restrict__ n_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned int kmin = 0xffffffffu, kmax = 0u;
  for (int i = tid; i < P; i += kTopkThreads) {
    const uint32_t key = key_of(i);
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  }
  for (int i = tid; i < kBins; i += kTopkThreads) sh.hist[0][i] = 0u;
  for (int i = tid; i < kRankMax; i += kTopkThreads) sh.rk_rank[i] = 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    sh.w_a[warp] = kmin;
    sh.w_b[warp] = kmax;
  }
  __syncthreads();
  kmin = lane < kTopkWarps ? sh.w_a[lane] : 0xffffffffu;
  kmax = lane < kTopkWarps ? sh.w_b[lane] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  __syncthreads();

  unsigned int lo = kmin, hi = kmax, krem = static_cast<unsigned int>(k);
  int cur = 0;
#pragma unroll 1
  for (int pass = 0; pass < 4 && lo < hi; ++pass) {
    const unsigned int cnt = narrow(sh, cur, lo, hi, krem, [&](unsigned int* hc, unsigned int l, unsigned int h, int shift) {
      for (int i = tid; i < P; i += kTopkThreads) {
        const uint32_t key = key_of(i);
        if (key >= l && key <= h) atomicAdd(&hc[(key - l) >> shift], 1u);
      }
    });
    cur ^= 1;
    if (lo < hi && cnt <= kRankMax) {
      for (int i = tid; i < P; i += kTopkThreads) {
        const uint32_t key = key_of(i);
        if (key >= lo && key <= hi) {
          const unsigned int pos = atomicAdd(&sh.s_fill, 1u);
          sh.rk_key[pos] = key;
          sh.rk_idx[pos] = i;
        }
      }
      __syncthreads();
      rank_bin(sh, cnt, lo, hi, krem);
      break;
    }
  }

  // warp w walks its chunk of pages with ballots; a taken page's slot =
  // #{greater before} + min(#{equal before}, krem).
  const uint32_t kth = lo;
  const int cw = (((P + kTopkWarps - 1) / kTopkWarps) + 31) & ~31;
  const int c0 = warp * cw, c1 = min(P, c0 + cw);
  unsigned int ng = 0u, ne = 0u;
  for (int i0 = c0; i0 < c1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < c1 ? key_of(i) : 0u;
    ng += __popc(__ballot_sync(0xffffffffu, i < c1 && key > kth));
    ne += __popc(__ballot_sync(0xffffffffu, i < c1 && key == kth));
  }
  if (lane == 0) {
    sh.w_a[warp] = ng;
    sh.w_b[warp] = ne;
  }
  __syncthreads();
  unsigned int xg = lane < kTopkWarps ? sh.w_a[lane] : 0u, xe = lane < kTopkWarps ? sh.w_b[lane] : 0u;
  unsigned int ig = xg, ie = xe;
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
    const uint32_t key = i < c1 ? key_of(i) : 0u;
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

// Dispatch on the list length.
template <class Keys, class IdxOf>
static __device__ void select_k(SelectShared& sh, int n, int k, const Keys& keys, IdxOf idx_of,
                         int32_t* __restrict__ out, int32_t* __restrict__ n_out) {
  if (k < 1) {
    if (threadIdx.x == 0) *n_out = 0;
    return;
  }
  if (n <= kKeysPerThread * kTopkThreads)
    select_k_reg<kKeysPerThread>(sh, n, k, keys, idx_of, out, n_out);
  else if (n <= kRegKeys)
    select_k_reg<2 * kKeysPerThread>(sh, n, k, keys, idx_of, out, n_out);
  else
    select_k_long(sh, n, k, keys, idx_of, out, n_out);
}

};

}  // namespace ekv
