// Top-k page selection — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.B, "Sélection de Pages Top-k": per (sequence, KV head), the k
// pages with the largest bounding-box score, ties to the lower logical page.
//
// One CTA per list.  Scores become order-preserving uint32 keys.  A list of
// at most kRegKeys entries is held in registers, each thread owning a
// contiguous run of 8 or 16 positions; a unit with more pages than that is
// done in two stages: chunks of pages each keep their own k best (any page of
// the unit's k best is among its chunk's k best under the same order), then
// one CTA selects k among those winners, read through their page indices, so
// ties and order are unchanged.  The k-th largest key K* is found by a radix
// select whose digits adapt to the keys: each pass bins the keys of the
// current interval [lo, hi] into at most 4096 equal bins that span exactly
// that interval (bin = (key − lo) >> shift), so scores spread over all bins
// instead of piling into the few bins their exponent bits would give.  The bin
// holding the k-th largest key becomes the next interval; once it holds few
// keys they are ranked directly, and a pass with shift 0 leaves a single key
// value, K*, after at most three passes.  The output gives each thread its run
// of positions: one block scan of (#key > K*, #key = K*) places every key
// > K* and the lowest-position (k − #{key > K*}) keys equal to K* in ascending
// page order.  All arithmetic on keys is integer.
#include "select_k.cuh"

namespace ekv {

namespace {

using Sel = Select<1024, 4096>;
using SelectShared = Sel::SelectShared;
constexpr int kTopkThreads = Sel::kTopkThreads;
constexpr int kRegKeys = Sel::kRegKeys;
constexpr int kChunk = 8192;                  // pages per first-stage chunk of a long unit

// Short lists (at most kShortList pages per sequence): 256 threads, 4 keys
// each, 1024 bins, so that many units' CTAs are resident at once.
using SelShort = Select<256, 1024, 1024>;
constexpr int kShortList = SelShort::kKeysPerThread * SelShort::kTopkThreads;

// One unit per CTA.
template <class SelT>
__global__ void __launch_bounds__(SelT::kTopkThreads)
    topk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                int max_pages, int Hkv, int k, int stride, int32_t* __restrict__ sel,
                int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  __shared__ typename SelT::SelectShared sh;
  const int unit = blockIdx.x, b = unit / Hkv, tid = threadIdx.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  int32_t* out = sel + static_cast<size_t>(unit) * stride;
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  if (P <= k) {
    for (int i = tid; i < P; i += SelT::kTopkThreads) out[i] = i;
    if (tid == 0) n_sel[unit] = P;
    return;
  }
  SelT::select_k(sh, P, k, RowKeys{row}, [](int i) { return i; }, out, n_sel + unit);
}

// First stage of a long unit: chunk c keeps its k best pages.
__global__ void __launch_bounds__(kTopkThreads)
    topk_chunk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                      int max_pages, int Hkv, int k, int chunk, int nchunk, int32_t* __restrict__ cand,
                      int32_t* __restrict__ ccount) {
  grid_dep_enter();
  __shared__ SelectShared sh;
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
  Sel::select_k(sh, n, k, RowKeys{row}, [&](int i) { return base + i; }, out, cnt);
}

// Second stage: the unit's k best among its chunks' winners (in page order).
__global__ void __launch_bounds__(kTopkThreads)
    topk_merge_kernel(const float* __restrict__ ub, int max_pages, int k, int nchunk,
                      const int32_t* __restrict__ cand, const int32_t* __restrict__ ccount, int stride,
                      int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  extern __shared__ int cl[];  // [nchunk·k] page indices of the chunks' winners
  __shared__ SelectShared sh;
  __shared__ int s_off[65];
  const int unit = blockIdx.x, tid = threadIdx.x;
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
  Sel::select_k(sh, n2, k, ListKeys{row, cl}, [&](int i) { return cl[i]; }, out, n_sel + unit);
}

}  // namespace

// Two-stage plan: chunk pages per first-stage CTA (0: one stage).  Only
// units whose keys exceed one CTA's registers split (measured: splitting shorter
// units to fill the GPU costs more in the second launch and its barriers
// than it saves).
struct TopkPlan {
  int chunk, nchunk;
};

TopkPlan topk_plan(int units, int max_pages, int k) {
  (void)units;
  TopkPlan pl{0, 1};
  if (max_pages <= kRegKeys) return pl;
  const int nchunk = (max_pages + kChunk - 1) / kChunk;
  if (nchunk > 64 || static_cast<size_t>(nchunk) * k > static_cast<size_t>(kRegKeys)) return pl;
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
  const TopkPlan pl = topk_plan(U, s.max_pages, k);
  if (ws != nullptr && pl.chunk > 0) {
    const int nchunk = pl.nchunk;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    int32_t* cand = static_cast<int32_t*>(ws);
    int32_t* ccount = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + al(static_cast<size_t>(U) * nchunk * k * sizeof(int32_t)));
    cudaError_t e = launch_k(topk_chunk_kernel, dim3(nchunk, U), dim3(kTopkThreads), 0, st, ub, s.seq_lens, S,
                             s.max_pages, Hkv, k, pl.chunk, nchunk, cand, ccount);
    if (e != cudaSuccess) return e;
    const size_t smem2 = static_cast<size_t>(nchunk) * k * sizeof(int32_t);
    if (smem2 + sizeof(SelectShared) + 512 > 48 * 1024) {
      e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem2));
      if (e != cudaSuccess) return e;
    }
    e = launch_k(topk_merge_kernel, dim3(U), dim3(kTopkThreads), smem2, st, ub, s.max_pages, k, nchunk,
                 cand, ccount, stride, sel, n_sel);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const cudaError_t le =
      s.max_pages <= kShortList
          ? launch_k(topk_kernel<SelShort>, dim3(U), dim3(SelShort::kTopkThreads), 0, st, ub, s.seq_lens, S,
                     s.max_pages, Hkv, k, stride, sel, n_sel)
          : launch_k(topk_kernel<Sel>, dim3(U), dim3(kTopkThreads), 0, st, ub, s.seq_lens, S, s.max_pages, Hkv, k,
                     stride, sel, n_sel);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

}  // namespace ekv
