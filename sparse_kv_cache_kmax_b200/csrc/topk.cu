// Top-k page selection — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.B, "Sélection de Pages Top-k": per (sequence, KV head), the k
// pages with the largest bounding-box score, ties to the lower logical page.
//
// One CTA per unit.  Scores are mapped to order-preserving uint32 keys and the
// k-th largest key K* is found by a 4 × 8-bit most-significant-digit radix
// select (histogram of the surviving prefix, suffix count from the top).  A
// final pass in ascending page order takes every key > K* plus the first
// (k − #{key > K*}) keys equal to K*, so the output is sorted by page index
// and the tie rule is exact.  All arithmetic on keys is integer.
#include "kernels.cuh"

namespace ekv {

namespace {

constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const float* __restrict__ ub, const int32_t* __restrict__ seq_lens, int S,
                int max_pages, int Hkv, int k, int stride, int32_t* __restrict__ sel,
                int32_t* __restrict__ n_sel) {
  const int unit = blockIdx.x, b = unit / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  int32_t* out = sel + static_cast<size_t>(unit) * stride;
  const float* row = ub + static_cast<size_t>(unit) * max_pages;
  if (P <= k) {
    for (int i = tid; i < P; i += blockDim.x) out[i] = i;
    if (tid == 0) n_sel[unit] = P;
    return;
  }

  __shared__ unsigned int hist[256];
  __shared__ unsigned int s_digit, s_above;
  __shared__ int scan_scratch[32];
  unsigned int prefix = 0u, mask = 0u, krem = static_cast<unsigned int>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < P; i += blockDim.x) {
      const uint32_t key = float_key(row[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l covers digits 255−8l … 248−8l, scanned from the top
      unsigned int c[8], local = 0u;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        c[r] = hist[255 - 8 * lane - r];
        local += c[r];
      }
      unsigned int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned int hit = __ballot_sync(0xffffffffu, incl >= krem);
      const int target = __ffs(hit) - 1;
      if (lane == target) {
        unsigned int before = incl - local;
        int r = 0;
        while (r < 7 && before + c[r] < krem) before += c[r++];
        s_digit = static_cast<unsigned int>(255 - 8 * lane - r);
        s_above = before;
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    krem -= s_above;
    __syncthreads();
  }

  // ascending pass: keys > K*, then the lowest-index keys == K*
  const uint32_t kth = prefix;
  int carry_take = 0, carry_eq = 0;
  for (int base = 0; base < P; base += blockDim.x) {
    const int i = base + tid;
    const uint32_t key = i < P ? float_key(row[i]) : 0u;
    const int gt = (i < P && key > kth) ? 1 : 0;
    const int eq = (i < P && key == kth) ? 1 : 0;
    int eq_total, take_total;
    const int eq_rank = block_exclusive_scan(eq, scan_scratch, &eq_total) + carry_eq;
    const int take = gt | (eq & (eq_rank < static_cast<int>(krem) ? 1 : 0));
    const int pos = block_exclusive_scan(take, scan_scratch, &take_total) + carry_take;
    if (take && pos < k) out[pos] = i;
    carry_eq += eq_total;
    carry_take += take_total;
  }
  if (tid == 0) n_sel[unit] = k;
}

}  // namespace

cudaError_t launch_topk(const ekv_seqs& s, int Hkv, int S, const float* ub, int k, int stride,
                        int32_t* sel, int32_t* n_sel, cudaStream_t st) {
  topk_kernel<<<s.batch * Hkv, kTopkThreads, 0, st>>>(ub, s.seq_lens, S, s.max_pages, Hkv, k,
                                                       stride, sel, n_sel);
  return cudaGetLastError();
}

}  // namespace ekv
