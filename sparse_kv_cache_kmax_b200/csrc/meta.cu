// Per-page key metadata — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.A: coordinate-wise k_min / k_max (the bounding box) and the
// first and second moments (mean, variance) of a page's keys.
//
// One thread owns one coordinate pair of one (page, KV head) and walks the
// page's valid tokens in order.  k_max / k_min are exact; the mean and the
// population variance are accumulated in float64 with explicit
// round-to-nearest operations (no contraction into FMA) in token order, then
// rounded once to the cache dtype, so the result is a fixed function of the
// stored keys.
#include "kernels.cuh"

namespace ekv {

namespace {

template <typename T>
struct Pair;
template <>
struct Pair<bf16> {
  __device__ static void load(const bf16* p, float& a, float& b) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    a = __uint_as_float(w << 16);
    b = __uint_as_float(w & 0xffff0000u);
  }
  __device__ static void store(bf16* p, double a, double b) {
    const uint32_t w = static_cast<uint32_t>(f64_to_bf16_bits(a)) |
                       (static_cast<uint32_t>(f64_to_bf16_bits(b)) << 16);
    *reinterpret_cast<uint32_t*>(p) = w;
  }
  __device__ static void store_exact(bf16* p, float a, float b) {
    const uint32_t w = (__float_as_uint(a) >> 16) | (__float_as_uint(b) & 0xffff0000u);
    *reinterpret_cast<uint32_t*>(p) = w;
  }
  __device__ static void copy(bf16* dst, const bf16* src) {
    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(src);
  }
};
template <>
struct Pair<float> {
  __device__ static void load(const float* p, float& a, float& b) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    a = v.x;
    b = v.y;
  }
  __device__ static void store(float* p, double a, double b) {
    *reinterpret_cast<float2*>(p) = make_float2(__double2float_rn(a), __double2float_rn(b));
  }
  __device__ static void store_exact(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
  }
  __device__ static void copy(float* dst, const float* src) {
    *reinterpret_cast<float2*>(dst) = *reinterpret_cast<const float2*>(src);
  }
};

// Metadata of one coordinate pair over tokens 0..n-1 of a page (1 ≤ n ≤ 32).
// When `inject` ≥ 0, token `inject` takes the values (xa, xb) instead of the
// pool.  The page's values are loaded first as one batch of independent,
// unconditional loads (a token past n reads token 0 again and is dropped):
// loads behind per-token branches were issued one after another.
template <typename T>
__device__ void page_pair_meta(const T* page_k, int D, int n, int j, int inject, float xa,
                               float xb, T* box_row, T* mom_row) {
  float va[32], vb[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const int tt = t < n ? t : 0;
    float a, b;
    Pair<T>::load(page_k + static_cast<size_t>(tt) * D + j, a, b);
    va[t] = t < n ? (t == inject ? xa : a) : 0.f;
    vb[t] = t < n ? (t == inject ? xb : b) : 0.f;
  }
  float mx0 = -INFINITY, mx1 = -INFINITY, mn0 = INFINITY, mn1 = INFINITY;
  double s0 = 0.0, s1 = 0.0;
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    if (t < n) {
      mx0 = fmaxf(mx0, va[t]);
      mx1 = fmaxf(mx1, vb[t]);
      mn0 = fminf(mn0, va[t]);
      mn1 = fminf(mn1, vb[t]);
      s0 = __dadd_rn(s0, static_cast<double>(va[t]));
      s1 = __dadd_rn(s1, static_cast<double>(vb[t]));
    }
  }
  const double dn = static_cast<double>(n);
  const double m0 = __ddiv_rn(s0, dn), m1 = __ddiv_rn(s1, dn);
  double v0 = 0.0, v1 = 0.0;
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    if (t < n) {
      const double d0 = __dsub_rn(static_cast<double>(va[t]), m0);
      const double d1 = __dsub_rn(static_cast<double>(vb[t]), m1);
      v0 = __dadd_rn(v0, __dmul_rn(d0, d0));
      v1 = __dadd_rn(v1, __dmul_rn(d1, d1));
    }
  }
  Pair<T>::store_exact(box_row + j, mx0, mx1);           // k_max row
  Pair<T>::store_exact(box_row + D + j, mn0, mn1);       // k_min row
  Pair<T>::store(mom_row + j, m0, m1);                   // mean row
  Pair<T>::store(mom_row + D + j, __ddiv_rn(v0, dn), __ddiv_rn(v1, dn));  // variance row
}

// grid: (page slice, batch, Hkv); block: D/2 threads.
template <typename T>
__global__ void build_meta_kernel(const T* __restrict__ k_pool, T* __restrict__ box,
                                  T* __restrict__ mom, const int32_t* __restrict__ page_table,
                                  const int32_t* __restrict__ seq_lens, int D, int S, int Hkv,
                                  int num_phys, int max_pages) {
  grid_dep_enter();
  const int b = blockIdx.y;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  const int h = blockIdx.z;
  const int j = 2 * threadIdx.x;
  for (int p = blockIdx.x; p < P; p += gridDim.x) {
    const int phys = page_table[static_cast<size_t>(b) * max_pages + p];
    if (!phys_ok(phys, num_phys)) continue;
    const int n = min(S, L - p * S);
    const size_t ph = static_cast<size_t>(phys) * Hkv + h;
    const size_t mh = static_cast<size_t>(h) * num_phys + phys;  // head-major metadata row
    page_pair_meta<T>(k_pool + ph * S * D, D, n, j, -1, 0.f, 0.f, box + mh * 2 * D,
                      mom + mh * 2 * D);
  }
}

// grid: (batch, Hkv); block: D/2 threads.  Token L−1 of sequence b.
template <typename T>
__global__ void append_kernel(T* __restrict__ k_pool, T* __restrict__ v_pool, T* __restrict__ box,
                              T* __restrict__ mom, const int32_t* __restrict__ page_table,
                              const int32_t* __restrict__ seq_lens, const T* __restrict__ k_new,
                              const T* __restrict__ v_new, int D, int S, int Hkv, int num_phys,
                              int max_pages) {
  grid_dep_enter();
  const int b = blockIdx.x;
  int L;
  seq_pages(seq_lens, b, S, max_pages, &L);
  if (L < 1) return;
  const int pos = L - 1, p = pos / S, slot = pos % S;
  const int phys = page_table[static_cast<size_t>(b) * max_pages + p];
  if (!phys_ok(phys, num_phys)) return;
  const int h = blockIdx.y;
  const int j = 2 * threadIdx.x;
  const size_t ph = static_cast<size_t>(phys) * Hkv + h;
  const size_t src = (static_cast<size_t>(b) * Hkv + h) * D + j;
  float xa, xb;
  Pair<T>::load(k_new + src, xa, xb);
  Pair<T>::copy(k_pool + (ph * S + slot) * D + j, k_new + src);
  Pair<T>::copy(v_pool + (ph * S + slot) * D + j, v_new + src);
  const size_t mh = static_cast<size_t>(h) * num_phys + phys;  // head-major metadata row
  page_pair_meta<T>(k_pool + ph * S * D, D, slot + 1, j, slot, xa, xb, box + mh * 2 * D,
                    mom + mh * 2 * D);
}

}  // namespace

cudaError_t launch_build_meta(const ekv_cache& c, const ekv_seqs& s, cudaStream_t st) {
  const int threads = c.head_dim / 2;
  const dim3 grid(static_cast<unsigned>(min(s.max_pages, 4096)), static_cast<unsigned>(s.batch),
                  static_cast<unsigned>(c.num_kv_heads));
  if (c.dtype == EKV_BF16)
    {
    const cudaError_t le_ = launch_k(build_meta_kernel<bf16>, grid, threads, 0, st, 
        static_cast<const bf16*>(c.k_pool), static_cast<bf16*>(c.box), static_cast<bf16*>(c.mom),
        s.page_table, s.seq_lens, c.head_dim, c.page_size, c.num_kv_heads, c.num_phys_pages,
        s.max_pages);
    if (le_ != cudaSuccess) return le_;
  }
  else
    {
    const cudaError_t le_ = launch_k(build_meta_kernel<float>, grid, threads, 0, st, 
        static_cast<const float*>(c.k_pool), static_cast<float*>(c.box),
        static_cast<float*>(c.mom), s.page_table, s.seq_lens, c.head_dim, c.page_size,
        c.num_kv_heads, c.num_phys_pages, s.max_pages);
    if (le_ != cudaSuccess) return le_;
  }
  return cudaGetLastError();
}

cudaError_t launch_append(const ekv_cache& c, const ekv_seqs& s, const void* k_new,
                          const void* v_new, cudaStream_t st) {
  const int threads = c.head_dim / 2;
  const dim3 grid(static_cast<unsigned>(s.batch), static_cast<unsigned>(c.num_kv_heads));
  if (c.dtype == EKV_BF16)
    {
    const cudaError_t le_ = launch_k(append_kernel<bf16>, grid, threads, 0, st, 
        static_cast<bf16*>(c.k_pool), static_cast<bf16*>(c.v_pool), static_cast<bf16*>(c.box),
        static_cast<bf16*>(c.mom), s.page_table, s.seq_lens, static_cast<const bf16*>(k_new),
        static_cast<const bf16*>(v_new), c.head_dim, c.page_size, c.num_kv_heads,
        c.num_phys_pages, s.max_pages);
    if (le_ != cudaSuccess) return le_;
  }
  else
    {
    const cudaError_t le_ = launch_k(append_kernel<float>, grid, threads, 0, st, 
        static_cast<float*>(c.k_pool), static_cast<float*>(c.v_pool), static_cast<float*>(c.box),
        static_cast<float*>(c.mom), s.page_table, s.seq_lens, static_cast<const float*>(k_new),
        static_cast<const float*>(v_new), c.head_dim, c.page_size, c.num_kv_heads,
        c.num_phys_pages, s.max_pages);
    if (le_ != cudaSuccess) return le_;
  }
  return cudaGetLastError();
}

}  // namespace ekv
