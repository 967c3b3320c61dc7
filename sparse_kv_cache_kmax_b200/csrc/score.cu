// Streaming kernels over the per-page metadata rows — EntmaxKV summary page
// (gist.science/fr/paper/2605.21649) §2.A:
//   * page scoring with the bounding-box upper bound
//       ub_{p,h} = scale·Σ_j max(q_hj·kmin_pj, q_hj·kmax_pj)
//               = scale·(q⁺_h·kmax_p + q⁻_h·kmin_p),  q⁺ = max(q,0), q⁻ = min(q,0),
//     reduced to the KV head's page score max_h ub_{p,h};
//   * the Gaussian page statistics of §2.A/§2.B.2: m = scale·q_h·μ_p and
//     s² = scale²·Σ_j q_hj²·σ²_pj per query head.
//
// Both read one 2·d-element row per (page, KV head) — [kmax | kmin] or
// [mean | var] — which is the whole per-step HBM traffic of selection.  Each
// lane of a warp owns one fixed 8-element chunk of the row, so its G query
// heads' coefficients stay in registers for every page; a page's row is one
// coalesced 512 B (bf16, d = 128) read by one warp (two pages per warp for
// d = 64).  Rows are loaded NB pages ahead to keep enough bytes in flight,
// products run as packed fp32 FMAs, and the G per-lane partial sums are
// reduced across the row's lanes with a transposing butterfly.
#include "kernels.cuh"

namespace ekv {

namespace {

struct StreamArgs {
  const void* rows;          // box or mom pool
  const int32_t* page_table;
  const int32_t* seq_lens;
  const void* q;
  float* ub;                 // score: [U, max_pages]
  GaussWs gws;               // Gaussian statistics outputs
  float scale, am1, inv_beta;
  int Hkv, Hq, S, num_phys, max_pages, chunks;
};

template <typename T>
struct Raw8 {  // 8 raw elements
  static constexpr int kVec = sizeof(T) / 2;  // uint4 count: 1 (bf16) or 2 (fp32)
  uint4 v[kVec];
};

template <typename T>
__device__ __forceinline__ float2 raw_pair(const Raw8<T>& r, int i);
template <>
__device__ __forceinline__ float2 raw_pair<bf16>(const Raw8<bf16>& r, int i) {
  const uint32_t w = i == 0 ? r.v[0].x : i == 1 ? r.v[0].y : i == 2 ? r.v[0].z : r.v[0].w;
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <>
__device__ __forceinline__ float2 raw_pair<float>(const Raw8<float>& r, int i) {
  const uint4& a = r.v[i >> 1];
  return (i & 1) ? make_float2(__uint_as_float(a.z), __uint_as_float(a.w))
                 : make_float2(__uint_as_float(a.x), __uint_as_float(a.y));
}

template <typename T, int D, int G, bool GAUSS>
__global__ void __launch_bounds__(256) meta_stream_kernel(StreamArgs a) {
  constexpr int LPP = D / 4;         // lanes per row (8 elements each of the 2·D)
  constexpr int PPW = 32 / LPP;      // rows per warp step
  constexpr int NB = 8 / PPW;        // warp steps loaded ahead
  constexpr int PPC = 8 * PPW * NB;  // rows per CTA (= kStreamPagesPerCta)
  constexpr int HALF = LPP / 2;
  static_assert(PPC == kStreamPagesPerCta, "CTA tile must match the host's chunking");

  const int unit = blockIdx.y, b = unit / a.Hkv, h = unit % a.Hkv;
  int L;
  const int P = seq_pages(a.seq_lens, b, a.S, a.max_pages, &L);
  const int p_begin = blockIdx.x * PPC;
  if (p_begin >= P) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ps = lane / LPP, wl = lane % LPP;
  const int e0 = wl * 8;
  const bool first = e0 < D;  // kmax / mean half of the row
  const int j0 = first ? e0 : e0 - D;

  float2 coef[G][4];
  {
    const T* qb = static_cast<const T*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(h) * G) * D + j0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float v[8];
      load8(qb + static_cast<size_t>(g) * D, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float c0, c1;
        if constexpr (GAUSS) {
          c0 = first ? v[2 * i] : v[2 * i] * v[2 * i];
          c1 = first ? v[2 * i + 1] : v[2 * i + 1] * v[2 * i + 1];
        } else {
          c0 = first ? fmaxf(v[2 * i], 0.f) : fminf(v[2 * i], 0.f);
          c1 = first ? fmaxf(v[2 * i + 1], 0.f) : fminf(v[2 * i + 1], 0.f);
        }
        coef[g][i] = make_float2(c0, c1);
      }
    }
  }

  Raw8<T> raw[NB];
  bool live[NB];
#pragma unroll
  for (int s = 0; s < NB; ++s) {
    const int p = p_begin + (s * 8 + warp) * PPW + ps;
    live[s] = false;
#pragma unroll
    for (int v = 0; v < Raw8<T>::kVec; ++v) raw[s].v[v] = make_uint4(0, 0, 0, 0);
    if (p < P) {
      const int phys = a.page_table[static_cast<size_t>(b) * a.max_pages + p];
      if (phys_ok(phys, a.num_phys)) {
        live[s] = true;
        const uint4* src = reinterpret_cast<const uint4*>(
            static_cast<const T*>(a.rows) + (static_cast<size_t>(phys) * a.Hkv + h) * 2 * D + e0);
#pragma unroll
        for (int v = 0; v < Raw8<T>::kVec; ++v) raw[s].v[v] = __ldcs(src + v);
      }
    }
  }

  float lo_best = -INFINITY;  // Gaussian: this lane's best lower bracket candidate
#pragma unroll
  for (int s = 0; s < NB; ++s) {
    const int p = p_begin + (s * 8 + warp) * PPW + ps;
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) a2 = ffma2(coef[g][i], raw_pair<T>(raw[s], i), a2);
      acc[g] = a2.x + a2.y;
    }
    if constexpr (!GAUSS) {
      warp_transpose_sum<G, LPP>(acc, lane);
      float m = acc[0];
#pragma unroll
      for (int o = LPP / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (wl == 0 && p < P)
        a.ub[static_cast<size_t>(unit) * a.max_pages + p] = live[s] ? a.scale * m : -INFINITY;
    } else {
      warp_transpose_sum<G, HALF>(acc, lane);
      const float s2 = __shfl_xor_sync(0xffffffffu, acc[0], HALF);
      if (first && transpose_owner<G, HALF>(lane) && p < P) {
        const int g = transpose_index<G, HALF>(lane);
        const size_t o = (static_cast<size_t>(unit) * G + g) * a.max_pages + p;
        const float n = static_cast<float>(min(a.S, L - p * a.S));
        const float m = a.scale * acc[0];
        const float sd = a.scale * sqrtf(fmaxf(s2, 0.f));
        float mu = a.am1 * m, sg = a.am1 * sd, hat = a.am1 * (m + sd * sqrtf(2.f * logf(n)));
        if (!live[s]) mu = hat = -INFINITY, sg = 0.f;
        a.gws.mu[o] = mu;
        a.gws.sig[o] = sg;
        a.gws.hat[o] = hat;
        lo_best = fmaxf(lo_best, mu - powf(n, -a.inv_beta));
      }
    }
  }

  if constexpr (GAUSS) {
    __shared__ unsigned int lo_key[G];
    if (threadIdx.x < G) lo_key[threadIdx.x] = 0u;
    __syncthreads();
    if (first && transpose_owner<G, HALF>(lane) && lo_best > -INFINITY)
      atomicMax(&lo_key[transpose_index<G, HALF>(lane)], float_key(lo_best));
    __syncthreads();
    if (threadIdx.x < G) {
      const unsigned int k = lo_key[threadIdx.x];
      a.gws.lo[(static_cast<size_t>(unit) * G + threadIdx.x) * a.chunks + blockIdx.x] =
          k == 0u ? -INFINITY : key_float(k);
    }
  }
}

template <typename T, bool GAUSS>
cudaError_t dispatch_stream(const ekv_cache& c, const ekv_seqs& s, StreamArgs& a, int G,
                            cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(a.chunks),
                  static_cast<unsigned>(s.batch * c.num_kv_heads));
#define EKV_STREAM_CASE(DD, GG)                                           \
  if (c.head_dim == DD && G == GG) {                                      \
    meta_stream_kernel<T, DD, GG, GAUSS><<<grid, 256, 0, st>>>(a);        \
    return cudaGetLastError();                                            \
  }
  EKV_STREAM_CASE(128, 1) EKV_STREAM_CASE(128, 2) EKV_STREAM_CASE(128, 4)
  EKV_STREAM_CASE(128, 8) EKV_STREAM_CASE(128, 16)
  EKV_STREAM_CASE(64, 1) EKV_STREAM_CASE(64, 2) EKV_STREAM_CASE(64, 4) EKV_STREAM_CASE(64, 8)
#undef EKV_STREAM_CASE
  if (!GAUSS && c.head_dim == 64 && G == 16) {
    meta_stream_kernel<T, 64, 16, false><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
  }
  return cudaErrorInvalidValue;
}

StreamArgs base_args(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq, float scale) {
  StreamArgs a{};
  a.page_table = s.page_table;
  a.seq_lens = s.seq_lens;
  a.q = q;
  a.scale = scale;
  a.Hkv = c.num_kv_heads;
  a.Hq = Hq;
  a.S = c.page_size;
  a.num_phys = c.num_phys_pages;
  a.max_pages = s.max_pages;
  a.chunks = stream_chunks(s.max_pages);
  return a;
}

}  // namespace

cudaError_t launch_score(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq, float scale,
                         float* ub, cudaStream_t st) {
  StreamArgs a = base_args(c, s, q, Hq, scale);
  a.rows = c.box;
  a.ub = ub;
  const int G = Hq / c.num_kv_heads;
  return c.dtype == EKV_BF16 ? dispatch_stream<bf16, false>(c, s, a, G, st)
                             : dispatch_stream<float, false>(c, s, a, G, st);
}

cudaError_t launch_gauss_stats(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                               float scale, float alpha, const GaussWs& ws, cudaStream_t st) {
  StreamArgs a = base_args(c, s, q, Hq, scale);
  a.rows = c.mom;
  a.gws = ws;
  a.am1 = alpha - 1.0f;
  a.inv_beta = alpha - 1.0f;
  const int G = Hq / c.num_kv_heads;
  return c.dtype == EKV_BF16 ? dispatch_stream<bf16, true>(c, s, a, G, st)
                             : dispatch_stream<float, true>(c, s, a, G, st);
}

}  // namespace ekv
