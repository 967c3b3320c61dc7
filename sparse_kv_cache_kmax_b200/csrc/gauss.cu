// Gaussian-aware entmax page selection — EntmaxKV summary page
// (gist.science/fr/paper/2605.21649) §2.B, "Sélection Entmax Consciente de
// Gaussienne": estimate the global α-entmax threshold τ̂ from per-page
// Gaussian score statistics, then keep the pages whose estimated maximum
// score clears τ̂ − Δ.
//
// τ̂ solves F(τ) = Σ_p n_p·E[(u_p − τ)_+^β] = 1 for u_p ~ N(μ_p, σ_p²) (in
// threshold units u = (α−1)·score, β = 1/(α−1) an integer).  With
// c = (τ − μ)/σ and J_k(c) = ∫_c^∞ (x − c)^k φ(x) dx,
//   E[(u − τ)_+^β] = σ^β J_β(c),   dE/dτ = −β σ^(β−1) J_(β−1)(c),
//   J_0 = Q(c),  J_1 = φ(c) − c·Q(c),  J_k = (k−1)·J_(k−2) − c·J_(k−1)
// (integration by parts with xφ = −φ').  F is convex and decreasing, so
// Newton's method started left of the root (Jensen's bound
// τ_lo = max_p μ_p − n_p^(−1/β), where F ≥ 1) climbs monotonically to it and
// never overshoots.  Pages with c > kPruneC at τ_lo contribute below
// n·σ^β·J_β(kPruneC) and stay negligible for every later τ (c only grows), so
// only the survivors are iterated, from shared memory.  The recurrence
// amplifies the rounding of Q and φ by about c^(2β)/β! for c > 0, so the fp32
// iterations only approach the root (they stop once a step is below 1e-5);
// the final Newton steps evaluate every term in float64.
#include "kernels.cuh"

namespace ekv {

namespace {

constexpr int kGaussThreads = 256;   // filter
constexpr int kTauThreads = 1024;    // τ̂ solve: one CTA per query head, every thread on its pages
constexpr int kGaussCand = 3072;
constexpr float kPruneC = 6.0f;

template <typename R>
__device__ __forceinline__ void normal_tail(R c, R& Q, R& phi);
template <>
__device__ __forceinline__ void normal_tail<float>(float c, float& Q, float& phi) {
  Q = 0.5f * erfcf(c * 0.70710678118654752f);
  phi = 0.39894228040143268f * expf(-0.5f * c * c);
}
template <>
__device__ __forceinline__ void normal_tail<double>(double c, double& Q, double& phi) {
  Q = 0.5 * erfc(c * 0.70710678118654752);
  phi = 0.39894228040143268 * exp(-0.5 * c * c);
}

// Adds page (μ, σ, n)'s n·E[(u−τ)_+^β] to F and n·β·E[(u−τ)_+^(β−1)] to dF,
// evaluating the tail functions in precision R.
template <typename R>
__device__ __forceinline__ void gauss_terms(float mu, float sg, float n, double tau, int beta,
                                            double& F, double& dF) {
  if (!(mu > -INFINITY)) return;
  if (sg <= 0.f) {
    const double w = static_cast<double>(mu) - tau;
    if (w > 0.0) {
      double wb1 = 1.0;
      for (int k = 1; k < beta; ++k) wb1 *= w;
      F += n * wb1 * w;
      dF += n * beta * wb1;
    }
    return;
  }
  const R c = static_cast<R>((tau - static_cast<double>(mu)) / static_cast<double>(sg));
  if (c > static_cast<R>(kPruneC)) return;
  R Q, phi;
  normal_tail<R>(c, Q, phi);
  R jm2 = Q, jm1 = phi - c * Q;  // J_0, J_1
  R jb = jm1, jb1 = jm2;         // J_β, J_(β−1) for β = 1
  for (int k = 2; k <= beta; ++k) {
    const R jk = static_cast<R>(k - 1) * jm2 - c * jm1;
    jb1 = jm1;
    jb = jk;
    jm2 = jm1;
    jm1 = jk;
  }
  double sb1 = 1.0;
  for (int k = 1; k < beta; ++k) sb1 *= sg;
  F += static_cast<double>(n) * sb1 * sg * static_cast<double>(jb > R(0) ? jb : R(0));
  dF += static_cast<double>(n) * beta * sb1 * static_cast<double>(jb1 > R(0) ? jb1 : R(0));
}

__global__ void __launch_bounds__(kTauThreads)
    gauss_tau_kernel(GaussWs ws, const int32_t* __restrict__ seq_lens, int S, int max_pages,
                     int Hkv, int G, int Hq, int beta, float* __restrict__ tau_out) {
  grid_dep_enter();
  const int row = blockIdx.x, unit = row / G, g = row % G, b = unit / Hkv, kvh = unit % Hkv;
  const int tid = threadIdx.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  __shared__ float c_mu[kGaussCand], c_sg[kGaussCand], c_n[kGaussCand];
  __shared__ float f_scratch[32];
  __shared__ double d_scratch[64];
  __shared__ int i_scratch[32];

  // Jensen's lower bracket: F(τ_lo) ≥ 1 at τ_lo = max_p μ_p − n_p^(−1/β)
  const size_t base = static_cast<size_t>(row) * max_pages;
  const float inv_beta = 1.0f / static_cast<float>(beta);
  float lo = -INFINITY;
  for (int p = tid; p < P; p += blockDim.x) {
    const float mu = ws.mu[base + p];
    if (mu > -INFINITY) lo = fmaxf(lo, mu - powf(static_cast<float>(min(S, L - p * S)), -inv_beta));
  }
  lo = block_reduce(lo, f_scratch, [](float x, float y) { return fmaxf(x, y); });
  if (P == 0 || !(lo > -INFINITY)) {
    if (tid == 0) {
      ws.tau_hat[row] = static_cast<double>(INFINITY);
      if (tau_out) tau_out[static_cast<size_t>(b) * Hq + kvh * G + g] = INFINITY;
    }
    return;
  }

  // Candidates: the pages with μ + kPruneC·σ above the current τ.  τ only
  // rises (Newton from the left), so a page dropped once stays negligible;
  // the list is cut again as τ climbs.  Gathered thread after thread
  // (thread t takes pages t, t + 256, …: coalesced loads; a fixed order, so
  // the sums below are deterministic); while too many pages are left for
  // shared memory, the steps read every page from global memory.
  auto live = [&](int p, double t) {
    const float mu = ws.mu[base + p], sg = ws.sig[base + p];
    return mu > -INFINITY && static_cast<double>(mu) + kPruneC * static_cast<double>(sg) > t;
  };
  int nc = 0;
  bool cached = false;
  auto gather = [&](double t) {  // every thread calls it
    int mine = 0;
    for (int p = tid; p < P; p += kTauThreads) mine += live(p, t) ? 1 : 0;
    int pos = block_exclusive_scan(mine, i_scratch, &nc);
    cached = nc <= kGaussCand;
    if (cached)
      for (int p = tid; p < P; p += kTauThreads)
        if (live(p, t)) {
          c_mu[pos] = ws.mu[base + p];
          c_sg[pos] = ws.sig[base + p];
          c_n[pos] = static_cast<float>(min(S, L - p * S));
          ++pos;
        }
    __syncthreads();
  };
  // cuts the cached list to the pages still above t, in place, order kept:
  // thread t owns entries [t·R, t·R + R) (R ≤ 4), holds its survivors in
  // registers across one barrier, then writes them at their new places
  auto recut = [&](double t) {
    constexpr int kMaxR = 4;
    static_assert(kGaussCand <= kMaxR * kTauThreads, "entries per thread");
    const int R = (nc + kTauThreads - 1) / kTauThreads;
    float m[kMaxR], sgm[kMaxR], nn[kMaxR];
    unsigned int keep = 0u;
#pragma unroll
    for (int j = 0; j < kMaxR; ++j) {
      const int i = tid * R + j;
      m[j] = sgm[j] = nn[j] = 0.f;
      if (j < R && i < nc) {
        m[j] = c_mu[i];
        sgm[j] = c_sg[i];
        nn[j] = c_n[i];
        if (static_cast<double>(m[j]) + kPruneC * static_cast<double>(sgm[j]) > t) keep |= 1u << j;
      }
    }
    int total;
    int pos = block_exclusive_scan(__popc(keep), i_scratch, &total);  // its barriers order the reads before the writes
#pragma unroll
    for (int j = 0; j < kMaxR; ++j)
      if ((keep >> j) & 1u) {
        c_mu[pos] = m[j];
        c_sg[pos] = sgm[j];
        c_n[pos] = nn[j];
        ++pos;
      }
    __syncthreads();
    nc = total;
  };
  gather(static_cast<double>(lo));

  // F(τ) and F'(τ) over the candidates (or every page), summed in a fixed order
  auto evaluate = [&](double t, bool exact, double& F, double& dF) {
    F = 0.0;
    dF = 0.0;
    if (cached) {
      for (int i = tid; i < nc; i += blockDim.x) {
        if (exact)
          gauss_terms<double>(c_mu[i], c_sg[i], c_n[i], t, beta, F, dF);
        else
          gauss_terms<float>(c_mu[i], c_sg[i], c_n[i], t, beta, F, dF);
      }
    } else {
      for (int p = tid; p < P; p += blockDim.x) {
        const float n = static_cast<float>(min(S, L - p * S));
        if (exact)
          gauss_terms<double>(ws.mu[base + p], ws.sig[base + p], n, t, beta, F, dF);
        else
          gauss_terms<float>(ws.mu[base + p], ws.sig[base + p], n, t, beta, F, dF);
      }
    }
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      F += __shfl_xor_sync(0xffffffffu, F, o);
      dF += __shfl_xor_sync(0xffffffffu, dF, o);
    }
    __syncthreads();  // the previous evaluation's partials are read
    if (lane == 0) {
      d_scratch[warp] = F;
      d_scratch[32 + warp] = dF;
    }
    __syncthreads();
    F = 0.0;
    dF = 0.0;
    for (int w = 0; w < kTauThreads / 32; ++w) {
      F += d_scratch[w];
      dF += d_scratch[32 + w];
    }
  };
  // fp32 terms: a monotone approach from the left while the steps are large
  // (the list cut every few steps); the float64 steps below converge
  // quadratically from there
  double tau = static_cast<double>(lo);
  for (int it = 0; it < 40; ++it) {
    double F, dF;
    evaluate(tau, false, F, dF);
    const double step = (F - 1.0) / dF;
    if (!(step > 0.0)) break;
    tau += step;
    if (step <= 1e-5 * fmax(1.0, fabs(tau))) break;
    if ((it & 3) == 3) {
      if (cached) recut(tau);
      else gather(tau);
    }
  }
  if (!cached) gather(tau);
  for (int it = 0; it < 3; ++it) {    // float64 terms: quadratic convergence (either side)
    double F, dF;
    evaluate(tau, true, F, dF);
    if (!(dF > 0.0)) break;
    const double step = (F - 1.0) / dF;
    tau += step;
    if (fabs(step) <= 1e-12 * fmax(1.0, fabs(tau))) break;
  }
  if (tid == 0) {
    ws.tau_hat[row] = tau;
    if (tau_out) tau_out[static_cast<size_t>(b) * Hq + kvh * G + g] = static_cast<float>(tau);
  }
}

// Keep page p when (α−1)·ŝ_{p,h} > τ̂_h − Δ for some query head h of the unit;
// compaction in ascending page order; fallback to the largest margin.
__global__ void __launch_bounds__(kGaussThreads)
    gauss_filter_kernel(GaussWs ws, const int32_t* __restrict__ seq_lens, int S, int max_pages,
                        int Hkv, int G, double delta, int cap, int32_t* __restrict__ sel,
                        int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  const int unit = blockIdx.x, b = unit / Hkv, tid = threadIdx.x;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  __shared__ double s_thr[16];
  __shared__ int scan_scratch[32];
  __shared__ double best_m[32];
  __shared__ int best_i[32];
  if (tid < G) s_thr[tid] = ws.tau_hat[static_cast<size_t>(unit) * G + tid] - delta;
  __syncthreads();
  int32_t* out = sel + static_cast<size_t>(unit) * cap;
  // warp w owns the pages [w·C, (w + 1)·C), its lanes consecutive pages
  // (coalesced loads): one pass counts the kept pages by ballots (and finds
  // the best margin), the warp counts are scanned, a second pass writes the
  // kept pages in ascending order
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kGaussThreads / 32;
  const int C = ((P + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int p0 = warp * C, p1 = min(P, p0 + C);
  auto margin = [&](int p) {
    double mg = -INFINITY;
    for (int g = 0; g < G; ++g) {
      const double m = static_cast<double>(ws.hat[(static_cast<size_t>(unit) * G + g) * max_pages + p]) - s_thr[g];
      mg = fmax(mg, m);
    }
    return mg;
  };
  double my_best = -INFINITY;
  int my_idx = 0x7fffffff;
  int wcount = 0;
  for (int q0 = p0; q0 < p1; q0 += 32) {
    const int p = q0 + lane;
    bool keep = false;
    if (p < p1) {
      const double mg = margin(p);
      keep = mg > 0.0;
      if (mg > my_best) {
        my_best = mg;
        my_idx = p;
      }
    }
    wcount += __popc(__ballot_sync(0xffffffffu, keep));
  }
  if (lane == 0) scan_scratch[warp] = wcount;
  __syncthreads();
  int before = 0, carry = 0;
  for (int w = 0; w < kWarps; ++w) {
    before += w < warp ? scan_scratch[w] : 0;
    carry += scan_scratch[w];
  }
  if (wcount > 0) {
    int pos = before;
    for (int q0 = p0; q0 < p1; q0 += 32) {
      const int p = q0 + lane;
      const bool keep = p < p1 && margin(p) > 0.0;
      const unsigned int bal = __ballot_sync(0xffffffffu, keep);
      const int at = pos + __popc(bal & ((1u << lane) - 1u));
      if (keep && at < cap) out[at] = p;
      pos += __popc(bal);
    }
  }
  if (carry > 0) {
    if (tid == 0) {
      n_sel[unit] = min(carry, cap);
      if (carry > cap) raise_flag(EKV_EFLAG_SEL_OVERFLOW);
    }
    return;
  }
  // fallback: the single page with the largest margin, lowest index on ties
  for (int o = 16; o > 0; o >>= 1) {
    const double om = __shfl_xor_sync(0xffffffffu, my_best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, my_idx, o);
    if (om > my_best || (om == my_best && oi < my_idx)) {
      my_best = om;
      my_idx = oi;
    }
  }
  if (lane == 0) {
    best_m[warp] = my_best;
    best_i[warp] = my_idx;
  }
  __syncthreads();
  if (tid == 0) {
    double bm = -INFINITY;
    int bi = 0x7fffffff;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
      if (best_m[w] > bm || (best_m[w] == bm && best_i[w] < bi)) {
        bm = best_m[w];
        bi = best_i[w];
      }
    }
    if (P > 0 && bi < P) {
      out[0] = bi;
      n_sel[unit] = 1;
    } else {
      n_sel[unit] = 0;
    }
  }
}

}  // namespace

cudaError_t launch_gauss_select(const ekv_cache& c, const ekv_seqs& s, int Hq, float alpha,
                                float delta, int cap, const GaussWs& ws, int32_t* sel,
                                int32_t* n_sel, float* tau_hat, cudaStream_t st) {
  const int Hkv = c.num_kv_heads, G = Hq / Hkv, U = s.batch * Hkv;
  const int beta = static_cast<int>(lrint(1.0 / (static_cast<double>(alpha) - 1.0)));
  {
    const cudaError_t le_ = launch_k(gauss_tau_kernel, U * G, kTauThreads, 0, st, ws, s.seq_lens, c.page_size, s.max_pages, Hkv,
                                                    G, Hq, beta, tau_hat);
    if (le_ != cudaSuccess) return le_;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le_ = launch_k(gauss_filter_kernel, U, kGaussThreads, 0, st, ws, s.seq_lens, c.page_size, s.max_pages, Hkv,
                                                   G, static_cast<double>(delta), cap, sel, n_sel);
    if (le_ != cudaSuccess) return le_;
  }
  return cudaGetLastError();
}

}  // namespace ekv
