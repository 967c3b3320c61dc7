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
// (integration by parts with xφ = −φ').  F^(1/β) is convex and decreasing
// (an L^β norm of (u − τ)_+), so Newton's method on it, started left of the
// root (Jensen's bound τ_lo = max_p μ_p − n_p^(−1/β), where F ≥ 1), climbs
// monotonically to the root and never overshoots; far from the root a
// flatter transform takes larger steps (see the solve below).  Pages with
// c > kPruneC at τ_lo contribute below
// n·σ^β·J_β(kPruneC) and stay negligible at every τ the lists are later cut
// at (points left of the root, which only rise: c only grows), so only the
// survivors are iterated, from shared memory.  The recurrence
// amplifies the rounding of Q and φ by about c^(2β)/β! for c > 0, so the fp32
// iterations only approach the root (they stop once a step is below 1e-4);
// the final Newton steps evaluate every term in float64.
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace ekv {

namespace cg = cooperative_groups;

namespace {

constexpr int kGaussThreads = 256;   // filter
constexpr int kTauThreads = 512;     // τ̂ solve: a cluster of up to kTauMaxCluster CTAs per query head
constexpr int kTauMaxCluster = 4;
constexpr int kGaussCand = 4096;     // candidate pages per CTA in shared memory
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
  // c in the precision of the terms (the fp32 steps only approach the root)
  R c;
  if constexpr (sizeof(R) == 8) c = (tau - static_cast<double>(mu)) / static_cast<double>(sg);
  else c = __fdividef(static_cast<float>(tau) - mu, sg);
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

// Partial sums every CTA of a head's cluster pushes to every other one.
struct TauExchange {
  double part[2][kTauMaxCluster][2];  // [step parity][rank][F, F']
  float lo[kTauMaxCluster];
};

// One cluster of C CTAs per query head; CTA r owns the r-th contiguous
// share of the head's pages.  Every sum is a fixed tree inside a CTA, then
// the C partials in rank order, so all CTAs hold the same value and take the
// same steps.  MIN_BLOCKS = 2 caps the registers so that two CTAs share an
// SM, for launches with more CTAs than SMs (all clusters resident at once,
// one wave); 1 leaves the compiler its registers.
template <int MIN_BLOCKS>
__global__ void __launch_bounds__(kTauThreads, MIN_BLOCKS)
    gauss_tau_kernel(GaussWs ws, const int32_t* __restrict__ seq_lens, int S, int max_pages, int Hkv, int G,
                     int Hq, int beta, float* __restrict__ tau_out) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks()), rank = static_cast<int>(cluster.block_rank());
  grid_dep_enter();
  const int row = blockIdx.y, unit = row / G, g = row % G, b = unit / Hkv, kvh = unit % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  const int per = (P + C - 1) / C, pa = min(P, rank * per), pb = min(P, pa + per);
  extern __shared__ float cand[];  // [3][kGaussCand]: μ, σ, n of the cached pages
  float* c_mu = cand;
  float* c_sg = cand + kGaussCand;
  float* c_n = cand + 2 * kGaussCand;
  __shared__ TauExchange tx;
  __shared__ float f_scratch[32];
  __shared__ double d_scratch[64];
  __shared__ int i_scratch[32];
  int par = 0;

  // fn(p, μ_p, σ_p) for this thread's pages pa + tid, pa + tid + 512, … in
  // order, read eight at a time with unconditional loads (a page past pb
  // reads page pa and is skipped): loads behind per-page branches or loop
  // exits are issued one after another
  const size_t base = static_cast<size_t>(row) * max_pages;
  auto for_pages = [&](auto fn) {
    constexpr int kB = 8;
    for (int p0 = pa + tid; p0 < pb; p0 += kB * kTauThreads) {
      float mu[kB], sg[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int p = p0 + k * kTauThreads;
        const size_t at = base + (p < pb ? p : pa);
        mu[k] = ws.mu[at];
        sg[k] = ws.sig[at];
      }
#pragma unroll
      for (int k = 0; k < kB; ++k)
        if (p0 + k * kTauThreads < pb) fn(p0 + k * kTauThreads, mu[k], sg[k]);
    }
  };
  // Jensen's lower bracket: F(τ_lo) ≥ 1 at τ_lo = max_p μ_p − n_p^(−1/β)
  const float inv_beta = 1.0f / static_cast<float>(beta);
  const float full_pow = powf(static_cast<float>(S), -inv_beta);  // every page but the last holds S tokens
  float lo = -INFINITY;
  for_pages([&](int p, float mu, float) {
    const int n = L - p * S;
    if (mu > -INFINITY) lo = fmaxf(lo, mu - (n >= S ? full_pow : powf(static_cast<float>(n), -inv_beta)));
  });
  lo = block_reduce(lo, f_scratch, [](float x, float y) { return fmaxf(x, y); });
  if (tid < C) cluster.map_shared_rank(&tx, tid)->lo[rank] = lo;
  cluster.sync();
  for (int r = 0; r < C; ++r) lo = fmaxf(lo, tx.lo[r]);
  if (P == 0 || !(lo > -INFINITY)) {
    if (rank == 0 && tid == 0) {
      ws.tau_hat[row] = static_cast<double>(INFINITY);
      if (tau_out) tau_out[static_cast<size_t>(b) * Hq + kvh * G + g] = INFINITY;
    }
    return;
  }

  // Candidates: this CTA's pages with μ + kPruneC·σ above the current τ.  τ
  // only rises (Newton from the left), so a page dropped once stays
  // negligible; the list is cut again as τ climbs.  Gathered thread after
  // thread (coalesced loads; a fixed order, so the sums are deterministic);
  // while too many pages are left for shared memory, the steps read every
  // page of the share from global memory.
  auto live = [&](float mu, float sg, double t) {
    return mu > -INFINITY && static_cast<double>(mu) + kPruneC * static_cast<double>(sg) > t;
  };
  int nc = 0;
  bool cached = false;
  auto gather = [&](double t) {  // every thread calls it
    int mine = 0;
    for_pages([&](int, float mu, float sg) { mine += live(mu, sg, t) ? 1 : 0; });
    int pos = block_exclusive_scan(mine, i_scratch, &nc);
    cached = nc <= kGaussCand;
    if (cached)
      for_pages([&](int p, float mu, float sg) {
        if (live(mu, sg, t)) {
          c_mu[pos] = mu;
          c_sg[pos] = sg;
          c_n[pos] = static_cast<float>(min(S, L - p * S));
          ++pos;
        }
      });
    __syncthreads();
  };
  // cuts the cached list to the pages still above t, in place, order kept:
  // thread t owns entries [t·R, t·R + R), holds its survivors in registers
  // across the scan's barriers, then writes them at their new places
  auto recut = [&](double t) {
    constexpr int kMaxR = kGaussCand / kTauThreads;
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

  // F(τ) and F'(τ) over the head's candidates: this CTA's terms in a fixed
  // tree, then the cluster's partials in rank order
  auto evaluate = [&](double t, bool exact, double& F, double& dF) {
    F = 0.0;
    dF = 0.0;
    if (cached) {
      for (int i = tid; i < nc; i += kTauThreads) {
        if (exact)
          gauss_terms<double>(c_mu[i], c_sg[i], c_n[i], t, beta, F, dF);
        else
          gauss_terms<float>(c_mu[i], c_sg[i], c_n[i], t, beta, F, dF);
      }
    } else {
      for (int p = pa + tid; p < pb; p += kTauThreads) {
        const float n = static_cast<float>(min(S, L - p * S));
        if (exact)
          gauss_terms<double>(ws.mu[base + p], ws.sig[base + p], n, t, beta, F, dF);
        else
          gauss_terms<float>(ws.mu[base + p], ws.sig[base + p], n, t, beta, F, dF);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      F += __shfl_xor_sync(0xffffffffu, F, o);
      dF += __shfl_xor_sync(0xffffffffu, dF, o);
    }
    if (lane == 0) {
      d_scratch[warp] = F;
      d_scratch[32 + warp] = dF;
    }
    __syncthreads();
    if (tid < C) {
      double sf = 0.0, sd = 0.0;
      for (int w = 0; w < kTauThreads / 32; ++w) {
        sf += d_scratch[w];
        sd += d_scratch[32 + w];
      }
      TauExchange* dst = cluster.map_shared_rank(&tx, tid);
      dst->part[par][rank][0] = sf;
      dst->part[par][rank][1] = sd;
    }
    cluster.sync();  // also orders this step's reads of d_scratch before the next step's writes
    F = 0.0;
    dF = 0.0;
    for (int r = 0; r < C; ++r) {
      F += tx.part[par][r][0];
      dF += tx.part[par][r][1];
    }
    par ^= 1;  // the next step writes the other half: a slow CTA may still read this one
  };
  // fp32 terms while the steps are large (the lists cut every few steps);
  // the float64 steps below converge quadratically from there.
  // Newton's method on h_p(τ) = F(τ)^(1/p).  For p = β, h_β is the L^β norm
  // of (u − τ)_+ under the pages' mixture: convex and decreasing like F, so
  // its steps from the left never pass the root, and from the right they
  // land left of it.  Where F falls off faster than a power (Gaussian tails
  // far above most pages' means) a step on h_β closes only part of the gap,
  // so while F > kFarF the steps use the flatter h_kFarP, which may pass the
  // root; the first time one does (F < 1), the far steps stop and h_β takes
  // over from the right.  The step (h_p − 1)/(−h_p') is
  // p·F^(1−1/p)·(F^(1/p) − 1)/(−F'), evaluated from F − 1 without
  // cancellation near the root.  Lists are cut at tau_safe, the largest τ
  // evaluated with F ≥ 1 (left of the root), never at a τ that passed it.
  constexpr double kFarF = 4.0, kFarP = 8.0;
  auto newton_step = [&](double F, double dF, double p) {
    const double l = log1p(F - 1.0);
    return p * exp((1.0 - 1.0 / p) * l) * expm1(l / p) / dF;
  };
  double tau = static_cast<double>(lo), tau_safe = tau;
  bool far = true;
  for (int it = 0; it < 40; ++it) {
    double F, dF;
    evaluate(tau, false, F, dF);
    if (F >= 1.0) tau_safe = fmax(tau_safe, tau);
    else far = false;
    if (!(F > 0.0) || !(dF > 0.0)) {  // past every page's mass: back off towards the last safe τ
      if (!(tau > tau_safe)) break;
      tau = 0.5 * (tau + tau_safe);
      continue;
    }
    const double step = newton_step(F, dF, far && F > kFarF ? kFarP : static_cast<double>(beta));
    tau += step;
    // the fp32 terms are good to ~1e-5 near the root: smaller steps are the
    // float64 steps' work, and they check their own convergence
    if (fabs(step) <= 1e-4 * fmax(1.0, fabs(tau))) break;
    if ((it & 3) == 3) {
      if (cached) recut(tau_safe);
      else gather(tau_safe);
    }
  }
  if (!cached) gather(fmin(tau, tau_safe));
  for (int it = 0; it < 3; ++it) {  // float64 terms: quadratic convergence (either side)
    double F, dF;
    evaluate(tau, true, F, dF);
    if (!(dF > 0.0) || !(F > 0.0)) break;
    const double step = newton_step(F, dF, static_cast<double>(beta));
    tau += step;
    // the error left after a step of size e is of order e², so a step below
    // 1e-7 leaves τ̂ within ~1e-14: no further evaluation is needed
    if (fabs(step) <= 1e-7 * fmax(1.0, fabs(tau))) break;
  }
  if (rank == 0 && tid == 0) {
    ws.tau_hat[row] = tau;
    if (tau_out) tau_out[static_cast<size_t>(b) * Hq + kvh * G + g] = static_cast<float>(tau);
  }
}

// Keep page p when (α−1)·ŝ_{p,h} > τ̂_h − Δ for some query head h of the unit,
// in ascending page order; when no page passes, keep the page of largest
// margin (lowest index on ties).  Two launches over chunks of kFilterChunk
// pages: the first counts each chunk's kept pages and finds its best margin,
// the second writes the kept pages at the place the counts of the earlier
// chunks give (chunk 0 also writes n_sel, and the fallback page).
struct FilterCtx {
  double thr[16];  // τ̂_h − Δ
  int scan[32];
  double best_m[32];
  int best_i[32];
};


// The chunk's pages [c0, c1): warp w takes [c0 + w·kPer, …), its lanes
// consecutive pages (coalesced loads).
constexpr int kFilterPerWarp = kFilterChunk / (kGaussThreads / 32);
constexpr int kFilterSteps = kFilterPerWarp / 32;  // pages per lane

// Margins of the lane's pages p0 + 32·i + lane (i < kFilterSteps) of the
// warp's run [p0, p1), p0 < p1, every head's ŝ read with unconditional loads
// first (a page past p1 reads page p0; its margin is not used): loads behind
// per-page branches are issued one after another.
__device__ __forceinline__ void lane_margins(const GaussWs& ws, const FilterCtx& fc, int unit, int G,
                                             int max_pages, int p0, int p1, double (&mg)[kFilterSteps]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kFilterSteps; ++i) mg[i] = -INFINITY;
  for (int g = 0; g < G; ++g) {
    float hv[kFilterSteps];
#pragma unroll
    for (int i = 0; i < kFilterSteps; ++i) {
      const int p = p0 + 32 * i + lane;
      hv[i] = ws.hat[(static_cast<size_t>(unit) * G + g) * max_pages + (p < p1 ? p : p0)];
    }
#pragma unroll
    for (int i = 0; i < kFilterSteps; ++i) mg[i] = fmax(mg[i], static_cast<double>(hv[i]) - fc.thr[g]);
  }
}

__global__ void __launch_bounds__(kGaussThreads)
    gauss_count_kernel(GaussWs ws, const int32_t* __restrict__ seq_lens, int S, int max_pages, int Hkv, int G,
                       double delta) {
  grid_dep_enter();
  const int chunk = blockIdx.x, unit = blockIdx.y, b = unit / Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  __shared__ FilterCtx fc;
  if (tid < G) fc.thr[tid] = ws.tau_hat[static_cast<size_t>(unit) * G + tid] - delta;
  __syncthreads();
  auto margins = [&](int a0, int a1, double (&mg)[kFilterSteps]) {
    lane_margins(ws, fc, unit, G, max_pages, a0, a1, mg);
  };
  const int p0 = chunk * kFilterChunk + warp * kFilterPerWarp, p1 = min(P, p0 + kFilterPerWarp);
  double my_best = -INFINITY;
  int my_idx = 0x7fffffff, cnt = 0;
  if (p0 < p1) {
    double mg[kFilterSteps];
    margins(p0, p1, mg);
#pragma unroll
    for (int i = 0; i < kFilterSteps; ++i) {
      const int p = p0 + 32 * i + lane;
      const bool keep = p < p1 && mg[i] > 0.0;
      if (p < p1 && mg[i] > my_best) {
        my_best = mg[i];
        my_idx = p;
      }
      cnt += __popc(__ballot_sync(0xffffffffu, keep));
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const double om = __shfl_xor_sync(0xffffffffu, my_best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, my_idx, o);
    if (om > my_best || (om == my_best && oi < my_idx)) {
      my_best = om;
      my_idx = oi;
    }
  }
  if (lane == 0) {
    fc.scan[warp] = cnt;
    fc.best_m[warp] = my_best;
    fc.best_i[warp] = my_idx;
  }
  __syncthreads();
  if (tid == 0) {
    int total = 0;
    double bm = -INFINITY;
    int bi = 0x7fffffff;
    for (int w = 0; w < kGaussThreads / 32; ++w) {
      total += fc.scan[w];
      if (fc.best_m[w] > bm || (fc.best_m[w] == bm && fc.best_i[w] < bi)) {
        bm = fc.best_m[w];
        bi = fc.best_i[w];
      }
    }
    const size_t at = static_cast<size_t>(unit) * ws.nchunk + chunk;
    ws.fcount[at] = total;
    ws.fbest[at] = bm;
    ws.fbest_at[at] = bi;
  }
}

__global__ void __launch_bounds__(kGaussThreads)
    gauss_write_kernel(GaussWs ws, const int32_t* __restrict__ seq_lens, int S, int max_pages, int Hkv, int G,
                       double delta, int cap, int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  grid_dep_enter();
  const int chunk = blockIdx.x, unit = blockIdx.y, b = unit / Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int L;
  const int P = seq_pages(seq_lens, b, S, max_pages, &L);
  __shared__ FilterCtx fc;
  __shared__ int s_before, s_total;
  if (tid < G) fc.thr[tid] = ws.tau_hat[static_cast<size_t>(unit) * G + tid] - delta;
  if (warp == 0) {
    // kept pages of the earlier chunks, and of all chunks
    int before = 0, total = 0;
    for (int c = lane; c < ws.nchunk; c += 32) {
      const int n = ws.fcount[static_cast<size_t>(unit) * ws.nchunk + c];
      before += c < chunk ? n : 0;
      total += n;
    }
    before = warp_sum(before);
    total = warp_sum(total);
    if (lane == 0) {
      s_before = before;
      s_total = total;
    }
  }
  __syncthreads();
  int32_t* out = sel + static_cast<size_t>(unit) * cap;
  const int total = s_total;
  if (total == 0) {
    // fallback: the page of largest margin over every chunk, lowest index on ties
    if (chunk == 0 && tid == 0) {
      double bm = -INFINITY;
      int bi = 0x7fffffff;
      for (int c = 0; c < ws.nchunk; ++c) {
        const size_t at = static_cast<size_t>(unit) * ws.nchunk + c;
        if (ws.fbest[at] > bm || (ws.fbest[at] == bm && ws.fbest_at[at] < bi)) {
          bm = ws.fbest[at];
          bi = ws.fbest_at[at];
        }
      }
      if (P > 0 && bi < P) {
        out[0] = bi;
        n_sel[unit] = 1;
      } else {
        n_sel[unit] = 0;
      }
    }
    return;
  }
  if (chunk == 0 && tid == 0) {
    n_sel[unit] = min(total, cap);
    if (total > cap) raise_flag(EKV_EFLAG_SEL_OVERFLOW);
  }
  auto margins = [&](int a0, int a1, double (&mg)[kFilterSteps]) {
    lane_margins(ws, fc, unit, G, max_pages, a0, a1, mg);
  };
  const int p0 = chunk * kFilterChunk + warp * kFilterPerWarp, p1 = min(P, p0 + kFilterPerWarp);
  int cnt = 0;
  double mg[kFilterSteps];
  if (p0 < p1) {
    margins(p0, p1, mg);
#pragma unroll
    for (int i = 0; i < kFilterSteps; ++i)
      cnt += __popc(__ballot_sync(0xffffffffu, p0 + 32 * i + lane < p1 && mg[i] > 0.0));
  }
  if (lane == 0) fc.scan[warp] = cnt;
  __syncthreads();
  int pos = s_before;
  for (int w = 0; w < warp; ++w) pos += fc.scan[w];
  if (cnt == 0) return;
#pragma unroll
  for (int i = 0; i < kFilterSteps; ++i) {
    const int p = p0 + 32 * i + lane;
    const bool keep = p < p1 && mg[i] > 0.0;
    const unsigned int bal = __ballot_sync(0xffffffffu, keep);
    const int at = pos + __popc(bal & ((1u << lane) - 1u));
    if (keep && at < cap) out[at] = p;
    pos += __popc(bal);
  }
}

}  // namespace

cudaError_t launch_gauss_select(const ekv_cache& c, const ekv_seqs& s, int Hq, float alpha,
                                float delta, int cap, const GaussWs& ws, int32_t* sel,
                                int32_t* n_sel, float* tau_hat, cudaStream_t st) {
  const int Hkv = c.num_kv_heads, G = Hq / Hkv, U = s.batch * Hkv;
  const int beta = static_cast<int>(lrint(1.0 / (static_cast<double>(alpha) - 1.0)));
  // CTAs per head: one up to 8192 pages (a cluster's barrier per step costs
  // more than it saves there), else enough to give the B200's SMs two CTAs
  // each, at most kTauMaxCluster
  constexpr int kSms = 148;
  const int rows = U * G;
  int C = 1;
  while (C < kTauMaxCluster && s.max_pages > 8192 && rows * C * 2 <= 2 * kSms) C *= 2;
  const bool two_per_sm = rows * C > kSms;
  auto* kernel = two_per_sm ? gauss_tau_kernel<2> : gauss_tau_kernel<1>;
  const size_t smem = 3 * kGaussCand * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(C), static_cast<unsigned>(rows));
    cfg.blockDim = dim3(kTauThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(C);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kernel, ws, s.seq_lens, c.page_size, s.max_pages, Hkv, G, Hq, beta,
                           tau_hat);
    if (e != cudaSuccess) return e;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 fgrid(static_cast<unsigned>(ws.nchunk), static_cast<unsigned>(U));
  e = launch_k(gauss_count_kernel, fgrid, kGaussThreads, 0, st, ws, s.seq_lens, c.page_size, s.max_pages, Hkv, G,
               static_cast<double>(delta));
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_k(gauss_write_kernel, fgrid, kGaussThreads, 0, st, ws, s.seq_lens, c.page_size, s.max_pages, Hkv, G,
               static_cast<double>(delta), cap, sel, n_sel);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ekv
