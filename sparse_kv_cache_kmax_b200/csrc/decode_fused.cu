// Sparse α-entmax decode over the selected pages, one thread-block cluster
// per (sequence, KV head) — EntmaxKV summary page (gist.science/fr/paper/
// 2605.21649) §2.C "Attention Entmax Parcimonieuse", with the support-only V
// read that §2–§3 make exact.
//
// The unit's selected pages are split into C equal runs, one per CTA of the
// cluster (C ≤ 16, chosen so that all units' clusters are resident at once).
// Each CTA works in three phases separated by cluster barriers:
//  1. K: every warp streams its own pages (page j of the run goes to warp
//     j mod 16) through a private ring of shared-memory slots filled by 1-D
//     bulk async copies (one copy = one contiguous S×d K tile) and scores
//     them on tensor cores (m16n8k16, rows of the tile loaded from shared
//     memory straight into A fragments).  Scores z and page maxima stay in
//     shared memory.  The CTA then pushes its per-head maxima to every CTA.
//  2. τ: query head h is solved by CTA h mod C on the head's scores of the
//     whole unit, gathered from the cluster's shared memory (DSMEM) in token
//     order: Σ[u − τ]_+^β = 1, β = 1/(α−1) (see cta_solve_tau).  The solver
//     writes the head's support bits and count and sends τ to every CTA.
//  3. V: each CTA lists the support tokens of its run (some head has
//     u > τ) and reads only their V rows from global memory, eight rows in
//     flight per warp; p = [u − τ]^β comes from the scores in shared memory.
//     CTA r owns a 1/C slice of the unit's G×d outputs: every CTA pushes its
//     partial of that slice to CTA r, which sums the C partials in rank
//     order.
// Every sum has a fixed order, so results are deterministic.
#include <cooperative_groups.h>

#include <mutex>
#include <vector>

#include "decode.cuh"

namespace ekv {

namespace {

namespace cg = cooperative_groups;

constexpr int kFWarps = 16;
constexpr int kFThreads = 32 * kFWarps;
constexpr int kFMaxCluster = 16;
constexpr int kFMaxSpw = 8;       // K ring slots per warp
constexpr int kFMaxHeads = 16;    // query heads per KV head (G)
constexpr int kTauBinsF = 256;
constexpr int kPairwiseMax = 256; // candidates for the pairwise support test

struct FusedGeom {
  int C;          // CTAs per unit (cluster size)
  int spc;        // selected slots per CTA
  int zpitch;     // floats per head row of the score array (spc·S + 4)
  int spw;        // K ring slots per warp
  int tile_bytes; // bytes of one S×d K or V tile
  int chunk;      // outputs owned per CTA: ceil(G·d / C)
  int off_ints, off_pm, off_zs, off_inbox, off_ring;  // byte offsets in dynamic shared memory
  int off_v;      // bytes of the ring the τ scratch, the V token list and the partials need
  int smem;       // dynamic shared memory bytes
};

struct TauShared {
  float f[2][kFWarps];   // fp32 partials, double-buffered: one barrier per reduction
  float f2[2][kFWarps];
  double d[3][kFWarps];  // fp64 partials
  int i[kFWarps];
  int hist[kTauBinsF];
  double tau;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Pairwise sum of the 16 per-warp partials (a fixed tree, so every thread
// computes the same value).
template <typename V>
__device__ __forceinline__ V tree16(const V* p) {
  const V a0 = (p[0] + p[1]) + (p[2] + p[3]), a1 = (p[4] + p[5]) + (p[6] + p[7]);
  const V a2 = (p[8] + p[9]) + (p[10] + p[11]), a3 = (p[12] + p[13]) + (p[14] + p[15]);
  return (a0 + a1) + (a2 + a3);
}
static_assert(kFWarps == 16, "tree16 sums one partial per warp");

// w^(β−1) for w > 0 in the precision of w.
template <typename V>
__device__ __forceinline__ V pow_bm1(V w, V beta, int ipow) {
  switch (ipow) {
    case 1: return V(1);
    case 2: return w;
    case 3: return w * w;
    case 4: return w * w * w;
    default:
      if constexpr (sizeof(V) == 8) return pow(w, beta - 1.0);
      else return powf(w, beta - 1.0f);
  }
}

// f(t) − 1 = Σ(u − t)_+^β − 1 and Σ(u − t)_+^(β−1) over the candidates, by
// one warp (solo) or by the CTA (one barrier, buffer parity `par`).
template <typename V>
__device__ __forceinline__ void f_df(const float* cand, int nc, V t, V beta, int ipow, bool solo,
                                     TauShared& sh, int par, V& f, V& df) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  V a = V(0), b = V(0);
  for (int i = solo ? lane : tid; i < nc; i += solo ? 32 : kFThreads) {
    const V w = static_cast<V>(cand[i]) - t;
    if (w > V(0)) {
      const V wb1 = pow_bm1<V>(w, beta, ipow);
      a += wb1 * w;
      b += wb1;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (!solo) {
    if constexpr (sizeof(V) == 4) {
      if (lane == 0) {
        sh.f[par][warp] = a;
        sh.f2[par][warp] = b;
      }
      __syncthreads();
      a = tree16(sh.f[par]);
      b = tree16(sh.f2[par]);
    } else {
      if (lane == 0) {
        sh.d[0][warp] = a;
        sh.d[1][warp] = b;
      }
      __syncthreads();
      a = tree16(sh.d[0]);
      b = tree16(sh.d[1]);
      __syncthreads();
    }
  }
  f = a - V(1);
  df = b;
}

// Sums of (c, s1, s2) over the CTA (fp64, fixed tree); every thread gets them.
__device__ __forceinline__ void cta_sum3(double& c, double& s1, double& s2, TauShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  if (lane == 0) {
    sh.d[0][warp] = c;
    sh.d[1][warp] = s1;
    sh.d[2][warp] = s2;
  }
  __syncthreads();
  c = tree16(sh.d[0]);
  s1 = tree16(sh.d[1]);
  s2 = tree16(sh.d[2]);
  __syncthreads();
}

// Closed-form τ on a support of c values with sums s1 = Σu, s2 = Σu²:
// β = 1: τ = (s1 − 1)/c;  β = 2: τ = M − √(M² − Q + 1/c), M = s1/c, Q = s2/c.
__device__ __forceinline__ double closed_tau(int ipow, double c, double s1, double s2) {
  if (ipow == 1) return (s1 - 1.0) / c;
  const double M = s1 / c, Q = s2 / c;
  return M - sqrt(fmax(M * M - Q + 1.0 / c, 0.0));
}

// Rare paths of cta_solve_tau, kept out of line so that the common path's
// code stays compact (code that runs once per CTA is fetched, not cached).

// Repeats the closed form on {u > τ} until the support is stable.
__device__ __noinline__ double repair_closed_tau(const float* cand, int nc, int ipow, double tau,
                                                  TauShared& sh) {
  const int tid = threadIdx.x;
  for (int rep = 0; rep < 8; ++rep) {
    double c = 0.0, s1 = 0.0, s2 = 0.0;
    for (int i = tid; i < nc; i += kFThreads) {
      const double u = cand[i];
      if (u > tau) {
        c += 1.0;
        s1 += u;
        s2 += u * u;
      }
    }
    cta_sum3(c, s1, s2, sh);
    if (c < 1.0) break;
    const double t_new = closed_tau(ipow, c, s1, s2);
    if (t_new == tau) break;
    tau = t_new;
  }
  return tau;
}

// Newton's method from the left in fp32 on the ℓ_β norm of (u − τ)_+ (convex
// and decreasing), then a float64 finish: the closed form for β ∈ {1,2}, one
// Newton step otherwise.  Up to kSoloMax candidates one warp iterates alone
// (no barrier per step); above that the CTA does, one barrier per step.
constexpr int kSoloMax = 128;
__device__ __noinline__ double newton_tau(const float* cand, int nc, double tau_lo, float um,
                                          float beta, int ipow, TauShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool closed = ipow == 1 || ipow == 2;
  double tau;
  const bool solo = nc <= kSoloMax;
  if (!solo || warp == 0) {
    float t = static_cast<float>(tau_lo);
    if (static_cast<double>(t) > tau_lo) t = nextafterf(t, -INFINITY);
    int par = 1;
    for (int it = 0; it < 64; ++it) {
      float f, df;
      par ^= 1;
      f_df<float>(cand, nc, t, beta, ipow, solo, sh, par, f, df);
      if (it == 0 && f < 0.0f) {  // bracket missed by rounding: restart from max u − 1
        t = um - 1.0f;
        continue;
      }
      const float step = norm_newton_step<float>(f, df, beta);
      if (!(step > 0.0f)) break;
      t += step;
      if (step <= 2e-7f * fmaxf(1.0f, fabsf(t))) break;
    }
    double tt = t;
    if (closed) {
      for (int rep = 0; rep < 4; ++rep) {
        double c = 0.0, s1 = 0.0, s2 = 0.0;
        for (int i = solo ? lane : tid; i < nc; i += solo ? 32 : kFThreads) {
          const double u = cand[i];
          if (u > tt) {
            c += 1.0;
            s1 += u;
            s2 += u * u;
          }
        }
        if (solo) {
          c = warp_sum(c);
          s1 = warp_sum(s1);
          s2 = warp_sum(s2);
        } else {
          cta_sum3(c, s1, s2, sh);
        }
        if (c < 1.0) break;
        const double t_new = closed_tau(ipow, c, s1, s2);
        if (t_new == tt) break;
        tt = t_new;
      }
    } else {
      double f, df;
      f_df<double>(cand, nc, tt, static_cast<double>(beta), ipow, solo, sh, 0, f, df);
      if (df > 0.0) tt += f / (static_cast<double>(beta) * df);
    }
    if (tid == 0) sh.tau = tt;
  }
  __syncthreads();
  tau = sh.tau;
  __syncthreads();
  return tau;
}

// τ of one query head without a closed form (β ∉ {1, 2}): Newton's method
// from the left on the ℓ_β norm of (u − τ)_+ over all n values u in shared
// memory, from max u − 1 (where the sum is ≥ 1: the maximum alone gives 1),
// one pass and one barrier per step, then one float64 Newton step.  The
// whole CTA calls it; it returns the fp32 τ every later step uses.
__device__ float cta_newton_tau(const float* u, int n, float um, float beta, int ipow, TauShared& sh) {
  float t = um - 1.0f;
  int par = 1;
  for (int it = 0; it < 64; ++it) {
    float f, df;
    par ^= 1;
    f_df<float>(u, n, t, beta, ipow, false, sh, par, f, df);
    const float step = norm_newton_step<float>(f, df, beta);
    if (!(step > 0.0f)) break;
    t += step;
    if (step <= 2e-7f * fmaxf(1.0f, fabsf(t))) break;
  }
  double tau = t, f, df;
  f_df<double>(u, n, tau, static_cast<double>(beta), ipow, false, sh, 0, f, df);
  if (df > 0.0) tau += f / (static_cast<double>(beta) * df);
  return static_cast<float>(tau);
}

// τ of one query head: Σ_i [u_i − τ]_+^β = 1 over the n values u[0..n) in
// shared memory (argument z), whose histogram over (um − 1, um] (um = max u,
// 256 bins from the top) is in sh.hist.  The whole CTA calls it; it leaves
// sh.hist zeroed.  cand: shared scratch of n floats.
//  1. Bracket: c values above an edge e force τ ≥ e − c^(−1/β) (c of them
//     would already carry mass ≥ 1); the best edge gives τ_lo.
//  2. The values above τ_lo are compacted (warp order, then scan order).
//  3. For β ∈ {1,2} and few candidates: u_j is in the support iff
//     f(u_j) = Σ_i (u_i − u_j)_+^β < 1 (f decreases, f(τ) = 1), tested for
//     every candidate at once; τ is the float64 closed form on that support,
//     kept if the support it implies is the same, else refined by repeating
//     the closed form on {u > τ}.  Otherwise Newton's method from the left in
//     fp32 on the ℓ_β norm of (u − τ)_+ (convex and decreasing) and a float64
//     finish: the closed form for β ∈ {1,2}, one float64 Newton step otherwise.
// Returns the fp32 τ every later step uses.
__device__ float cta_solve_tau(const float* z, int n, float um, float* cand, float beta, int ipow,
                               TauShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // 1. bracket, computed by every warp from the histogram (no barrier)
  float cb = um - 1.0f;
  {
    constexpr int kPer = kTauBinsF / 32;
    int cnt[kPer], tot = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      tot += sh.hist[lane * kPer + k];
      cnt[k] = tot;
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int before = incl - tot;
    // c^(−1/β) without libm: exact-enough reciprocals for β ∈ {1,2}, fast
    // exp2/log2 otherwise; the slack below keeps τ_lo a lower bound
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int c = before + cnt[k];
      if (c > 0) {
        const float fc = static_cast<float>(c);
        const float r = ipow == 1 ? 1.0f / fc : (ipow == 2 ? rsqrtf(fc) : exp2f(-__log2f(fc) / beta));
        cb = fmaxf(cb, um - static_cast<float>(lane * kPer + k + 1) / kTauBinsF - r);
      }
    }
    cb = warp_max(cb);
  }
  const double tau_lo = static_cast<double>(cb) - 4e-6 * (1.0 + fabs(static_cast<double>(um)));
  // fp32 copy rounded down: comparisons against it stay on the safe side
  float tau_lo_f = static_cast<float>(tau_lo);
  if (static_cast<double>(tau_lo_f) > tau_lo) tau_lo_f = nextafterf(tau_lo_f, -INFINITY);
  // 2. compaction: warp w takes elements k·512 + 32w + lane; order (w, k, lane)
  int nc;
  {
    int mine = 0;
    for (int base = 0; base < n; base += kFThreads) {
      const int i = base + tid;
      const bool in = i < n && z[i] > tau_lo_f;
      mine += __popc(__ballot_sync(0xffffffffu, in));
    }
    if (lane == 0) sh.i[warp] = mine;
    __syncthreads();
    int pos = 0;
    nc = 0;
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) {
      const int c = sh.i[w];
      pos += w < warp ? c : 0;
      nc += c;
    }
    for (int base = 0; base < n; base += kFThreads) {
      const int i = base + tid;
      const float u = i < n ? z[i] : -INFINITY;
      const bool in = i < n && u > tau_lo_f;
      const unsigned int bal = __ballot_sync(0xffffffffu, in);
      if (in) cand[pos + __popc(bal & ((1u << lane) - 1u))] = u;
      pos += __popc(bal);
    }
    for (int i = tid; i < kTauBinsF; i += kFThreads) sh.hist[i] = 0;  // ready for the next head
    __syncthreads();
  }
  // 3. τ
  double tau;
  if ((ipow == 1 || ipow == 2) && nc <= kPairwiseMax) {
    bool in = false;
    float ut = 0.f;
    double c = 0.0, s1 = 0.0, s2 = 0.0;
    if (tid < nc) {
      ut = cand[tid];
      float fs = 0.f;
#pragma unroll 4
      for (int i = 0; i < nc; ++i) {
        const float w = cand[i] - ut;
        if (w > 0.f) fs = fmaf(ipow == 1 ? 1.0f : w, w, fs);
      }
      in = fs < 1.0f;
      if (in) {
        c = 1.0;
        s1 = ut;
        s2 = static_cast<double>(ut) * ut;
      }
    }
    cta_sum3(c, s1, s2, sh);
    tau = closed_tau(ipow, c, s1, s2);
    const bool bad = tid < nc && (in != (static_cast<double>(ut) > tau));
    if (__syncthreads_or(bad)) tau = repair_closed_tau(cand, nc, ipow, tau, sh);
  } else {
    tau = newton_tau(cand, nc, tau_lo, um, beta, ipow, sh);
  }
  return static_cast<float>(tau);
}

// IPOW: β when it is 1 or 2 (α = 2 or 1.5), fixed at compile time so that
// those kernels carry no code for other exponents; 0: β read at run time.
template <int D, int G, int IPOW>
__global__ void __launch_bounds__(kFThreads, 1) fused_decode_kernel(DecodeArgs a, FusedGeom f) {
  const int ipow = IPOW != 0 ? IPOW : a.ipow;
  constexpr int KP = D / 32, NT = (G + 7) / 8, DPL = D / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t bars[kFWarps * kFMaxSpw];
  __shared__ TauShared tsh;
  __shared__ float s_tau[G];
  __shared__ float mall[kFMaxHeads][kFMaxCluster];  // run maxima: [head][CTA rank]
  __shared__ int scan_scratch[32];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int C = f.C;
  const int unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const int S = a.S, spc = f.spc, zp = f.zpitch, spw = f.spw;
  int* phys_s = reinterpret_cast<int*>(smem + f.off_ints);  // [spc]
  int* nv_s = phys_s + spc;                                  // [spc]
  float* pm = reinterpret_cast<float*>(smem + f.off_pm);     // [G][spc] page maxima of z
  float* zs = reinterpret_cast<float*>(smem + f.off_zs);     // [G][zpitch] scores z
  float* inbox = reinterpret_cast<float*>(smem + f.off_inbox);  // [C][chunk] partial outputs
  unsigned char* ring = smem + f.off_ring;

  if (tid == 0) {
    for (int s = 0; s < kFWarps * spw; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  for (int i = tid; i < kTauBinsF; i += kFThreads) tsh.hist[i] = 0;
  // The page table is written by no kernel of the step: this CTA's share of
  // the sequence's row is brought into L2 while the selection is still being
  // made (a hint; the row is read again after the wait)
  {
    const int per = (a.max_pages + C - 1) / C;
    const int p0 = rank * per, p1 = min(a.max_pages, p0 + per);
    const int* row = a.page_table + static_cast<size_t>(b) * a.max_pages;
    for (int p = p0 + 32 * tid; p < p1; p += 32 * kFThreads) prefetch_l2(row + p);
  }
  __syncthreads();
  grid_dep_enter();
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int s0 = rank * spc;
  const int np = max(0, min(spc, n_slots - s0));

  // ---------------------------------------------------------------- 1. K
  // Warp w owns pages w, w+16, ... of the run: its lanes resolve them, and
  // the lanes of its first spw pages start their copies at once.
  const int cnt_w = warp < np ? (np - warp + kFWarps - 1) / kFWarps : 0;
  const size_t tile_elems = static_cast<size_t>(S) * D;
  auto issue = [&](int i, int ph) {  // page i of this warp into its slot
    uint64_t* bar = &bars[warp * spw + i % spw];
    if (ph < 0) {
      mbar_arrive(bar);  // nothing to copy: complete the phase
      return;
    }
    mbar_arrive_expect_tx(bar, static_cast<unsigned int>(f.tile_bytes));
    const bf16* src = static_cast<const bf16*>(a.k_pool) + (static_cast<size_t>(ph) * a.Hkv + kvh) * tile_elems;
    bulk_g2s(ring + static_cast<size_t>(warp * spw + i % spw) * f.tile_bytes, src,
             static_cast<unsigned int>(f.tile_bytes), bar);
  };
  for (int i = lane; i < cnt_w; i += 32) {
    const int j = warp + i * kFWarps;
    int nv;
    const int ph = slot_page(a, unit, b, s0 + j, P, L, &nv);
    phys_s[j] = ph;
    nv_s[j] = nv;
    if (i < spw) issue(i, ph);
  }
  __syncwarp();
  uint32_t bfrag[2 * KP][NT][2];
  load_q_frags<D, G>(a, b, kvh, g, t, bfrag);

  for (int i = 0; i < cnt_w; ++i) {
    const int j = warp + i * kFWarps, sl = warp * spw + i % spw;
    const unsigned int parity = static_cast<unsigned int>(i / spw) & 1u;
    if (!mbar_wait(&bars[sl], parity)) mbar_wait(&bars[sl], parity);  // second bounded wait: no copy left in flight
    const unsigned char* tile = ring + static_cast<size_t>(sl) * f.tile_bytes;
    const int nv = phys_s[j] < 0 ? 0 : nv_s[j];
    float pmx[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) pmx[nt][0] = pmx[nt][1] = -INFINITY;
    for (int mt = 0; mt < S / 16; ++mt) {
      const int tok0 = mt * 16;
      const uint4* rlo = reinterpret_cast<const uint4*>(tile + static_cast<size_t>(tok0 + g) * D * 2) + t;
      const uint4* rhi = reinterpret_cast<const uint4*>(tile + static_cast<size_t>(tok0 + g + 8) * D * 2) + t;
      uint4 va[KP], vb[KP];
#pragma unroll
      for (int c = 0; c < KP; ++c) {
        va[c] = rlo[4 * c];
        vb[c] = rhi[4 * c];
      }
      float acc[NT][4];
      score_mtile<D, G>(va, vb, bfrag, acc);
      const bool ok_lo = tok0 + g < nv, ok_hi = tok0 + g + 8 < nv;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hd = nt * 8 + 2 * t + e;
          const float zl = ok_lo ? a.scale * acc[nt][e] : -INFINITY;
          const float zh = ok_hi ? a.scale * acc[nt][2 + e] : -INFINITY;
          if (hd < G) {
            float* zr = zs + hd * zp + j * S + tok0;
            zr[g] = zl;
            zr[g + 8] = zh;
          }
          float m = fmaxf(zl, zh);
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
          pmx[nt][e] = fmaxf(pmx[nt][e], m);
        }
    }
    if (g == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hd = nt * 8 + 2 * t + e;
          if (hd < G) pm[hd * spc + j] = pmx[nt][e];
        }
    }
    __syncwarp();
    if (lane == 0 && i + spw < cnt_w) {
      fence_proxy_async_smem();  // the slot's reads come before the copy that refills it
      issue(i + spw, phys_s[warp + (i + spw) * kFWarps]);
    }
  }
  __syncthreads();
  // run maxima per head, pushed to every CTA of the cluster
  for (int h = warp; h < G; h += kFWarps) {
    float m = -INFINITY;
    for (int j = lane; j < np; j += 32) m = fmaxf(m, pm[h * spc + j]);
    m = warp_max(m);
    if (lane < C) cluster.map_shared_rank(&mall[0][0], lane)[h * kFMaxCluster + rank] = m;
  }
  cluster.sync();
  // ---------------------------------------------------------------- 2. τ
  const int tpc = spc * S;
  const int n_tok = n_slots * S;
  float* zh = reinterpret_cast<float*>(ring);  // u = (α−1)·z of the head being solved
  const bool closed = ipow == 1 || ipow == 2;
  float* cand = zh + ((n_tok + 31) & ~31);
  const size_t words = static_cast<size_t>(a.words);
  for (int h = rank; h < G; h += C) {
    const size_t orow = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + h;
    float m = -INFINITY;
    for (int r = 0; r < C; ++r) m = fmaxf(m, mall[h][r]);
    float tau = INFINITY;  // no finite score: no support, zero output
    if (m > -INFINITY) {
      const float um = a.am1 * m;
      for (int i = 4 * tid; i < n_tok; i += 4 * kFThreads) {
        const int r = i / tpc;
        const float4 v = *reinterpret_cast<const float4*>(cluster.map_shared_rank(zs, r) + h * zp + (i - r * tpc));
        const float uu[4] = {a.am1 * v.x, a.am1 * v.y, a.am1 * v.z, a.am1 * v.w};
        *reinterpret_cast<float4*>(zh + i) = make_float4(uu[0], uu[1], uu[2], uu[3]);
        if (!closed) continue;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (uu[k] > um - 1.0f)
            atomicAdd(&tsh.hist[min(kTauBinsF - 1, static_cast<int>((um - uu[k]) * kTauBinsF))], 1);
      }
      __syncthreads();
      // β ∈ {1, 2}: bracket, candidates, pairwise support test and closed
      // form; otherwise Newton over every value from max u − 1 (f ≥ 0 there:
      // the maximum alone gives 1), one barrier per step, without a bracket
      tau = closed ? cta_solve_tau(zh, n_tok, um, cand, a.beta, ipow, tsh)
                   : cta_newton_tau(zh, n_tok, um, a.beta, ipow, tsh);
    }
    if (tid < C) cluster.map_shared_rank(s_tau, tid)[h] = tau;
    if (tid == 0 && a.tau_out) a.tau_out[orow] = tau;
    if (a.bits_out == nullptr && a.count_out == nullptr) {
      __syncthreads();  // zh, cand and tsh are reused by the next head
      continue;
    }
    int cnt = 0;
    for (int base = 0; base < n_tok; base += kFThreads) {
      const int i = base + tid;
      const bool in = i < n_tok && tau < INFINITY && zh[i] > tau;
      cnt += in ? 1 : 0;
      const unsigned int bal = __ballot_sync(0xffffffffu, in);
      if (a.bits_out && lane == 0 && i < n_tok) a.bits_out[orow * words + i / 32] = bal;
    }
    if (a.bits_out)
      for (int w = (n_tok + 31) / 32 + tid; w < a.words; w += kFThreads) a.bits_out[orow * words + w] = 0u;
    cnt = warp_sum(cnt);
    if (lane == 0) tsh.i[warp] = cnt;
    __syncthreads();
    if (tid == 0 && a.count_out) {
      int c = 0;
      for (int w = 0; w < kFWarps; ++w) c += tsh.i[w];
      a.count_out[orow] = c;
    }
    __syncthreads();  // zh, cand and tsh are reused by the next head
  }
  cluster.sync();

  // ---------------------------------------------------------------- 3. V
  // The run's support tokens (some head has u > τ; every valid token with
  // dense_v), listed in token order over the free ring, then read row by row:
  // warp w takes rows w·8 … w·8+7 of each block of 128, eight V rows in
  // flight per warp, p = [u − τ]_+^β from the scores in shared memory.
  int* tl = reinterpret_cast<int*>(ring);  // [np·S] token j·S + t of the run
  int ntl = 0;
  for (int x0 = 0; x0 < np * S; x0 += kFThreads) {
    const int x = x0 + tid;
    int sup = 0;
    if (x < np * S) {
      const int j = x / S;
      if (phys_s[j] >= 0 && x - j * S < nv_s[j]) {
        if (a.dense_v) {
          sup = 1;
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h)
            if (a.am1 * zs[h * zp + x] > s_tau[h]) sup = 1;
        }
      }
    }
    int tot;
    const int pos = block_exclusive_scan(sup, scan_scratch, &tot);
    if (sup) tl[ntl + pos] = x;
    ntl += tot;
  }
  __syncthreads();
  float acc[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
  // Each batch: eight V rows in flight per warp; lane q computes the weight
  // of (row q / G, head q mod G) once and the FMAs take it by shuffle, so the
  // loop body stays small (it runs once per launch on every SM: its
  // instructions are fetched cold).
  constexpr int kRowsInFlight = 8;
  constexpr int kPairs = kRowsInFlight * G;
  constexpr int kPerLane = (kPairs + 31) / 32;
#pragma unroll 1
  for (int e0 = warp * kRowsInFlight; e0 < ntl; e0 += kFWarps * kRowsInFlight) {
    // every row is loaded unconditionally (a row past the list reads list
    // entry e0, which exists, and is zeroed after): loads behind per-row
    // branches are issued one after another
    float v[kRowsInFlight][DPL];
#pragma unroll
    for (int r = 0; r < kRowsInFlight; ++r) {
      const int e = e0 + r;
      const bool in = e < ntl;
      const int tok = tl[in ? e : e0], j = tok / S;
      const bf16* src = static_cast<const bf16*>(a.v_pool) +
                        ((static_cast<size_t>(phys_s[j]) * a.Hkv + kvh) * S + (tok - j * S)) * D + lane * DPL;
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(src);
        v[r][0] = in ? __uint_as_float(w.x << 16) : 0.f;
        v[r][1] = in ? __uint_as_float(w.x & 0xffff0000u) : 0.f;
        v[r][2] = in ? __uint_as_float(w.y << 16) : 0.f;
        v[r][3] = in ? __uint_as_float(w.y & 0xffff0000u) : 0.f;
      } else {
        const uint32_t w = *reinterpret_cast<const unsigned int*>(src);
        v[r][0] = in ? __uint_as_float(w << 16) : 0.f;
        v[r][1] = in ? __uint_as_float(w & 0xffff0000u) : 0.f;
      }
    }
    float pl[kPerLane];
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
      const int q = k * 32 + lane, r = q / G, h = q - r * G;
      float pt = 0.f;
      if (q < kPairs && e0 + r < ntl) {
        const float w = a.am1 * zs[h * zp + tl[e0 + r]] - s_tau[h];
        if (w > 0.f) pt = pow_beta_fast(w, a.beta, ipow);
      }
      pl[k] = pt;
    }
#pragma unroll
    for (int r = 0; r < kRowsInFlight; ++r)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pt = __shfl_sync(0xffffffffu, pl[(r * G + h) / 32], (r * G + h) % 32);
#pragma unroll
        for (int x = 0; x < DPL; ++x) acc[h][x] = fmaf(pt, v[r][x], acc[h][x]);
      }
  }
  __syncthreads();  // the token list is read by every warp before the partials overwrite it
  // warp partials → CTA partial (warp order) → the owner's inbox
  float* red = reinterpret_cast<float*>(ring);  // [kFWarps][G][D], over the finished τ scratch
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) red[(warp * G + h) * D + lane * DPL + e] = acc[h][e];
  __syncthreads();
  for (int i = tid; i < G * D; i += kFThreads) {
    float pw[kFWarps];
#pragma unroll
    for (int w = 0; w < kFWarps; ++w) pw[w] = red[w * G * D + i];
    const int owner = i / f.chunk;
    cluster.map_shared_rank(inbox, owner)[rank * f.chunk + (i - owner * f.chunk)] = tree16(pw);
  }
  cluster.sync();

  // ---------------------------------------------------------------- 4. owner sums
  const int GD = G * D;
  for (int k = tid; k < f.chunk; k += kFThreads) {
    const int i = rank * f.chunk + k;
    if (i >= GD) break;
    float s = 0.f;
    for (int r = 0; r < C; ++r) s += inbox[r * f.chunk + k];
    const int h = i / D, d = i - h * D;
    a.out[(static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + h) * D + d] = s;
  }
}

// ------------------------------------------------------------------ host side
int round_up(int x, int m) { return (x + m - 1) / m * m; }

struct DeviceLimits {
  int sms = 0;
  int smem_optin = 0;
};

DeviceLimits device_limits() {
  static std::mutex mu;
  static std::vector<DeviceLimits> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  DeviceLimits& l = cache[dev];
  if (l.sms == 0) {
    cudaDeviceGetAttribute(&l.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&l.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  }
  return l;
}

// Geometry for C CTAs per unit; smem = 0 when it does not fit.
template <int D, int G>
FusedGeom plan(int C, int cap, int S, int smem_limit) {
  FusedGeom f{};
  f.C = C;
  f.spc = (cap + C - 1) / C;
  const int step = S >= 32 ? 1 : 32 / S;  // each CTA's tokens start on a 32-token word
  f.spc = round_up(f.spc, step);
  f.zpitch = f.spc * S + 4;
  f.tile_bytes = S * D * 2;
  f.chunk = (G * D + C - 1) / C;
  int off = 0;
  f.off_ints = off;
  off += round_up(4 * f.spc * 4, 128);
  f.off_pm = off;
  off += round_up(G * f.spc * 4, 128);
  f.off_zs = off;
  off += round_up(G * f.zpitch * 4, 128);
  f.off_inbox = off;
  off += round_up(C * f.chunk * 4, 128);
  f.off_ring = off;
  const int n_tok_max = cap * S;
  f.off_v = round_up(std::max(2 * round_up(n_tok_max, 32) * 4, kFWarps * G * D * 4), 128);
  const int pages_per_warp = (f.spc + kFWarps - 1) / kFWarps;
  const int avail = smem_limit - off;
  const int spw = std::min(std::min(pages_per_warp, kFMaxSpw), avail / (kFWarps * f.tile_bytes));
  if (spw < 1) return FusedGeom{};
  f.spw = spw;
  const int ring_k = kFWarps * spw * f.tile_bytes;
  const int ring = std::max(ring_k, f.off_v);
  if (off + ring > smem_limit) return FusedGeom{};
  f.smem = off + ring;
  return f;
}

template <int D, int G>
int max_active_clusters(int C, int smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(C), 1);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fused_decode_kernel<D, G, 0>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int D, int G>
cudaError_t prepare_kernel(int smem_limit) {
  static std::mutex mu;
  static std::vector<char> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(done.size()) <= dev) done.resize(dev + 1, 0);
  if (done[dev]) return cudaSuccess;
  for (auto kern : {fused_decode_kernel<D, G, 0>, fused_decode_kernel<D, G, 1>, fused_decode_kernel<D, G, 2>}) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_limit);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  done[dev] = 1;
  return cudaSuccess;
}

// Chosen geometry per (device, units, cap, S): the largest cluster whose
// clusters for all units are resident together, else one CTA per unit.
template <int D, int G>
FusedGeom choose(int units, int cap, int S) {
  struct Entry {
    int dev, units, cap, S;
    FusedGeom f;
  };
  static std::mutex mu;
  static std::vector<Entry> memo;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : memo)
      if (e.dev == dev && e.units == units && e.cap == cap && e.S == S) return e.f;
  }
  const DeviceLimits lim = device_limits();
  cudaFuncAttributes fa{};
  FusedGeom best{};
  const bool have_attr = cudaFuncGetAttributes(&fa, fused_decode_kernel<D, G, 0>) == cudaSuccess;
  const int smem_limit = lim.smem_optin - static_cast<int>(fa.sharedSizeBytes);
  if (have_attr && prepare_kernel<D, G>(smem_limit) == cudaSuccess) {
    for (int C = kFMaxCluster; C >= 1; C >>= 1) {
      if (C > 1 && (cap + C - 1) / C < 2) continue;
      const FusedGeom f = plan<D, G>(C, cap, S, smem_limit);
      if (f.smem == 0) continue;
      if (C == 1) {
        best = f;
        break;
      }
      if (max_active_clusters<D, G>(C, f.smem) >= units) {
        best = f;
        break;
      }
    }
  }
  std::lock_guard<std::mutex> lock(mu);
  memo.push_back(Entry{dev, units, cap, S, best});
  return best;
}

}  // namespace

template <int D, int G>
bool fused_decode_fits(int units, int cap, int S) {
  if (S % 16 != 0 || cap < 1) return false;
  return choose<D, G>(units, cap, S).smem > 0;
}

template <int D, int G>
int fused_decode_cluster(int units, int cap, int S) {
  if (S % 16 != 0 || cap < 1) return 0;
  const FusedGeom f = choose<D, G>(units, cap, S);
  return f.smem > 0 ? f.C : 0;
}

template <int D, int G>
cudaError_t run_fused_decode(DecodeArgs& a, int units, cudaStream_t st) {
  const FusedGeom f = choose<D, G>(units, a.cap, a.S);
  if (f.smem == 0) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(f.C), static_cast<unsigned>(units));
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(f.smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(f.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, a.ipow == 1 ? fused_decode_kernel<D, G, 1> : (a.ipow == 2 ? fused_decode_kernel<D, G, 2> : fused_decode_kernel<D, G, 0>),
      a, f);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

#define EKV_FUSED_INST(DD, GG)                                            \
  template bool fused_decode_fits<DD, GG>(int, int, int);                 \
  template int fused_decode_cluster<DD, GG>(int, int, int);               \
  template cudaError_t run_fused_decode<DD, GG>(DecodeArgs&, int, cudaStream_t);
EKV_FUSED_INST(128, 1)
EKV_FUSED_INST(128, 2)
EKV_FUSED_INST(128, 4)
EKV_FUSED_INST(128, 8)
EKV_FUSED_INST(128, 16)
EKV_FUSED_INST(64, 1)
EKV_FUSED_INST(64, 2)
EKV_FUSED_INST(64, 4)
EKV_FUSED_INST(64, 8)
EKV_FUSED_INST(64, 16)
#undef EKV_FUSED_INST

}  // namespace ekv
