// Sparse α-entmax decode over the selected pages — EntmaxKV summary page
// (gist.science/fr/paper/2605.21649) §2.C, "Attention Entmax Parcimonieuse",
// with the support-only V read that §2 and §3 make exact: if the selected
// tokens contain the α-entmax support, the output equals the full-cache one.
//
// Three kernels, all on the caller's stream:
//  1. qk: z = scale·q·k for every valid token of every selected page and the
//     G query heads of the unit.  A (page, KV head) K tile is one contiguous
//     block of S rows; for bf16 each 16-token half is the A operand of a
//     tensor-core MMA (m16n8k16) whose B operand is the group's queries, with
//     rows loaded straight into fragment registers (the same k permutation
//     as the page-score kernel).  Scores land in an L2-resident scratch with
//     per-page and per-CTA maxima.
//  2. tau: per query head, τ with Σ_i [u_i − τ]_+^β = 1, u = (α−1)·z,
//     β = 1/(α−1).  f(τ) = Σ[u − τ]_+^β is convex and decreasing, so Newton's
//     method started left of the root rises to it without overshooting.  The
//     start comes from a 256-bin histogram of u over (max u − 1, max u]: if
//     c values exceed an edge e then τ ≥ e − c^(−1/β) (c of them would give
//     mass ≥ 1 at that τ), which lands within a bin of the root.  For β ∈ {1,2}
//     the final τ is the closed form on the support found.
//  3. pv: each CTA lists the selected pages of its run that hold support
//     (some head has a token with u > τ) and its warps read only those V
//     pages, one whole row per load instruction; CTA partials are added by
//     the unit's last CTA (an atomic ticket, no waiting) in CTA order, so
//     results are deterministic.
#include "decode.cuh"

namespace ekv {

namespace {

// ------------------------------------------------------------------ 1. qk (bf16 tensor cores)
constexpr int kQkWarps = kQkTokensPerCta / 32;

template <int D, int G>
__global__ void __launch_bounds__(32 * kQkWarps, 2) qk_mma_kernel(DecodeArgs a) {
  // the τ kernel that follows is let in only at the end: its CTAs, resident
  // early, would take the SM slots of this launch's many short CTAs
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int KP = D / 32;          // 32-element chunks per K row
  constexpr int NT = (G + 7) / 8;     // 8-head tiles of the B operand
  __shared__ unsigned int cta_key[G];
  const int split = blockIdx.x, unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int S = a.S;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int ppc = kQkTokensPerCta / S;  // pages per CTA
  const int s_begin = split * ppc;
  if (tid < G) cta_key[tid] = 0u;
  if (split == 0 && tid == 0) a.ws.counter[unit] = 0;
  __syncthreads();

  // this warp's 32 token rows form two 16-row m-tiles of one or two pages
  const int row0 = warp * 32;
  int phys[2], nv[2], slot[2];
  bool live[2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int r = row0 + mt * 16;
    slot[mt] = s_begin + r / S;
    live[mt] = slot[mt] < n_slots;
    phys[mt] = -1;
    nv[mt] = 0;
    if (live[mt]) phys[mt] = slot_page(a, unit, b, slot[mt], P, L, &nv[mt]);
  }
  // K rows straight into A fragments: rows g and g + 8 of each m-tile
  uint4 va[2][KP], vb[2][KP];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int tok0 = (row0 + mt * 16) % S;
    const bool ok_lo = phys[mt] >= 0 && tok0 + g < nv[mt];
    const bool ok_hi = phys[mt] >= 0 && tok0 + g + 8 < nv[mt];
    const bf16* kb = static_cast<const bf16*>(a.k_pool) +
                     ((static_cast<size_t>(phys[mt] < 0 ? 0 : phys[mt]) * a.Hkv + kvh) * S + tok0) * D;
    const uint4* row_lo = reinterpret_cast<const uint4*>(kb + g * D) + t;
    const uint4* row_hi = reinterpret_cast<const uint4*>(kb + (g + 8) * D) + t;
#pragma unroll
    for (int c = 0; c < KP; ++c) {
      va[mt][c] = ok_lo ? __ldcs(row_lo + 4 * c) : make_uint4(0, 0, 0, 0);
      vb[mt][c] = ok_hi ? __ldcs(row_hi + 4 * c) : make_uint4(0, 0, 0, 0);
    }
  }
  // B fragments: the group's queries under the same k permutation
  uint32_t bfrag[2 * KP][NT][2];
  load_q_frags<D, G>(a, b, kvh, g, t, bfrag);
  const size_t zrow = static_cast<size_t>(a.cap) * S;
  float pm[2][NT][2];  // page maxima per m-tile for heads 2t, 2t+1 of each tile
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    float acc[NT][4];
    score_mtile<D, G>(va[mt], vb[mt], bfrag, acc);
    const int tok0 = (row0 + mt * 16) % S;
    const bool ok_lo = phys[mt] >= 0 && tok0 + g < nv[mt];
    const bool ok_hi = phys[mt] >= 0 && tok0 + g + 8 < nv[mt];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hd = nt * 8 + 2 * t + e;
        const float zl = ok_lo ? a.scale * acc[nt][e] : -INFINITY;
        const float zh = ok_hi ? a.scale * acc[nt][2 + e] : -INFINITY;
        if (live[mt] && hd < G) {
          float* zr = a.ws.zbuf + (static_cast<size_t>(unit) * G + hd) * zrow + static_cast<size_t>(slot[mt]) * S + tok0;
          zr[g] = zl;
          zr[g + 8] = zh;
        }
        float m = fmaxf(zl, zh);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        pm[mt][nt][e] = m;
      }
  }
  // page maxima: one page per m-tile (S = 16) or per warp (S = 32)
  if (g == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hd = nt * 8 + 2 * t + e;
        if (hd >= G) continue;
        float* prow = a.ws.pmax + (static_cast<size_t>(unit) * G + hd) * a.cap;
        if (S == 16) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            if (live[mt]) {
              prow[slot[mt]] = pm[mt][nt][e];
              if (pm[mt][nt][e] > -INFINITY) atomicMax(&cta_key[hd], float_key(pm[mt][nt][e]));
            }
        } else if (live[0]) {
          const float m = fmaxf(pm[0][nt][e], pm[1][nt][e]);
          prow[slot[0]] = m;
          if (m > -INFINITY) atomicMax(&cta_key[hd], float_key(m));
        }
      }
  }
  __syncthreads();
  if (tid < G) {
    const unsigned int k = cta_key[tid];
    a.ws.cmax[(static_cast<size_t>(unit) * G + tid) * a.ws.nqk + split] = k == 0u ? -INFINITY : key_float(k);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ 1'. qk (CUDA cores, fp32 caches)
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) qk_cc_kernel(DecodeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // dependents let in at the end, as qk_mma_kernel
  constexpr int PAD = 16 / sizeof(T);
  constexpr int RP = D + PAD;  // padded row pitch: rows start in different bank groups
  constexpr int TP = 4;        // pages staged per round
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* q_s = reinterpret_cast<float*>(smem_raw);
  T* ktile = reinterpret_cast<T*>(smem_raw + G * D * sizeof(float));
  __shared__ int s_phys[TP], s_nv[TP];
  __shared__ unsigned int cta_key[G];

  const int split = blockIdx.x, unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, S = a.S;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int ppc = kQkTokensPerCta / S;
  const int s0 = split * ppc, s1 = min(s0 + ppc, n_slots);
  if (split == 0 && tid == 0) a.ws.counter[unit] = 0;

  const T* qb = static_cast<const T*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G) * D;
  for (int i = tid; i < G * D; i += blockDim.x) q_s[i] = to_f32(qb[i]);
  if (tid < G) cta_key[tid] = 0u;
  __syncthreads();

  const size_t zrow = static_cast<size_t>(a.cap) * S;
  constexpr int CPR = D * sizeof(T) / 16;  // 16 B chunks per row
  for (int base = s0; base < s1; base += TP) {
    const int np = min(TP, s1 - base);
    if (tid < np) {
      int nv;
      s_phys[tid] = slot_page(a, unit, b, base + tid, P, L, &nv);
      s_nv[tid] = nv;
    }
    __syncthreads();
    for (int i = tid; i < np * S * CPR; i += blockDim.x) {
      const int tp = i / (S * CPR), r = (i / CPR) % S, c = i % CPR;
      const int phys = s_phys[tp];
      if (phys >= 0 && r < s_nv[tp]) {
        const uint4* src = reinterpret_cast<const uint4*>(
            static_cast<const T*>(a.k_pool) + ((static_cast<size_t>(phys) * a.Hkv + kvh) * S + r) * D) + c;
        *reinterpret_cast<uint4*>(ktile + (tp * S + r) * RP + c * (16 / sizeof(T))) = __ldcs(src);
      }
    }
    __syncthreads();
    const int items = (TP * G * S + 31) / 32 * 32;  // whole warps (page maxima shuffle across S lanes)
    for (int it = tid; it < items; it += blockDim.x) {
      const int tp = it / (G * S), g = (it / S) % G, t = it % S;
      float z = -INFINITY;
      if (tp < np && t < s_nv[tp]) {
        const T* kr = ktile + (tp * S + t) * RP;
        const float* qr = q_s + g * D;
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          float v[8];
          load8(kr + 8 * c, v);
          const float4 q0 = *reinterpret_cast<const float4*>(qr + 8 * c);
          const float4 q1 = *reinterpret_cast<const float4*>(qr + 8 * c + 4);
          acc = ffma2(make_float2(q0.x, q0.y), make_float2(v[0], v[1]), acc);
          acc = ffma2(make_float2(q0.z, q0.w), make_float2(v[2], v[3]), acc);
          acc = ffma2(make_float2(q1.x, q1.y), make_float2(v[4], v[5]), acc);
          acc = ffma2(make_float2(q1.z, q1.w), make_float2(v[6], v[7]), acc);
        }
        z = a.scale * (acc.x + acc.y);
      }
      const size_t row = static_cast<size_t>(unit) * G + g;
      if (tp < np) a.ws.zbuf[row * zrow + static_cast<size_t>(base + tp) * S + t] = z;
      float pmx = z;
      for (int o = S / 2; o > 0; o >>= 1) pmx = fmaxf(pmx, __shfl_xor_sync(0xffffffffu, pmx, o));
      if (t == 0 && tp < np) {
        a.ws.pmax[row * a.cap + base + tp] = pmx;
        if (pmx > -INFINITY) atomicMax(&cta_key[g], float_key(pmx));
      }
    }
    __syncthreads();
  }
  __syncthreads();
  if (tid < G) {
    const unsigned int k = cta_key[tid];
    a.ws.cmax[(static_cast<size_t>(unit) * G + tid) * a.ws.nqk + split] = k == 0u ? -INFINITY : key_float(k);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ 2. tau
constexpr int kTauThreads = 256;
constexpr int kTauBins = 256;

// Sums three doubles over the block; every thread gets the totals.
__device__ __forceinline__ void block_sum3(double& x, double& y, double& z, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, o);
    y += __shfl_xor_sync(0xffffffffu, y, o);
    z += __shfl_xor_sync(0xffffffffu, z, o);
  }
  __syncthreads();
  if (lane == 0) {
    scratch[3 * warp] = x;
    scratch[3 * warp + 1] = y;
    scratch[3 * warp + 2] = z;
  }
  __syncthreads();
  x = y = z = 0.0;
  for (int w = 0; w < nw; ++w) {
    x += scratch[3 * w];
    y += scratch[3 * w + 1];
    z += scratch[3 * w + 2];
  }
}

constexpr int kTauCand = 4096;

template <int VPT>
__global__ void __launch_bounds__(kTauThreads) tau_kernel(DecodeArgs a, int G) {
  grid_dep_enter();
  const int row = blockIdx.x, unit = row / G, g = row % G, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  __shared__ float f_scratch[32];
  __shared__ double d_scratch[3 * 32];
  __shared__ int i_scratch[32];
  __shared__ int hist[kTauBins];
  __shared__ float cand[kTauCand];
  __shared__ double s_tau;
  int L;
  const int P = seq_pages(a.seq_lens, b, a.S, a.max_pages, &L);
  const int n = unit_slots(a, unit, P) * a.S;
  const float* z = a.ws.zbuf + static_cast<size_t>(row) * a.cap * a.S;
  const size_t orow = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + g;
  const float am1 = a.am1, beta = a.beta;
  const int ib = a.ibeta;

  float m = -INFINITY;
  for (int s = tid; s < a.ws.nqk; s += nt) m = fmaxf(m, a.ws.cmax[static_cast<size_t>(row) * a.ws.nqk + s]);
  m = block_reduce(m, f_scratch, [](float x, float y) { return fmaxf(x, y); });

  float uv[VPT > 0 ? VPT : 1];
#pragma unroll
  for (int k = 0; k < (VPT > 0 ? VPT : 1); ++k) {
    const int i = tid + k * nt;
    uv[k] = (VPT > 0 && i < n) ? am1 * z[i] : -INFINITY;
  }
  // applies fn(u) to every value of the row (registers, or a pass over the scratch)
  auto for_values = [&](auto fn) {
    if constexpr (VPT > 0) {
#pragma unroll
      for (int k = 0; k < VPT; ++k) fn(uv[k]);
    } else {
      for (int i = tid; i < n; i += nt) fn(am1 * z[i]);
    }
  };

  float tau_f = INFINITY;  // no token: no support, zero output
  if (n > 0 && m > -INFINITY) {
    const float um = am1 * m;
    // 1. lower bracket from the histogram of u over (um − 1, um]
    for (int i = tid; i < kTauBins; i += nt) hist[i] = 0;
    __syncthreads();
    for_values([&](float u) {
      if (u > um - 1.0f) atomicAdd(&hist[min(kTauBins - 1, static_cast<int>((um - u) * kTauBins))], 1);
    });
    __syncthreads();
    float cb = um - 1.0f;
    {
      const int h = tid < kTauBins ? hist[tid] : 0;
      int total;
      const int c = block_exclusive_scan(h, i_scratch, &total) + h;  // values in bins 0..tid
      if (tid < kTauBins && c > 0)
        cb = fmaxf(cb, um - static_cast<float>(tid + 1) / kTauBins - powf(static_cast<float>(c), -1.0f / beta));
    }
    cb = block_reduce(cb, f_scratch, [](float x, float y) { return fmaxf(x, y); });
    const double tau_lo = static_cast<double>(cb) - 1e-6 * (1.0 + fabs(static_cast<double>(um)));
    // 2. τ only rises from tau_lo, so only values above it can ever count:
    //    compact them (block-scan order, deterministic) and iterate on those
    int mine = 0;
    for_values([&](float u) { mine += static_cast<double>(u) > tau_lo ? 1 : 0; });
    int nc;
    int pos = block_exclusive_scan(mine, i_scratch, &nc);
    const bool fits = nc <= kTauCand;
    if (fits)
      for_values([&](float u) {
        if (static_cast<double>(u) > tau_lo) cand[pos++] = u;
      });
    __syncthreads();
    auto sums = [&](double t, double& f, double& df, bool block) {
      f = 0.0;
      df = 0.0;
      auto term = [&](float u) {
        const double w = static_cast<double>(u) - t;
        if (w > 0.0) {
          if (ib == 1) {
            f += w;
            df += 1.0;
          } else if (ib == 2) {
            f += w * w;
            df += w;
          } else {
            const double wb1 = pow(w, static_cast<double>(beta) - 1.0);
            f += wb1 * w;
            df += wb1;
          }
        }
      };
      if (fits) {
        for (int i = block ? tid : lane; i < nc; i += block ? nt : 32) term(cand[i]);
      } else {
        for_values(term);
      }
      if (block) {
        double unused = 0.0;
        block_sum3(f, df, unused, d_scratch);
      } else {
        f = warp_sum(f);
        df = warp_sum(df);
      }
    };
    // one warp iterates when the candidates are few (no block barriers)
    const bool solo = fits && nc <= 1024;
    if (!solo || warp == 0) {
      double tau = tau_lo;
      for (int it = 0; it < 100; ++it) {
        double f, df;
        sums(tau, f, df, !solo);
        if (it == 0 && f < 1.0) {  // bracket missed (rounding): restart from max u − 1
          tau = static_cast<double>(um) - 1.0;
          continue;
        }
        const double step = norm_newton_step<double>(f - 1.0, df, static_cast<double>(beta));
        if (!(step > 0.0)) break;
        tau += step;
        if (step <= 1e-11 * fmax(1.0, fabs(tau))) break;
      }
      if (ib == 1 || ib == 2) {
        // closed form on the support found: β = 1: τ = (Σu − 1)/k;
        // β = 2: τ = M − √(M² − Q + 1/k) with M, Q the mean and mean square
        for (int rep = 0; rep < 4; ++rep) {
          double c = 0.0, s1 = 0.0, s2 = 0.0;
          auto add = [&](float u) {
            if (static_cast<double>(u) > tau) {
              c += 1.0;
              s1 += u;
              s2 += static_cast<double>(u) * u;
            }
          };
          if (fits) {
            for (int i = solo ? lane : tid; i < nc; i += solo ? 32 : nt) add(cand[i]);
          } else {
            for_values(add);
          }
          if (solo) {
            c = warp_sum(c);
            s1 = warp_sum(s1);
            s2 = warp_sum(s2);
          } else {
            block_sum3(c, s1, s2, d_scratch);
          }
          if (c < 1.0) break;
          double t_new;
          if (ib == 1) {
            t_new = (s1 - 1.0) / c;
          } else {
            const double M = s1 / c, Q = s2 / c;
            t_new = M - sqrt(fmax(M * M - Q + 1.0 / c, 0.0));
          }
          if (t_new == tau) break;
          tau = t_new;
        }
      }
      if (tid == 0) s_tau = tau;
    }
    __syncthreads();
    tau_f = static_cast<float>(s_tau);
  }

  // support of this head with the fp32 threshold every later stage uses
  int cnt = 0;
  const int words = a.words;
  for (int base = 0; base < (n + nt - 1) / nt * nt; base += nt) {
    const int i = base + tid;
    bool in = false;
    if constexpr (VPT > 0) {
      const int k = base / nt;
#pragma unroll
      for (int kk = 0; kk < VPT; ++kk)
        if (kk == k) in = i < n && uv[kk] > tau_f;
    } else {
      in = i < n && am1 * z[i] > tau_f;
    }
    cnt += in ? 1 : 0;
    const unsigned int bal = __ballot_sync(0xffffffffu, in);
    if (a.bits_out && lane == 0 && (i >> 5) < words) a.bits_out[orow * words + (i >> 5)] = bal;
  }
  cnt = block_reduce(cnt, i_scratch, [](int x, int y) { return x + y; });
  if (a.bits_out)
    for (int w = (n + 31) / 32 + tid; w < words; w += nt) a.bits_out[orow * words + w] = 0u;
  if (tid == 0) {
    a.ws.taus[row] = tau_f;
    if (a.tau_out) a.tau_out[orow] = tau_f;
    if (a.count_out) a.count_out[orow] = cnt;
  }
}

// ------------------------------------------------------------------ 3. pv
constexpr int kPvWarps = 8;
constexpr int kPvRows = 32;  // V rows in flight per warp (a multiple of the page size)

// One lane's share of a V row (DPL = D/32 consecutive elements), loaded in
// its stored form with one aligned load and widened to fp32 when used.
template <typename T, int DPL>
struct PvRaw;
template <>
struct PvRaw<bf16, 4> {
  using Row = uint2;
  static __device__ __forceinline__ Row zero() { return make_uint2(0u, 0u); }
  static __device__ __forceinline__ Row load(const bf16* p) { return *reinterpret_cast<const uint2*>(p); }
  static __device__ __forceinline__ void widen(Row w, float* v) {
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xffff0000u);
  }
};
template <>
struct PvRaw<bf16, 2> {
  using Row = uint32_t;
  static __device__ __forceinline__ Row zero() { return 0u; }
  static __device__ __forceinline__ Row load(const bf16* p) { return *reinterpret_cast<const uint32_t*>(p); }
  static __device__ __forceinline__ void widen(Row w, float* v) {
    v[0] = __uint_as_float(w << 16);
    v[1] = __uint_as_float(w & 0xffff0000u);
  }
};
template <>
struct PvRaw<float, 4> {
  using Row = float4;
  static __device__ __forceinline__ Row zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  static __device__ __forceinline__ Row load(const float* p) { return *reinterpret_cast<const float4*>(p); }
  static __device__ __forceinline__ void widen(Row w, float* v) {
    v[0] = w.x;
    v[1] = w.y;
    v[2] = w.z;
    v[3] = w.w;
  }
};
template <>
struct PvRaw<float, 2> {
  using Row = float2;
  static __device__ __forceinline__ Row zero() { return make_float2(0.f, 0.f); }
  static __device__ __forceinline__ Row load(const float* p) { return *reinterpret_cast<const float2*>(p); }
  static __device__ __forceinline__ void widen(Row w, float* v) {
    v[0] = w.x;
    v[1] = w.y;
  }
};

// Two CTAs per SM where the batch of packed rows, the accumulators and the
// weights fit in 128 registers a thread, one otherwise (no spills).
template <typename T, int D, int G>
constexpr int pv_min_blocks() {
  constexpr int regs = kPvRows * static_cast<int>(sizeof(typename PvRaw<T, D / 32>::Row)) / 4 + G * (D / 32) + G + 24;
  return regs <= 120 ? 2 : 1;
}

// PS: the page size (16 or 32), a template parameter so that every row of a
// batch is addressed from its page's base with a constant offset.
template <typename T, int D, int G, int PS>
__global__ void __launch_bounds__(32 * kPvWarps, pv_min_blocks<T, D, G>()) pv_kernel(DecodeArgs a) {
  static_assert(kPvRows % PS == 0, "a batch holds whole pages");
  grid_dep_enter();
  constexpr int DPL = D / 32;  // output columns per lane
  extern __shared__ __align__(16) float red[];  // [kPvWarps][G][D]
  __shared__ float s_tau[G];
  __shared__ int s_list[32 * kPvWarps], s_phys[32 * kPvWarps], s_nv[32 * kPvWarps];
  __shared__ int scan_scratch[32];
  __shared__ int s_last;

  const int split = blockIdx.x, unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int S = PS;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int s0 = split * a.spp_pv, s1 = min(s0 + a.spp_pv, n_slots);
  if (tid < G) s_tau[tid] = a.ws.taus[static_cast<size_t>(unit) * G + tid];
  __syncthreads();

  float acc[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
  const size_t zrow = static_cast<size_t>(a.cap) * S;

  for (int w0 = s0; w0 < s1; w0 += blockDim.x) {
    // the window's pages that hold support, in ascending order; each thread
    // resolves its slot's page id in the same pass as the support test
    const int slot = w0 + tid;
    int sup = 0, phys = -1, nv = 0;
    if (slot < s1) {
      phys = slot_page(a, unit, b, slot, P, L, &nv);
      if (a.dense_v) {
        sup = 1;
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h)
          if (a.am1 * a.ws.pmax[(static_cast<size_t>(unit) * G + h) * a.cap + slot] > s_tau[h]) sup = 1;
      }
      if (phys < 0) sup = 0;
    }
    int nsup;
    const int pos = block_exclusive_scan(sup, scan_scratch, &nsup);
    if (sup) {
      s_list[pos] = slot;
      s_phys[pos] = phys;
      s_nv[pos] = nv;
    }
    __syncthreads();
    // warp w takes PP consecutive listed pages per batch (PP·S = kPvRows
    // rows: two 16-token pages or one 32-token page); row r of the batch is
    // token r mod S of page r / S.  The rows stay packed until used, so a
    // whole batch is in flight; lane r computes row r's weight per head.
    constexpr int PP = kPvRows / S;
    for (int e0 = warp * PP; e0 < nsup; e0 += kPvWarps * PP) {
      const T* vbase[PP];
      int nvp[PP];
#pragma unroll
      for (int q = 0; q < PP; ++q) {
        const bool ok = e0 + q < nsup;
        nvp[q] = ok ? s_nv[e0 + q] : 0;
        vbase[q] = static_cast<const T*>(a.v_pool) +
                   ((static_cast<size_t>(ok ? s_phys[e0 + q] : 0) * a.Hkv + kvh) * S) * D + lane * DPL;
      }
      typename PvRaw<T, DPL>::Row raw[kPvRows];
#pragma unroll
      for (int r = 0; r < kPvRows; ++r)
      {
        // unconditional load of a row inside the page tile, zeroed after
        const auto x = PvRaw<T, DPL>::load(vbase[r / S] + (r % S) * D);
        raw[r] = (r % S) < nvp[r / S] ? x : PvRaw<T, DPL>::zero();
      }
      float p[G];
      {
        const int e = e0 + lane / S, t = lane % S;
        const bool ok = e < nsup && t < s_nv[e];
        const size_t zi = ok ? static_cast<size_t>(s_list[e]) * S + t : 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          p[h] = 0.f;
          if (ok) {
            const float w = a.am1 * a.ws.zbuf[(static_cast<size_t>(unit) * G + h) * zrow + zi] - s_tau[h];
            if (w > 0.f) p[h] = pow_beta(w, a.beta, a.ipow);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kPvRows; ++r) {
        float v[DPL];
        PvRaw<T, DPL>::widen(raw[r], v);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float ph_t = __shfl_sync(0xffffffffu, p[h], r);
#pragma unroll
          for (int e2 = 0; e2 < DPL; ++e2) acc[h][e2] = fmaf(ph_t, v[e2], acc[h][e2]);
        }
      }
    }
    __syncthreads();
  }

  // CTA partial → workspace; the unit's last CTA adds the partials in order
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) red[(warp * G + h) * D + lane * DPL + e] = acc[h][e];
  __syncthreads();
  float* part = a.ws.part + (static_cast<size_t>(unit) * a.ws.npv + split) * G * D;
  for (int i = tid; i < G * D; i += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < kPvWarps; ++w) s += red[w * G * D + i];
    part[i] = s;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int ticket = atomicAdd(&a.ws.counter[unit], 1);
    s_last = ticket == a.ws.npv - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* part0 = a.ws.part + static_cast<size_t>(unit) * a.ws.npv * G * D;
  for (int i = tid; i < G * D; i += blockDim.x) {
    float s = 0.f;
    for (int sp = 0; sp < a.ws.npv; ++sp) s += __ldcg(part0 + static_cast<size_t>(sp) * G * D + i);
    const int h = i / D, j = i % D;
    a.out[(static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + h) * D + j] = s;
  }
  if (tid == 0) a.ws.counter[unit] = 0;
}

template <typename T, int D, int G>
cudaError_t launch_pv(DecodeArgs& a, int U, cudaStream_t st) {
  void (*kernel)(DecodeArgs) = a.S == 16 ? pv_kernel<T, D, G, 16> : pv_kernel<T, D, G, 32>;
  const size_t pv_smem = static_cast<size_t>(kPvWarps) * G * D * sizeof(float);
  if (pv_smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pv_smem));
    if (e != cudaSuccess) return e;
  }
  const dim3 gp(static_cast<unsigned>(a.ws.npv), static_cast<unsigned>(U));
  const cudaError_t e = launch_k(kernel, gp, 32 * kPvWarps, pv_smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t run_decode(DecodeArgs& a, int U, cudaStream_t st) {
  cudaError_t e;
  const dim3 gq(static_cast<unsigned>(a.ws.nqk), static_cast<unsigned>(U));
  if constexpr (sizeof(T) == 2) {
    {
    const cudaError_t le_ = launch_k(qk_mma_kernel<D, G>, gq, 32 * kQkWarps, 0, st, a);
    if (le_ != cudaSuccess) return le_;
  }
  } else {
    const size_t smem = static_cast<size_t>(G) * D * sizeof(float) + 4 * static_cast<size_t>(a.S) * (D + 16 / sizeof(T)) * sizeof(T);
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(qk_cc_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    {
    const cudaError_t le_ = launch_k(qk_cc_kernel<T, D, G>, gq, 256, smem, st, a);
    if (le_ != cudaSuccess) return le_;
  }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_max = a.cap * a.S;
  if (n_max <= 16 * kTauThreads)
    {
    const cudaError_t le_ = launch_k(tau_kernel<16>, U * G, kTauThreads, 0, st, a, G);
    if (le_ != cudaSuccess) return le_;
  }
  else if (n_max <= 64 * kTauThreads)
    {
    const cudaError_t le_ = launch_k(tau_kernel<64>, U * G, kTauThreads, 0, st, a, G);
    if (le_ != cudaSuccess) return le_;
  }
  else
    {
    const cudaError_t le_ = launch_k(tau_kernel<0>, U * G, kTauThreads, 0, st, a, G);
    if (le_ != cudaSuccess) return le_;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_pv<T, D, G>(a, U, st);
}

}  // namespace

template <int D, int G>
cudaError_t run_dense_v_pass(DecodeArgs& a, int units, cudaStream_t st) {
  return launch_pv<bf16, D, G>(a, units, st);
}
#define EKV_PV_INST(DD, GG) template cudaError_t run_dense_v_pass<DD, GG>(DecodeArgs&, int, cudaStream_t);
EKV_PV_INST(128, 1)
EKV_PV_INST(128, 2)
EKV_PV_INST(128, 4)
EKV_PV_INST(128, 8)
EKV_PV_INST(128, 16)
EKV_PV_INST(64, 1)
EKV_PV_INST(64, 2)
EKV_PV_INST(64, 4)
EKV_PV_INST(64, 8)
EKV_PV_INST(64, 16)
#undef EKV_PV_INST

int decode_kernel_count(const ekv_cache& c, const ekv_seqs& s, int Hq, int cap, int dense_v) {
  const int G = Hq / c.num_kv_heads, U = s.batch * c.num_kv_heads;
  if (c.dtype != EKV_BF16 || U > 65535) return 3;
#define EKV_CNT_CASE(DD, GG)                                                                 \
  if (c.head_dim == DD && G == GG)                                                           \
    switch (choose_decode_path<DD, GG>(U, cap, c.page_size, dense_v)) {                           \
      case DecodePath::kFused: return 1;                                                            \
      case DecodePath::kSplit: return dense_v ? 3 : 2;                                              \
      default: return 3;                                                                            \
    }
  EKV_CNT_CASE(128, 1) EKV_CNT_CASE(128, 2) EKV_CNT_CASE(128, 4) EKV_CNT_CASE(128, 8) EKV_CNT_CASE(128, 16)
  EKV_CNT_CASE(64, 1) EKV_CNT_CASE(64, 2) EKV_CNT_CASE(64, 4) EKV_CNT_CASE(64, 8) EKV_CNT_CASE(64, 16)
#undef EKV_CNT_CASE
  return 3;
}

cudaError_t launch_decode(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                          float scale, float alpha, const int32_t* sel, const int32_t* n_sel,
                          int cap, int dense_v, float* out, float* tau, int32_t* support_count,
                          uint32_t* support_bits, const DecodeWs& ws, cudaStream_t st) {
  DecodeArgs a{};
  a.k_pool = c.k_pool;
  a.v_pool = c.v_pool;
  a.page_table = s.page_table;
  a.seq_lens = s.seq_lens;
  a.q = q;
  a.sel = sel;
  a.n_sel = n_sel;
  a.out = out;
  a.tau_out = tau;
  a.count_out = support_count;
  a.bits_out = support_bits;
  a.ws = ws;
  a.scale = scale;
  a.am1 = alpha - 1.0f;
  a.beta = static_cast<float>(1.0 / (static_cast<double>(alpha) - 1.0));
  a.ibeta = (alpha == 2.0f) ? 1 : (alpha == 1.5f ? 2 : 0);
  {
    const double bd = 1.0 / (static_cast<double>(alpha) - 1.0);
    a.ipow = (bd == 1.0 || bd == 2.0 || bd == 3.0 || bd == 4.0) ? static_cast<int>(bd) : 0;
  }
  a.Hkv = c.num_kv_heads;
  a.Hq = Hq;
  a.S = c.page_size;
  a.num_phys = c.num_phys_pages;
  a.max_pages = s.max_pages;
  a.cap = cap;
  a.spp_pv = (cap + ws.npv - 1) / ws.npv;
  a.dense_v = dense_v;
  a.words = (cap * c.page_size + 31) / 32;
  const int G = Hq / c.num_kv_heads, U = s.batch * c.num_kv_heads;
#define EKV_DEC_CASE(TT, DD, GG) \
  if (c.head_dim == DD && G == GG) return run_decode<TT, DD, GG>(a, U, st);
#define EKV_DEC_BF16(DD, GG)                                                         \
  if (c.head_dim == DD && G == GG) {                                                 \
    switch (choose_decode_path<DD, GG>(U, cap, c.page_size, dense_v)) {              \
      case DecodePath::kFused: return run_fused_decode<DD, GG>(a, U, st);            \
      case DecodePath::kSplit: return run_split_decode<DD, GG>(a, U, st);            \
      default: return run_decode<bf16, DD, GG>(a, U, st);                            \
    }                                                                                \
  }
  if (c.dtype == EKV_BF16) {
    EKV_DEC_BF16(128, 1) EKV_DEC_BF16(128, 2) EKV_DEC_BF16(128, 4)
    EKV_DEC_BF16(128, 8) EKV_DEC_BF16(128, 16)
    EKV_DEC_BF16(64, 1) EKV_DEC_BF16(64, 2) EKV_DEC_BF16(64, 4)
    EKV_DEC_BF16(64, 8) EKV_DEC_BF16(64, 16)
  } else {
    EKV_DEC_CASE(float, 128, 1) EKV_DEC_CASE(float, 128, 2) EKV_DEC_CASE(float, 128, 4)
    EKV_DEC_CASE(float, 128, 8) EKV_DEC_CASE(float, 128, 16)
    EKV_DEC_CASE(float, 64, 1) EKV_DEC_CASE(float, 64, 2) EKV_DEC_CASE(float, 64, 4)
    EKV_DEC_CASE(float, 64, 8) EKV_DEC_CASE(float, 64, 16)
  }
#undef EKV_DEC_CASE
#undef EKV_DEC_BF16
  return cudaErrorInvalidValue;
}

}  // namespace ekv
