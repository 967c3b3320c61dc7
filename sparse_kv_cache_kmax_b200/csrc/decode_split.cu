// Sparse α-entmax decode over the selected pages in two launches — EntmaxKV
// summary page (gist.science/fr/paper/2605.21649) §2.C "Attention Entmax
// Parcimonieuse", with the support-only V read that §2–§3 make exact.
//
//  1. k_score_kernel, grid (CTAs per unit, units): every CTA scores chunks of
//     256 selected tokens (8 warps × 32 rows, straight from global memory into
//     tensor-core A fragments) for the G query heads of its unit, chunk after
//     chunk up to the unit's own selection, and writes
//     the scores z, the chunk's per-head maxima and the physical page of each
//     selected slot to an L2-resident scratch.
//  2. head_warp_kernel, one warp per query head, when the selection holds at
//     most 512 tokens (below); otherwise head_decode_kernel, one CTA of 256
//     threads per query head (1024 when streaming; a streaming CTA whose
//     unit selected at most 128 tokens runs the one-warp path): the head's
//     scores u = (α−1)·z sit in registers (VPT per thread; above 16384
//     selected tokens they are read again from L2 at each pass); a 256-bin
//     histogram of u over (max u − 1, max u] brackets τ from the left (c
//     values above an edge e force τ ≥ e − c^(−1/β): they alone would carry
//     mass ≥ 1 below it); the values above the bracket are compacted; for
//     β ∈ {1, 2} and few candidates the support is found by testing every
//     candidate at once (u_j is in the support iff
//     Σ_i (u_i − u_j)_+^β < 1) and τ is the float64 closed form on it,
//     otherwise Newton's method from the left on the ℓ_β norm of (u − τ)_+
//     (convex and decreasing; one warp alone when the candidates are few)
//     with a float64 finish.  The
//     head's support tokens are then compacted and only their V rows are
//     read, eight rows in flight per warp; warp partials are summed in warp
//     order.
// The heads of a unit read the same V rows at about the same time, so a row
// they share comes from DRAM once.  With dense V, the per-head CTAs stop
// after τ and the V pass of the three-kernel decode reads every valid row
// once for all heads of the unit (pv_kernel, decode.cu).  Every sum has a
// fixed order, so results are deterministic.
#include <algorithm>

#include "decode.cuh"

namespace ekv {

namespace {

constexpr int kKsWarps = 8;
constexpr int kKsThreads = 32 * kKsWarps;
constexpr int kKsTokens = 32 * kKsWarps;   // selected tokens per CTA of the score launch
constexpr int kHdThreads = 256;           // per-head CTA when the scores sit in registers
constexpr int kHdStreamThreads = 1024;    // per-head CTA when they are read from L2 at each pass
constexpr int kHdMaxWarps = 32;
constexpr int kHdBins = 256;
constexpr int kHdCand = 2048;              // candidates / support tokens held in shared memory at once
constexpr int kHdPairMax = 256;            // candidates for the all-at-once support test
constexpr int kHdRows = 8;                 // V rows in flight per warp
constexpr int kHdBatch = 4;                // 16-byte score loads in flight per thread when streaming
constexpr int kHdMaxVpt = 64;              // values per thread held in registers (more: read per pass)
constexpr int kSplitMaxTokens = 1 << 20;   // selected tokens per unit on this path
static_assert(kHdBins <= kHdThreads, "one histogram bin per thread");

// ------------------------------------------------------------------ 1. K scores
template <int D, int G>
__global__ void __launch_bounds__(kKsThreads, 2) k_score_kernel(DecodeArgs a) {
  constexpr int KP = D / 32, NT = (G + 7) / 8;
  __shared__ unsigned int cta_key[G];
  // wait for the previous kernel; the per-head kernel that follows is let in
  // only at the end (its CTAs hold many registers: resident early, they
  // would crowd this launch's CTAs off the SMs)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int S = a.S;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int ppc = kKsTokens / S;  // pages per chunk
  if (blockIdx.x == 0 && tid == 0) a.ws.counter[unit] = 0;  // the dense V pass's ticket
  uint32_t bfrag[2 * KP][NT][2];
  load_q_frags<D, G>(a, b, kvh, g, t, bfrag);
  const size_t zrow_len = static_cast<size_t>(a.cap) * S;
  // CTA x takes chunks x, x + gridDim.x, …: the grid is sized for the cap,
  // the loop stops at the unit's own selection
  for (int split = blockIdx.x; split * ppc < n_slots; split += gridDim.x) {
    const int s_begin = split * ppc;
    if (tid < G) cta_key[tid] = 0u;
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
    // the physical page of each selected slot, for the V pass
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
      if (lane == 0 && live[mt] && (row0 + mt * 16) % S == 0)
        a.ws.sphys[static_cast<size_t>(unit) * a.cap + slot[mt]] = phys[mt];
    __syncthreads();  // cta_key initialised
    float wmax[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) wmax[nt][0] = wmax[nt][1] = -INFINITY;
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
            float* zr = a.ws.zbuf + (static_cast<size_t>(unit) * G + hd) * zrow_len + static_cast<size_t>(slot[mt]) * S + tok0;
            zr[g] = zl;
            zr[g + 8] = zh;
          }
          wmax[nt][e] = fmaxf(wmax[nt][e], fmaxf(zl, zh));
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float m = wmax[nt][e];
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        const int hd = nt * 8 + 2 * t + e;
        if (g == 0 && hd < G && m > -INFINITY) atomicMax(&cta_key[hd], float_key(m));
      }
    __syncthreads();
    if (tid < G) {
      const unsigned int k = cta_key[tid];
      a.ws.cmax[(static_cast<size_t>(unit) * G + tid) * a.ws.nqk + split] = k == 0u ? -INFINITY : key_float(k);
    }
    __syncthreads();  // cta_key is reset by the next chunk
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ 2. τ and V per head
struct HdShared {
  int hist[kHdBins];
  float cu[kHdCand];  // candidates above the bracket, then the support's weights
  int ci[kHdCand];    // their token indices
  float f[kHdMaxWarps];
  double d[3][kHdMaxWarps];
  int i[kHdMaxWarps];
};

// Sums of (x, y, z) over the CTA in a fixed order; every thread gets them.
__device__ __forceinline__ void hd_sum3(double& x, double& y, double& z, HdShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  x = warp_sum(x);
  y = warp_sum(y);
  z = warp_sum(z);
  __syncthreads();  // the previous sums' reads are done
  if (lane == 0) {
    sh.d[0][warp] = x;
    sh.d[1][warp] = y;
    sh.d[2][warp] = z;
  }
  __syncthreads();
  x = y = z = 0.0;
  for (int w = 0; w < nw; ++w) {
    x += sh.d[0][w];
    y += sh.d[1][w];
    z += sh.d[2][w];
  }
}

__device__ __forceinline__ double hd_closed_tau(int ipow, double c, double s1, double s2) {
  if (ipow == 1) return (s1 - 1.0) / c;
  const double M = s1 / c, Q = s2 / c;
  return M - sqrt(fmax(M * M - Q + 1.0 / c, 0.0));
}

// w^(β−1) for w > 0.
template <typename V>
__device__ __forceinline__ V hd_pow_bm1(V w, V beta, int ipow) {
  switch (ipow) {
    case 1: return V(1);
    case 2: return w;
    case 3: return w * w;
    case 4: return w * w * w;
    default:
      if constexpr (sizeof(V) == 8) return pow(w, beta - 1.0);
      else return exp2f((beta - 1.0f) * __log2f(w));
  }
}

template <int D, int VPL>
__device__ __forceinline__ void warp_head(const DecodeArgs& a, int G, int row, float* s_p, int* s_i);

// A streamed head whose selection holds at most 32·kHdSmallVpl tokens (a cap
// far above the selection: the Gaussian policy's cap is a bound, its
// selections can be a few pages) is done by one warp, with no block barrier.
constexpr int kHdSmallVpl = 4;

template <int D, int VPT, int THREADS>
__global__ void __launch_bounds__(THREADS) head_decode_kernel(DecodeArgs a, int G) {
  constexpr int kHdWarps = THREADS / 32;
  constexpr int DPL = D / 32;
  __shared__ HdShared sh;
  __shared__ float red[kHdWarps][D];
  grid_dep_enter();
  const int row = blockIdx.x, unit = row / G, hg = row - unit * G, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.S;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n = unit_slots(a, unit, P) * S;
  const size_t orow = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + hg;
  const float* z = a.ws.zbuf + static_cast<size_t>(row) * a.cap * S;
  const float am1 = a.am1, beta = a.beta;
  const int ipow = a.ipow;

  // value k of this thread: held in registers (VPT > 0) as token
  // k·THREADS + tid, or read again from the scratch at every pass (VPT == 0)
  // four consecutive tokens per 16-byte load: token 4·((k/4)·THREADS + tid) +
  // k mod 4 (tok(k) gives it)
  constexpr bool kReg = VPT > 0;
  if constexpr (!kReg) {
    if (n <= 32 * kHdSmallVpl) {  // uniform over the CTA: the others leave before any barrier
      if (warp == 0) warp_head<D, kHdSmallVpl>(a, G, row, sh.cu, sh.ci);
      return;
    }
  }
  const int NK = kReg ? VPT : 4 * ((n + 4 * THREADS - 1) / (4 * THREADS));
  auto tok = [&](int k) { return kReg ? k * THREADS + tid : 4 * ((k >> 2) * THREADS + tid) + (k & 3); };
  float uv[kReg ? VPT : 1];
  if constexpr (kReg) {
#pragma unroll
    for (int k = 0; k < (kReg ? VPT : NK); ++k) {
      const int i = k * THREADS + tid;
      const float zi = z[i < n ? i : 0];  // unconditional load (see the V rows below)
      uv[k] = i < n ? am1 * zi : -INFINITY;
    }
  }
  // fn(k, u) for every value of this thread in order of k; read from the
  // scratch in batches of kHdBatch independent 16-byte loads when not in
  // registers (n is a multiple of 4, so a load starting below n stays in
  // the row; fn may hold warp collectives: k runs alike on every lane)
  auto for_values = [&](auto fn) {
    if constexpr (kReg) {
#pragma unroll
      for (int k = 0; k < VPT; ++k) fn(k, uv[k]);
    } else {
      for (int q0 = 0; q0 < NK / 4; q0 += kHdBatch) {
        float4 v[kHdBatch];
#pragma unroll
        for (int j = 0; j < kHdBatch; ++j) {
          const int i = 4 * ((q0 + j) * THREADS + tid);
          const bool in = q0 + j < NK / 4 && i < n;
          const float4 x = __ldcg(reinterpret_cast<const float4*>(z + (in ? i : 0)));  // n ≥ 4 here
          v[j] = in ? x : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
#pragma unroll
        for (int j = 0; j < kHdBatch; ++j)
          if (q0 + j < NK / 4) {
            const int k = 4 * (q0 + j);
            fn(k, am1 * v[j].x);
            fn(k + 1, am1 * v[j].y);
            fn(k + 2, am1 * v[j].z);
            fn(k + 3, am1 * v[j].w);
          }
      }
    }
  };
  // the head's maximum from the chunk maxima
  const int nchunk = (n + kKsTokens - 1) / kKsTokens;
  float m = -INFINITY;
  for (int c = lane; c < nchunk; c += 32) m = fmaxf(m, a.ws.cmax[static_cast<size_t>(row) * a.ws.nqk + c]);
  m = warp_max(m);  // every warp reads them all: no barrier
  if (tid < kHdBins) sh.hist[tid] = 0;
  __syncthreads();

  float tau = INFINITY;  // no finite score: no support, zero output
  int n_listed = -1;     // candidates listed in shared memory (−1: too many)
  if (m > -INFINITY) {
    const float um = am1 * m;
    // 1. bracket from the histogram of u over (um − 1, um], bin 0 at the top
    for_values([&](int, float u) {
      if (u > um - 1.0f) atomicAdd(&sh.hist[min(kHdBins - 1, static_cast<int>((um - u) * kHdBins))], 1);
    });
    __syncthreads();
    float cb = um - 1.0f;
    {
      const int h = tid < kHdBins ? sh.hist[tid] : 0;
      int total;
      const int c = block_exclusive_scan(h, sh.i, &total) + h;  // values in bins 0..tid
      if (tid < kHdBins && c > 0) {
        const float fc = static_cast<float>(c);
        const float inv = ipow == 1 ? 1.0f / fc : (ipow == 2 ? rsqrtf(fc) : exp2f(-__log2f(fc) / beta));
        cb = fmaxf(cb, um - static_cast<float>(tid + 1) / kHdBins - inv);
      }
    }
    cb = warp_max(cb);
    if (lane == 0) sh.f[warp] = cb;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kHdWarps; ++w) cb = fmaxf(cb, sh.f[w]);
    // slack for the fp32 rounding of the bound: τ_lo stays below τ
    const double tau_lo = static_cast<double>(cb) - 4e-6 * (1.0 + fabs(static_cast<double>(um)));
    float tlo = static_cast<float>(tau_lo);
    if (static_cast<double>(tlo) > tau_lo) tlo = nextafterf(tlo, -INFINITY);

    // 2. compaction of the values above τ_lo: thread after thread (a fixed
    //    order, so every later sum is deterministic), one block scan
    int nc;
    {
      int mine = 0;
      for_values([&](int, float u) { mine += u > tlo ? 1 : 0; });
      int p = block_exclusive_scan(mine, sh.i, &nc);
      if (nc <= kHdCand)
        for_values([&](int k, float u) {
          if (u > tlo) {
            sh.cu[p] = u;
            sh.ci[p] = tok(k);
            ++p;
          }
        });
      __syncthreads();
    }
    const bool listed = nc <= kHdCand;
    if (listed) n_listed = nc;

    // 3. τ
    const bool closed = ipow == 1 || ipow == 2;
    double tt;
    if (closed && nc <= kHdPairMax) {
      // u_j is in the support iff Σ_i (u_i − u_j)_+^β < 1 (f decreases and f(τ) = 1)
      double c = 0.0, s1 = 0.0, s2 = 0.0;
      if (tid < nc) {
        const float uj = sh.cu[tid];
        float fs = 0.f;
        for (int i = 0; i < nc; ++i) {
          const float w = sh.cu[i] - uj;
          if (w > 0.f) fs = fmaf(ipow == 1 ? 1.0f : w, w, fs);
        }
        if (fs < 1.0f) {
          c = 1.0;
          s1 = uj;
          s2 = static_cast<double>(uj) * uj;
        }
      }
      hd_sum3(c, s1, s2, sh);
      tt = hd_closed_tau(ipow, c, s1, s2);
      // the closed form must imply the support it was built on; if rounding
      // at the edge says otherwise, repeat it on {u > τ} until it is stable
      for (int rep = 0; rep < 8; ++rep) {
        double c2 = 0.0, t1 = 0.0, t2 = 0.0;
        if (tid < nc) {
          const double u = sh.cu[tid];
          if (u > tt) {
            c2 = 1.0;
            t1 = u;
            t2 = u * u;
          }
        }
        hd_sum3(c2, t1, t2, sh);
        if (c2 == c || c2 < 1.0) break;
        c = c2;
        const double t_new = hd_closed_tau(ipow, c2, t1, t2);
        if (t_new == tt) break;
        tt = t_new;
      }
    } else {
      // Newton from the left in fp32 over the candidates (or every value),
      // then a float64 finish
      auto sums = [&](auto t, auto& f, auto& df) {
        using V = decltype(t);
        V x = V(0), y = V(0);
        auto term = [&](float u) {
          const V w = static_cast<V>(u) - t;
          if (w > V(0)) {
            const V wb1 = hd_pow_bm1<V>(w, static_cast<V>(beta), ipow);
            x += wb1 * w;
            y += wb1;
          }
        };
        if (listed) {
          for (int j = tid; j < nc; j += THREADS) term(sh.cu[j]);
        } else {
          for_values([&](int, float u) { term(u); });
        }
        double dx = x, dy = y, dz = 0.0;
        hd_sum3(dx, dy, dz, sh);
        f = static_cast<V>(dx - 1.0);
        df = static_cast<V>(dy);
      };
      // one warp alone over a short candidate list (no barriers per step)
      auto warp_sums = [&](auto t, auto& f, auto& df) {
        using V = decltype(t);
        V x = V(0), y = V(0);
        for (int j = lane; j < nc; j += 32) {
          const V w = static_cast<V>(sh.cu[j]) - t;
          if (w > V(0)) {
            const V wb1 = hd_pow_bm1<V>(w, static_cast<V>(beta), ipow);
            x += wb1 * w;
            y += wb1;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          x += __shfl_xor_sync(0xffffffffu, x, o);
          y += __shfl_xor_sync(0xffffffffu, y, o);
        }
        f = x - V(1);
        df = y;
      };
      const bool solo = listed && nc <= 128;  // one warp alone only when the candidates are few
      if (solo) {
        if (warp == 0) {
          float t = tlo;
          for (int it = 0; it < 100; ++it) {
            float f, df;
            warp_sums(t, f, df);
            if (it == 0 && f < 0.0f) {
              t = um - 1.0f;
              continue;
            }
            const float step = norm_newton_step<float>(f, df, beta);
            if (!(step > 0.0f)) break;
            t += step;
            if (step <= 2e-7f * fmaxf(1.0f, fabsf(t))) break;
          }
          double d = t;
          if (closed) {
            for (int rep = 0; rep < 4; ++rep) {
              double c3 = 0.0, t1 = 0.0, t2 = 0.0;
              for (int j = lane; j < nc; j += 32) {
                const double u = sh.cu[j];
                if (u > d) {
                  c3 += 1.0;
                  t1 += u;
                  t2 += u * u;
                }
              }
              c3 = warp_sum(c3);
              t1 = warp_sum(t1);
              t2 = warp_sum(t2);
              if (c3 < 1.0) break;
              const double t_new = hd_closed_tau(ipow, c3, t1, t2);
              if (t_new == d) break;
              d = t_new;
            }
          } else {
            double f, df;
            warp_sums(d, f, df);
            if (df > 0.0) d += f / (static_cast<double>(beta) * df);
          }
          if (lane == 0) sh.d[0][0] = d;
        }
        __syncthreads();
        tt = sh.d[0][0];
      } else {
      float t = tlo;
      for (int it = 0; it < 64; ++it) {
        float f, df;
        sums(t, f, df);
        if (it == 0 && f < 0.0f) {  // bracket missed by rounding: restart from max u − 1
          t = um - 1.0f;
          continue;
        }
        const float step = norm_newton_step<float>(f, df, beta);
        if (!(step > 0.0f)) break;
        t += step;
        if (step <= 2e-7f * fmaxf(1.0f, fabsf(t))) break;
      }
      tt = t;
      if (closed) {
        for (int rep = 0; rep < 4; ++rep) {
          double c3 = 0.0, t1 = 0.0, t2 = 0.0;
          auto add = [&](float uf) {
            const double u = uf;
            if (u > tt) {
              c3 += 1.0;
              t1 += u;
              t2 += u * u;
            }
          };
          if (listed) {
            for (int j = tid; j < nc; j += THREADS) add(sh.cu[j]);
          } else {
            for_values([&](int, float u) { add(u); });
          }
          hd_sum3(c3, t1, t2, sh);
          if (c3 < 1.0) break;
          const double t_new = hd_closed_tau(ipow, c3, t1, t2);
          if (t_new == tt) break;
          tt = t_new;
        }
      } else {
        double f, df;
        sums(tt, f, df);
        if (df > 0.0) tt += f / (static_cast<double>(beta) * df);
      }
      }
    }
    tau = static_cast<float>(tt);
  }
  __syncthreads();  // the candidate area is reused for the support list

  // 4. support with the fp32 τ every later step uses, listed at places
  //    base .. base + kHdCand − 1 (thread after thread) with the weights
  //    p = (u − τ)^β.  The support lies inside the candidates (u > τ ≥ τ_lo):
  //    when they are listed, the support is cut from their list (same order)
  //    and its bits are set one token at a time; otherwise compact(base)
  //    passes over every value and the bits come from ballots.
  auto compact = [&](int base) {
    int mine = 0;
    for_values([&](int k, float u) { mine += (tok(k) < n && u > tau) ? 1 : 0; });
    int ns;
    int p = block_exclusive_scan(mine, sh.i, &ns) - base;
    for_values([&](int k, float u) {
      const int i = tok(k);
      if (i < n && u > tau) {
        if (p >= 0 && p < kHdCand) {
          sh.cu[p] = pow_beta_fast(u - tau, beta, ipow);
          sh.ci[p] = i;
        }
        ++p;
      }
    });
    __syncthreads();
    return ns;
  };
  int ns;
  if (n_listed >= 0) {
    constexpr int kPer = (kHdCand + THREADS - 1) / THREADS;
    float cu_r[kPer];
    int ci_r[kPer];
    int mine = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int j = tid * kPer + q;
      cu_r[q] = -INFINITY;
      ci_r[q] = 0;
      if (j < n_listed) {
        cu_r[q] = sh.cu[j];
        ci_r[q] = sh.ci[j];
        mine += cu_r[q] > tau ? 1 : 0;
      }
    }
    int p = block_exclusive_scan(mine, sh.i, &ns);  // every candidate is read before it returns
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (cu_r[q] > tau) {
        sh.cu[p] = pow_beta_fast(cu_r[q] - tau, beta, ipow);
        sh.ci[p] = ci_r[q];
        ++p;
      }
    if (a.bits_out)
      for (int w = tid; w < a.words; w += THREADS) a.bits_out[orow * a.words + w] = 0u;
    __syncthreads();
    if (a.bits_out)
      for (int e = tid; e < ns; e += THREADS) {
        const int i = sh.ci[e];
        atomicOr(&a.bits_out[orow * a.words + (i >> 5)], 1u << (i & 31));
      }
  } else if (kReg) {
    if (a.bits_out)
      for_values([&](int k, float u) {
        const int i = k * THREADS + tid;
        const unsigned int bal = __ballot_sync(0xffffffffu, i < n && u > tau);
        if (lane == 0 && (i >> 5) < a.words) a.bits_out[orow * a.words + (i >> 5)] = bal;
      });
    ns = compact(0);
    if (a.bits_out)
      for (int w = (VPT * THREADS) / 32 + tid; w < a.words; w += THREADS)
        a.bits_out[orow * a.words + w] = 0u;  // words past the ballots above
  } else {
    // streamed values: a warp's lanes hold tokens four apart, so the bits
    // are set one token at a time after the row is cleared
    if (a.bits_out) {
      for (int w = tid; w < a.words; w += THREADS) a.bits_out[orow * a.words + w] = 0u;
      __syncthreads();
      for_values([&](int k, float u) {
        const int i = tok(k);
        if (i < n && u > tau) atomicOr(&a.bits_out[orow * a.words + (i >> 5)], 1u << (i & 31));
      });
    }
    ns = compact(0);
  }
  if (tid == 0) {
    if (a.tau_out) a.tau_out[orow] = tau;
    if (a.count_out) a.count_out[orow] = ns;
    if (a.dense_v) a.ws.taus[row] = tau;
  }
  if (a.dense_v) return;  // every V row is read by the V pass that follows

  // 5. V of the support rows: warp w takes rows w·8 … w·8+7 of each block of 64
  float acc[DPL];
#pragma unroll
  for (int x = 0; x < DPL; ++x) acc[x] = 0.f;
  for (int base = 0; base < ns; base += kHdCand) {
    if (base > 0) compact(base);
    const int nl = min(ns - base, kHdCand);
    for (int e0 = warp * kHdRows; e0 < nl; e0 += kHdWarps * kHdRows) {
      float v[kHdRows][DPL];
      float p[kHdRows];
#pragma unroll
      for (int r = 0; r < kHdRows; ++r) {
        const int e = e0 + r;
        // unconditional load (a row past the list reads entry e0, which
        // exists; an invalid page reads page 0) zeroed after: loads behind
        // per-row branches are issued one after another
        const bool in_list = e < nl;
        const int tok = sh.ci[in_list ? e : e0];
        const int ph = a.ws.sphys[static_cast<size_t>(unit) * a.cap + tok / S];
        const bool in = in_list && ph >= 0;
        p[r] = in ? sh.cu[in_list ? e : e0] : 0.f;
        const bf16* src = static_cast<const bf16*>(a.v_pool) +
                          ((static_cast<size_t>(ph >= 0 ? ph : 0) * a.Hkv + kvh) * S + (tok % S)) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const uint2 w2 = *reinterpret_cast<const uint2*>(src);
          v[r][0] = in ? __uint_as_float(w2.x << 16) : 0.f;
          v[r][1] = in ? __uint_as_float(w2.x & 0xffff0000u) : 0.f;
          v[r][2] = in ? __uint_as_float(w2.y << 16) : 0.f;
          v[r][3] = in ? __uint_as_float(w2.y & 0xffff0000u) : 0.f;
        } else {
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(src);
          v[r][0] = in ? __uint_as_float(w1 << 16) : 0.f;
          v[r][1] = in ? __uint_as_float(w1 & 0xffff0000u) : 0.f;
        }
      }
#pragma unroll
      for (int r = 0; r < kHdRows; ++r)
#pragma unroll
        for (int x = 0; x < DPL; ++x) acc[x] = fmaf(p[r], v[r][x], acc[x]);
    }
    __syncthreads();  // the list is rewritten for the next kHdCand support tokens
  }
#pragma unroll
  for (int x = 0; x < DPL; ++x) red[warp][lane * DPL + x] = acc[x];
  __syncthreads();
  for (int i = tid; i < D; i += THREADS) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kHdWarps; ++w) s += red[w][i];
    a.out[orow * D + i] = s;
  }
}

// ------------------------------------------------------------------ 2'. one warp per head
// For selections of at most 32·VPL tokens a whole query head fits one warp
// (VPL values per lane, token k·32 + lane), and the head needs no block
// barrier at all: Newton's method on the ℓ_β norm over every value from
// max u − 1 (where the sum is ≥ 1), the float64 closed form on the support
// for β ∈ {1, 2} (one float64 Newton step otherwise), the support's bits by
// ballots, its tokens and weights listed in token order in the warp's
// shared memory, then its V rows, eight in flight, each lane summing its own
// output columns.
template <int VPL>
constexpr int head_warps() {
  return 8;
}

// Query head `row` by the calling warp alone; s_p, s_i: 32·VPL entries of
// shared memory that only this warp uses.
template <int D, int VPL>
__device__ __forceinline__ void warp_head(const DecodeArgs& a, int G, int row, float* s_p, int* s_i) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int unit = row / G, hg = row - unit * G, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int S = a.S;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n = unit_slots(a, unit, P) * S;
  const size_t orow = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + hg;
  const float* z = a.ws.zbuf + static_cast<size_t>(row) * a.cap * S;
  const float am1 = a.am1, beta = a.beta;
  const int ipow = a.ipow;
  float u[VPL];
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int i = k * 32 + lane;
    const float zi = __ldcg(z + (i < n ? i : 0));  // unconditional load, dropped past n
    u[k] = i < n ? am1 * zi : -INFINITY;
    m = fmaxf(m, u[k]);
  }
  m = warp_max(m);

  float tau = INFINITY;  // no finite score: no support, zero output
  if (m > -INFINITY) {
    float t = m - 1.0f;
    for (int it = 0; it < 100; ++it) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const float w = u[k] - t;
        if (w > 0.f) {
          const float wb1 = hd_pow_bm1<float>(w, beta, ipow);
          x += wb1 * w;
          y += wb1;
        }
      }
      x = warp_sum(x);
      y = warp_sum(y);
      const float step = norm_newton_step<float>(x - 1.0f, y, beta);
      if (!(step > 0.0f)) break;
      t += step;
      if (step <= 2e-7f * fmaxf(1.0f, fabsf(t))) break;
    }
    double d = t;
    if (ipow == 1 || ipow == 2) {
      // the closed form on {u > τ}, repeated while the support it implies moves
      for (int rep = 0; rep < 4; ++rep) {
        double c = 0.0, s1 = 0.0, s2 = 0.0;
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
          const double uu = u[k];
          if (uu > d) {
            c += 1.0;
            s1 += uu;
            s2 += uu * uu;
          }
        }
        c = warp_sum(c);
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (c < 1.0) break;
        const double t_new = hd_closed_tau(ipow, c, s1, s2);
        if (t_new == d) break;
        d = t_new;
      }
    } else {
      double x = 0.0, y = 0.0;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const double w = static_cast<double>(u[k]) - d;
        if (w > 0.0) {
          const double wb1 = hd_pow_bm1<double>(w, static_cast<double>(beta), ipow);
          x += wb1 * w;
          y += wb1;
        }
      }
      x = warp_sum(x);
      y = warp_sum(y);
      if (y > 0.0) d += (x - 1.0) / (static_cast<double>(beta) * y);
    }
    tau = static_cast<float>(d);
  }

  // support: bits by ballots (word k holds tokens k·32 …), list in token order
  int ns = 0;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int i = k * 32 + lane;
    const bool in = i < n && u[k] > tau;
    const unsigned int bal = __ballot_sync(0xffffffffu, in);
    if (a.bits_out && lane == 0 && k < a.words) a.bits_out[orow * a.words + k] = bal;
    if (in) {
      const int at = ns + __popc(bal & ((1u << lane) - 1u));
      s_p[at] = pow_beta_fast(u[k] - tau, beta, ipow);
      s_i[at] = i;
    }
    ns += __popc(bal);
  }
  if (a.bits_out)
    for (int w = VPL + lane; w < a.words; w += 32) a.bits_out[orow * a.words + w] = 0u;
  if (lane == 0) {
    if (a.tau_out) a.tau_out[orow] = tau;
    if (a.count_out) a.count_out[orow] = ns;
    if (a.dense_v) a.ws.taus[row] = tau;
  }
  if (a.dense_v) return;  // every V row is read by the V pass that follows
  __syncwarp();

  float acc[DPL];
#pragma unroll
  for (int x = 0; x < DPL; ++x) acc[x] = 0.f;
  for (int e0 = 0; e0 < ns; e0 += kHdRows) {
    float v[kHdRows][DPL];
    float p[kHdRows];
#pragma unroll
    for (int r = 0; r < kHdRows; ++r) {
      const int e = e0 + r;
      // unconditional load (a row past the list reads entry e0, which
      // exists; an invalid page reads page 0) zeroed after: loads behind
      // per-row branches are issued one after another
      const bool in_list = e < ns;
      const int tok = s_i[in_list ? e : e0];
      const int ph = a.ws.sphys[static_cast<size_t>(unit) * a.cap + tok / S];
      const bool in = in_list && ph >= 0;
      p[r] = in ? s_p[in_list ? e : e0] : 0.f;
      const bf16* src = static_cast<const bf16*>(a.v_pool) +
                        ((static_cast<size_t>(ph >= 0 ? ph : 0) * a.Hkv + kvh) * S + (tok % S)) * D + lane * DPL;
      if constexpr (DPL == 4) {
        const uint2 w2 = *reinterpret_cast<const uint2*>(src);
        v[r][0] = in ? __uint_as_float(w2.x << 16) : 0.f;
        v[r][1] = in ? __uint_as_float(w2.x & 0xffff0000u) : 0.f;
        v[r][2] = in ? __uint_as_float(w2.y << 16) : 0.f;
        v[r][3] = in ? __uint_as_float(w2.y & 0xffff0000u) : 0.f;
      } else {
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(src);
        v[r][0] = in ? __uint_as_float(w1 << 16) : 0.f;
        v[r][1] = in ? __uint_as_float(w1 & 0xffff0000u) : 0.f;
      }
    }
#pragma unroll
    for (int r = 0; r < kHdRows; ++r)
#pragma unroll
      for (int x = 0; x < DPL; ++x) acc[x] = fmaf(p[r], v[r][x], acc[x]);
  }
#pragma unroll
  for (int x = 0; x < DPL; ++x) a.out[orow * D + lane * DPL + x] = acc[x];
}

template <int D, int VPL>
__global__ void __launch_bounds__(32 * head_warps<VPL>()) head_warp_kernel(DecodeArgs a, int G, int rows) {
  constexpr int kWarps = head_warps<VPL>();
  __shared__ float s_p[kWarps][32 * VPL];
  __shared__ int s_i[kWarps][32 * VPL];
  grid_dep_enter();
  const int warp = threadIdx.x >> 5;
  const int row = blockIdx.x * kWarps + warp;
  if (row >= rows) return;  // warp-uniform, and no block barrier follows
  warp_head<D, VPL>(a, G, row, s_p[warp], s_i[warp]);
}

template <int D>
cudaError_t launch_head_decode(DecodeArgs& a, int rows, int G, cudaStream_t st) {
  const int n_max = a.cap * a.S;
#define EKV_HW_CASE(VV)                                                                                    \
  if (n_max <= 32 * (VV)) {                                                                                \
    constexpr int W = head_warps<VV>();                                                                    \
    const cudaError_t e =                                                                                  \
        launch_k(head_warp_kernel<D, VV>, dim3((rows + W - 1) / W), dim3(32 * W), 0, st, a, G, rows);      \
    if (e != cudaSuccess) return e;                                                                        \
    return cudaGetLastError();                                                                             \
  }
  EKV_HW_CASE(4) EKV_HW_CASE(8) EKV_HW_CASE(16)
#undef EKV_HW_CASE
#define EKV_HD_CASE(VV)                                                                                      \
  if (n_max <= (VV) * kHdThreads) {                                                                          \
    const cudaError_t e = launch_k(head_decode_kernel<D, VV, kHdThreads>, dim3(rows), dim3(kHdThreads), 0, st, a, G); \
    if (e != cudaSuccess) return e;                                                                          \
    return cudaGetLastError();                                                                               \
  }
  EKV_HD_CASE(4) EKV_HD_CASE(16) EKV_HD_CASE(32) EKV_HD_CASE(kHdMaxVpt)
#undef EKV_HD_CASE
  const cudaError_t e = launch_k(head_decode_kernel<D, 0, kHdStreamThreads>, dim3(rows), dim3(kHdStreamThreads), 0,
                                 st, a, G);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

template <int D, int G>
bool split_decode_fits(int cap, int S) {
  return S % 16 == 0 && cap >= 1 && static_cast<long long>(cap) * S <= kSplitMaxTokens;
}

template <int D, int G>
cudaError_t run_split_decode(DecodeArgs& a, int units, cudaStream_t st) {
  // about eight CTAs per SM of a B200 in all; each loops over its chunks
  const int per_unit = std::max(1, std::min(a.ws.nqk, (8 * 148) / std::max(1, units)));
  const dim3 grid(static_cast<unsigned>(per_unit), static_cast<unsigned>(units));
  cudaError_t e = launch_k(k_score_kernel<D, G>, grid, dim3(kKsThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_head_decode<D>(a, units * G, G, st);
  if (e != cudaSuccess || !a.dense_v) return e;
  return run_dense_v_pass<D, G>(a, units, st);
}

#define EKV_SPLIT_INST(DD, GG)                               \
  template bool split_decode_fits<DD, GG>(int, int);         \
  template cudaError_t run_split_decode<DD, GG>(DecodeArgs&, int, cudaStream_t);
EKV_SPLIT_INST(128, 1)
EKV_SPLIT_INST(128, 2)
EKV_SPLIT_INST(128, 4)
EKV_SPLIT_INST(128, 8)
EKV_SPLIT_INST(128, 16)
EKV_SPLIT_INST(64, 1)
EKV_SPLIT_INST(64, 2)
EKV_SPLIT_INST(64, 4)
EKV_SPLIT_INST(64, 8)
EKV_SPLIT_INST(64, 16)
#undef EKV_SPLIT_INST

}  // namespace ekv
