// Softmax decode over the paged cache, split over pages — the full-cache
// baseline that the EntmaxKV summary page (gist.science/fr/paper/2605.21649)
// §4 measures the sparse α-entmax decode against ("the full cache read
// dominates").  o_h = Σ_i e^{z_i − m} v_i / Σ_i e^{z_i − m} with
// z_i = scale·q_h·k_i, over every valid token of the selected pages (every
// page of the sequence when sel is NULL).
//
// Grid (nsplit, units): CTA s of unit u takes an equal run of the unit's page
// slots; its page ids are resolved once into shared memory.  Each of its 4
// warps streams its pages (every 4th) through a private ring of 3 slots that
// hold the page's K and V tiles (two 1-D bulk copies on one mbarrier),
// scores the page on tensor cores (m16n8k16, rows loaded from shared memory
// into A fragments, the group's queries as B), and folds it into a running
// maximum, sum and p·v per query head (the online softmax, in base 2), lane
// l owning columns DPL·l .. DPL·l + DPL − 1 of every head.  The warps, then
// the splits, are merged in fixed order — the splits by the unit's last CTA
// (an atomic ticket) — so results are deterministic.
#include "decode.cuh"

namespace ekv {

namespace {

constexpr int kSmWarps = 4;
constexpr int kSmThreads = 32 * kSmWarps;
constexpr int kSmStages = 3;
constexpr int kSmTargetCtas = 8 * 296;  // about eight waves of two CTAs per SM

struct SoftmaxArgs {
  const void* k_pool;
  const void* v_pool;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const void* q;
  const int32_t* sel;
  const int32_t* n_sel;
  float* out;
  float* lse;
  float* part;   // [U, nsplit, G, D] partial p·v of each split
  float* ml;     // [U, nsplit, G, 2] its (max, sum) in base 2
  int* counter;  // [U] finished splits (zeroed before the launch)
  float scale_log2;  // scale · log2(e)
  int Hkv, Hq, S, num_phys, max_pages, cap, nsplit, spp;
};

template <int D, int G>
__global__ void __launch_bounds__(kSmThreads, 2) softmax_split_kernel(SoftmaxArgs a) {
  constexpr int KP = D / 32, NT = (G + 7) / 8, DPL = D / 32, GP = (G + 3) / 4 * 4;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t bars[kSmWarps * kSmStages];
  __shared__ float s_corr[kSmWarps][GP];
  __shared__ float s_ml[kSmWarps][G][2];
  __shared__ int s_last;

  const int split = blockIdx.x, unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const int S = a.S;
  const int tile = S * D * 2;                  // bytes of one K or V tile
  unsigned char* ring = smem;                  // [warps][stages][K tile | V tile]
  float* zw = reinterpret_cast<float*>(smem + static_cast<size_t>(kSmWarps) * kSmStages * 2 * tile);  // [warps][S][GP]
  int* phys_s = reinterpret_cast<int*>(zw + kSmWarps * S * GP);  // [spp]
  int* nv_s = phys_s + a.spp;                                    // [spp]

  if (tid < kSmWarps * kSmStages) {
    mbar_init(&bars[tid], 1);
    fence_mbar_init();
  }
  grid_dep_enter();
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int s0 = split * a.spp, npg = max(0, min(a.spp, n_slots - s0));
  for (int j = tid; j < npg; j += kSmThreads) {
    int nv;
    phys_s[j] = slot_page(a, unit, b, s0 + j, P, L, &nv);
    nv_s[j] = nv;
  }
  __syncthreads();

  const int cnt_w = warp < npg ? (npg - warp + kSmWarps - 1) / kSmWarps : 0;
  const size_t tile_elems = static_cast<size_t>(S) * D;
  unsigned char* wring = ring + static_cast<size_t>(warp) * kSmStages * 2 * tile;
  uint64_t* wbar = bars + warp * kSmStages;
  auto issue = [&](int i) {  // lane 0: page i of this warp into slot i mod stages
    const int j = warp + i * kSmWarps, sl = i % kSmStages, ph = phys_s[j];
    if (ph < 0) {
      mbar_arrive(&wbar[sl]);
      return;
    }
    const size_t off = (static_cast<size_t>(ph) * a.Hkv + kvh) * tile_elems;
    mbar_arrive_expect_tx(&wbar[sl], static_cast<unsigned int>(2 * tile));
    bulk_g2s(wring + static_cast<size_t>(sl) * 2 * tile, static_cast<const bf16*>(a.k_pool) + off,
             static_cast<unsigned int>(tile), &wbar[sl]);
    bulk_g2s(wring + static_cast<size_t>(sl) * 2 * tile + tile, static_cast<const bf16*>(a.v_pool) + off,
             static_cast<unsigned int>(tile), &wbar[sl]);
  };
  if (lane == 0)
    for (int i = 0; i < min(kSmStages, cnt_w); ++i) issue(i);
  uint32_t bfrag[2 * KP][NT][2];
  load_q_frags<D, G>(a, b, kvh, g, t, bfrag);

  float* wz = zw + warp * S * GP;
  float m_own = -INFINITY, l_own = 0.f;  // head `lane` (lanes < G): running max and sum
  float acc[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;

  for (int i = 0; i < cnt_w; ++i) {
    const int j = warp + i * kSmWarps, sl = i % kSmStages;
    const unsigned int parity = static_cast<unsigned int>(i / kSmStages) & 1u;
    if (!mbar_wait(&wbar[sl], parity)) mbar_wait(&wbar[sl], parity);
    const unsigned char* kt = wring + static_cast<size_t>(sl) * 2 * tile;
    const unsigned char* vt = kt + tile;
    const int nv = phys_s[j] < 0 ? 0 : nv_s[j];
    // scores of the page's tokens, base 2, into the warp's scratch
    for (int mt = 0; mt < S / 16; ++mt) {
      const int tok0 = mt * 16;
      const uint4* rlo = reinterpret_cast<const uint4*>(kt + static_cast<size_t>(tok0 + g) * D * 2) + t;
      const uint4* rhi = reinterpret_cast<const uint4*>(kt + static_cast<size_t>(tok0 + g + 8) * D * 2) + t;
      uint4 va[KP], vb[KP];
#pragma unroll
      for (int c = 0; c < KP; ++c) {
        va[c] = rlo[4 * c];
        vb[c] = rhi[4 * c];
      }
      float sc[NT][4];
      score_mtile<D, G>(va, vb, bfrag, sc);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hd = nt * 8 + 2 * t + e;
          if (hd < G) {
            wz[(tok0 + g) * GP + hd] = tok0 + g < nv ? a.scale_log2 * sc[nt][e] : -INFINITY;
            wz[(tok0 + g + 8) * GP + hd] = tok0 + g + 8 < nv ? a.scale_log2 * sc[nt][2 + e] : -INFINITY;
          }
        }
    }
    __syncwarp();
    // lane h < G: rescale head h's state to the new maximum and turn the
    // page's scores into weights 2^(z − m)
    if (lane < G) {
      float pm = -INFINITY;
      for (int r = 0; r < S; ++r) pm = fmaxf(pm, wz[r * GP + lane]);
      const float mn = fmaxf(m_own, pm);
      float corr = 1.f, psum = 0.f;
      if (mn > -INFINITY) {
        corr = exp2f(m_own - mn);  // 0 while m_own is −inf
        for (int r = 0; r < S; ++r) {
          const float w = exp2f(wz[r * GP + lane] - mn);
          wz[r * GP + lane] = w;
          psum += w;
        }
        m_own = mn;
      }
      l_own = l_own * corr + psum;
      s_corr[warp][lane] = corr;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float c = s_corr[warp][h];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[h][e] *= c;
    }
    const unsigned char* vrow = vt + lane * DPL * 2;
#pragma unroll 4
    for (int r = 0; r < nv; ++r) {
      float v[DPL];
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vrow + static_cast<size_t>(r) * D * 2);
        v[0] = __uint_as_float(w.x << 16);
        v[1] = __uint_as_float(w.x & 0xffff0000u);
        v[2] = __uint_as_float(w.y << 16);
        v[3] = __uint_as_float(w.y & 0xffff0000u);
      } else {
        const uint32_t w = *reinterpret_cast<const unsigned int*>(vrow + static_cast<size_t>(r) * D * 2);
        v[0] = __uint_as_float(w << 16);
        v[1] = __uint_as_float(w & 0xffff0000u);
      }
      const float4* pr = reinterpret_cast<const float4*>(wz + r * GP);
#pragma unroll
      for (int h4 = 0; h4 < GP / 4; ++h4) {
        const float4 pp = pr[h4];
        const float ph[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          if (h4 * 4 + k4 < G) {
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h4 * 4 + k4][e] = fmaf(ph[k4], v[e], acc[h4 * 4 + k4][e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0 && i + kSmStages < cnt_w) {
      fence_proxy_async_shared();  // the slot's reads come before the copies that refill it
      issue(i + kSmStages);
    }
  }

  // warps → CTA partial (warp order), over the ring (all copies consumed)
  if (lane < G) {
    s_ml[warp][lane][0] = m_own;
    s_ml[warp][lane][1] = l_own;
  }
  __syncthreads();
  float* red = reinterpret_cast<float*>(ring);  // [warps][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) red[(warp * G + h) * D + lane * DPL + e] = acc[h][e];
  __syncthreads();
  const size_t pbase = (static_cast<size_t>(unit) * a.nsplit + split) * G;
  for (int i = tid; i < G * D; i += kSmThreads) {
    const int h = i / D;
    float mc = -INFINITY;
#pragma unroll
    for (int w = 0; w < kSmWarps; ++w) mc = fmaxf(mc, s_ml[w][h][0]);
    float val = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kSmWarps; ++w) {
      const float f = mc > -INFINITY ? exp2f(s_ml[w][h][0] - mc) : 0.f;
      val += red[(w * G + h) * D + (i - h * D)] * f;
      lsum += s_ml[w][h][1] * f;
    }
    a.part[pbase * D + i] = val;
    if (i - h * D == 0) {
      a.ml[(pbase + h) * 2] = mc;
      a.ml[(pbase + h) * 2 + 1] = lsum;
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(&a.counter[unit], 1) == a.nsplit - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // the unit's last CTA merges the splits in split order
  const size_t ubase = static_cast<size_t>(unit) * a.nsplit * G;
  for (int i = tid; i < G * D; i += kSmThreads) {
    const int h = i / D, dcol = i - h * D;
    float M = -INFINITY;
    for (int sp = 0; sp < a.nsplit; ++sp) M = fmaxf(M, __ldcg(a.ml + (ubase + static_cast<size_t>(sp) * G + h) * 2));
    float num = 0.f, den = 0.f;
    if (M > -INFINITY) {
      for (int sp = 0; sp < a.nsplit; ++sp) {
        const size_t o = ubase + static_cast<size_t>(sp) * G + h;
        const float f = exp2f(__ldcg(a.ml + o * 2) - M);
        num += __ldcg(a.part + o * D + dcol) * f;
        den += __ldcg(a.ml + o * 2 + 1) * f;
      }
    }
    const size_t orow = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + h;
    a.out[orow * D + dcol] = den > 0.f ? num / den : 0.f;
    if (dcol == 0 && a.lse) a.lse[orow] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
  }
  if (tid == 0) a.counter[unit] = 0;
}

}  // namespace

int softmax_splits(int units, int cap) {
  int ns = (kSmTargetCtas + units / 2) / units;
  const int max_ns = (cap + 7) / 8;      // at least 8 pages per split
  const int min_ns = (cap + 4095) / 4096;  // at most 4096 pages (their ids live in shared memory)
  if (ns > max_ns) ns = max_ns;
  if (ns < min_ns) ns = min_ns;
  if (ns < 1) ns = 1;
  const int spp = (cap + ns - 1) / ns;
  return (cap + spp - 1) / spp;
}

size_t softmax_ws_bytes(int units, int Hq, int Hkv, int d, int cap) {
  const size_t G = static_cast<size_t>(Hq / Hkv), ns = static_cast<size_t>(softmax_splits(units, cap));
  const size_t part = static_cast<size_t>(units) * ns * G * d * sizeof(float);
  const size_t ml = static_cast<size_t>(units) * ns * G * 2 * sizeof(float);
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return al(part) + al(ml) + al(static_cast<size_t>(units) * sizeof(int));
}

cudaError_t launch_softmax_decode(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                                  float scale, const int32_t* sel, const int32_t* n_sel, int cap,
                                  float* out, float* lse, void* ws, cudaStream_t st) {
  const int Hkv = c.num_kv_heads, G = Hq / Hkv, U = s.batch * Hkv, D = c.head_dim;
  SoftmaxArgs a{};
  a.k_pool = c.k_pool;
  a.v_pool = c.v_pool;
  a.page_table = s.page_table;
  a.seq_lens = s.seq_lens;
  a.q = q;
  a.sel = sel;
  a.n_sel = n_sel;
  a.out = out;
  a.lse = lse;
  a.nsplit = softmax_splits(U, cap);
  a.spp = (cap + a.nsplit - 1) / a.nsplit;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  char* p = static_cast<char*>(ws);
  a.part = reinterpret_cast<float*>(p);
  p += al(static_cast<size_t>(U) * a.nsplit * G * D * sizeof(float));
  a.ml = reinterpret_cast<float*>(p);
  p += al(static_cast<size_t>(U) * a.nsplit * G * 2 * sizeof(float));
  a.counter = reinterpret_cast<int*>(p);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.Hkv = Hkv;
  a.Hq = Hq;
  a.S = c.page_size;
  a.num_phys = c.num_phys_pages;
  a.max_pages = s.max_pages;
  a.cap = cap;
  cudaError_t e = cudaMemsetAsync(a.counter, 0, static_cast<size_t>(U) * sizeof(int), st);
  if (e != cudaSuccess) return e;
  const size_t tile = static_cast<size_t>(c.page_size) * D * 2;
  const size_t smem = static_cast<size_t>(kSmWarps) * kSmStages * 2 * tile +
                      static_cast<size_t>(kSmWarps) * c.page_size * ((G + 3) / 4 * 4) * sizeof(float) +
                      2 * static_cast<size_t>(a.spp) * sizeof(int);
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(U));
#define EKV_SM_CASE(DD, GG)                                                                        \
  if (D == DD && G == GG) {                                                                        \
    e = cudaFuncSetAttribute(softmax_split_kernel<DD, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(smem));                                              \
    if (e != cudaSuccess) return e;                                                                \
    e = launch_k(softmax_split_kernel<DD, GG>, grid, kSmThreads, smem, st, a);                      \
    if (e != cudaSuccess) return e;                                                                \
    return cudaGetLastError();                                                                     \
  }
  EKV_SM_CASE(128, 1) EKV_SM_CASE(128, 2) EKV_SM_CASE(128, 4) EKV_SM_CASE(128, 8) EKV_SM_CASE(128, 16)
  EKV_SM_CASE(64, 1) EKV_SM_CASE(64, 2) EKV_SM_CASE(64, 4) EKV_SM_CASE(64, 8) EKV_SM_CASE(64, 16)
#undef EKV_SM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ekv
