// Sparse α-entmax decode over the selected pages — EntmaxKV summary page
// (gist.science/fr/paper/2605.21649) §2.C, "Attention Entmax Parcimonieuse",
// with the support-only V read that §2 and §3 make exact: if the selected
// tokens contain the α-entmax support, the output equals the full-cache one.
//
// Three kernels, all on the caller's stream:
//  1. qk: split over selected pages.  K pages are staged in shared memory
//     (16 B vector loads, padded rows), the G query heads of the unit share
//     each tile, and z = scale·q·k lands in an L2-resident scratch together
//     with per-page and per-split maxima.
//  2. tau: one CTA per query head solves Σ_i [u_i − τ]_+^β = 1, u = (α−1)·z,
//     by Newton's method from τ₀ = max(u) − 1 (the function is convex and
//     decreasing, so iterates rise monotonically to the root), then for
//     β ∈ {1, 2} re-solves in closed form on the support it found.
//  3. pv: split over selected pages again; a page's V is read only when some
//     head of the unit has a token with u > τ in it.  Splits write partial
//     outputs and the last split of a unit (an atomic ticket, no waiting)
//     adds them in split order, so results are deterministic.
#include "kernels.cuh"

namespace ekv {

namespace {

struct DecodeArgs {
  const void* k_pool;
  const void* v_pool;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const void* q;
  const int32_t* sel;
  const int32_t* n_sel;
  float* out;
  float* tau_out;
  int32_t* count_out;
  uint32_t* bits_out;
  DecodeWs ws;
  float scale, am1, beta;
  int ibeta;  // β when it is 1 or 2, else 0
  int Hkv, Hq, S, num_phys, max_pages, cap, nsplit, sps, tp, dense_v, words;
};

__device__ __forceinline__ int unit_slots(const DecodeArgs& a, int unit, int P) {
  if (a.sel == nullptr) return min(P, a.cap);
  const int n = a.n_sel[unit];
  return max(0, min(n, a.cap));
}

// Logical page of a selected slot → (physical page, valid tokens); −1 when bad.
__device__ __forceinline__ int slot_page(const DecodeArgs& a, int unit, int b, int slot, int P,
                                         int L, int* nv) {
  const int lp = a.sel ? a.sel[static_cast<size_t>(unit) * a.cap + slot] : slot;
  *nv = 0;
  if (lp < 0 || lp >= P) {
    raise_flag(EKV_EFLAG_BAD_SEL);
    return -1;
  }
  const int phys = a.page_table[static_cast<size_t>(b) * a.max_pages + lp];
  if (!phys_ok(phys, a.num_phys)) return -1;
  *nv = min(a.S, L - lp * a.S);
  return phys;
}

__device__ __forceinline__ float pow_beta(float w, float beta, int ibeta) {
  if (ibeta == 1) return w;
  if (ibeta == 2) return w * w;
  return powf(w, beta);
}

// ------------------------------------------------------------------ 1. qk
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) qk_kernel(DecodeArgs a) {
  constexpr int PAD = 16 / sizeof(T);
  constexpr int RP = D + PAD;  // padded row pitch: rows start in different bank groups
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* q_s = reinterpret_cast<float*>(smem_raw);
  T* ktile = reinterpret_cast<T*>(smem_raw + G * D * sizeof(float));
  __shared__ int s_phys[8], s_nv[8];
  __shared__ unsigned int cta_key[G];

  const int split = blockIdx.x, unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, S = a.S, TP = a.tp;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int s0 = split * a.sps, s1 = min(s0 + a.sps, n_slots);
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
    // whole warps iterate (the page maxima below shuffle across S lanes)
    const int items = (TP * G * S + 31) / 32 * 32;
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
      float pm = z;
      for (int o = S / 2; o > 0; o >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
      if (t == 0 && tp < np) {
        a.ws.pmax[row * a.cap + base + tp] = pm;
        if (pm > -INFINITY) atomicMax(&cta_key[g], float_key(pm));
      }
    }
    __syncthreads();
  }
  __syncthreads();
  if (tid < G) {
    const unsigned int k = cta_key[tid];
    a.ws.cmax[(static_cast<size_t>(unit) * G + tid) * a.nsplit + split] = k == 0u ? -INFINITY : key_float(k);
  }
}

// ------------------------------------------------------------------ 2. tau
constexpr int kTauThreads = 512;

template <int VPT>
__global__ void __launch_bounds__(kTauThreads) tau_kernel(DecodeArgs a, int G) {
  const int row = blockIdx.x, unit = row / G, g = row % G, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, nt = blockDim.x;
  __shared__ float f_scratch[32];
  __shared__ double d_scratch[32];
  __shared__ int i_scratch[32];
  int L;
  const int P = seq_pages(a.seq_lens, b, a.S, a.max_pages, &L);
  const int n = unit_slots(a, unit, P) * a.S;
  const float* z = a.ws.zbuf + static_cast<size_t>(row) * a.cap * a.S;
  const size_t orow = static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + g;

  float m = -INFINITY;
  for (int s = tid; s < a.nsplit; s += nt) m = fmaxf(m, a.ws.cmax[static_cast<size_t>(row) * a.nsplit + s]);
  m = block_reduce(m, f_scratch, [](float x, float y) { return fmaxf(x, y); });

  float tau_f = INFINITY;  // no token: no support, zero output
  if (n > 0 && m > -INFINITY) {
    const float am1 = a.am1, beta = a.beta;
    const int ib = a.ibeta;
    float uv[VPT > 0 ? VPT : 1];
#pragma unroll
    for (int k = 0; k < (VPT > 0 ? VPT : 1); ++k) {
      const int i = tid + k * nt;
      uv[k] = (VPT > 0 && i < n) ? am1 * z[i] : -INFINITY;
    }
    auto accumulate = [&](double t, double& f, double& df) {
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
      if (VPT > 0) {
#pragma unroll
        for (int k = 0; k < (VPT > 0 ? VPT : 1); ++k) term(uv[k]);
      } else {
        for (int i = tid; i < n; i += nt) term(am1 * z[i]);
      }
    };
    double tau = static_cast<double>(am1 * m) - 1.0;
    for (int it = 0; it < 200; ++it) {
      double f, df;
      accumulate(tau, f, df);
      f = block_reduce(f, d_scratch, [](double x, double y) { return x + y; });
      df = block_reduce(df, d_scratch, [](double x, double y) { return x + y; });
      const double step = (f - 1.0) / (static_cast<double>(beta) * df);
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
        if (VPT > 0) {
#pragma unroll
          for (int k = 0; k < (VPT > 0 ? VPT : 1); ++k) add(uv[k]);
        } else {
          for (int i = tid; i < n; i += nt) add(am1 * z[i]);
        }
        c = block_reduce(c, d_scratch, [](double x, double y) { return x + y; });
        s1 = block_reduce(s1, d_scratch, [](double x, double y) { return x + y; });
        s2 = block_reduce(s2, d_scratch, [](double x, double y) { return x + y; });
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
    tau_f = static_cast<float>(tau);
  }

  // support of this head with the fp32 threshold every later stage uses
  int cnt = 0;
  const int words = a.words;
  for (int base = 0; base < (n + nt - 1) / nt * nt; base += nt) {
    const int i = base + tid;
    const bool in = i < n && a.am1 * z[i] > tau_f;
    cnt += in ? 1 : 0;
    const unsigned int bal = __ballot_sync(0xffffffffu, in);
    if (a.bits_out && (tid & 31) == 0 && (i >> 5) < words)
      a.bits_out[orow * words + (i >> 5)] = bal;
  }
  cnt = block_reduce(cnt, i_scratch, [](int x, int y) { return x + y; });
  if (a.bits_out) {
    // clear words past the tokens of this unit
    for (int w = (n + 31) / 32 + tid; w < words; w += nt) a.bits_out[orow * words + w] = 0u;
  }
  if (tid == 0) {
    a.ws.taus[row] = tau_f;
    if (a.tau_out) a.tau_out[orow] = tau_f;
    if (a.count_out) a.count_out[orow] = cnt;
  }
}

// ------------------------------------------------------------------ 3. pv
constexpr int kPvPages = 4;

template <typename T, int D, int G>
__global__ void __launch_bounds__(256) pv_kernel(DecodeArgs a) {
  constexpr int NPAIR = G * D / 2;
  constexpr int IPT = (NPAIR + 255) / 256;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* vtile = reinterpret_cast<T*>(smem_raw);                                  // [kPvPages][S][D]
  float* p_s = reinterpret_cast<float*>(smem_raw + kPvPages * a.S * D * sizeof(T));  // [kPvPages][G][S]
  __shared__ float s_tau[G];
  __shared__ int s_list[256];
  __shared__ int s_phys[kPvPages], s_nv[kPvPages], s_slot[kPvPages];
  __shared__ int scan_scratch[32];
  __shared__ int s_last;

  const int split = blockIdx.x, unit = blockIdx.y, b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int tid = threadIdx.x, S = a.S;
  int L;
  const int P = seq_pages(a.seq_lens, b, S, a.max_pages, &L);
  const int n_slots = unit_slots(a, unit, P);
  const int s0 = split * a.sps, s1 = min(s0 + a.sps, n_slots);
  if (tid < G) s_tau[tid] = a.ws.taus[static_cast<size_t>(unit) * G + tid];
  __syncthreads();

  float2 acc[IPT];
#pragma unroll
  for (int k = 0; k < IPT; ++k) acc[k] = make_float2(0.f, 0.f);
  const size_t zrow = static_cast<size_t>(a.cap) * S;

  for (int wbase = s0; wbase < s1; wbase += 256) {
    const int slot = wbase + tid;
    int sup = 0;
    if (slot < s1) {
      if (a.dense_v) {
        sup = 1;
      } else {
        for (int g = 0; g < G; ++g)
          if (a.am1 * a.ws.pmax[(static_cast<size_t>(unit) * G + g) * a.cap + slot] > s_tau[g]) sup = 1;
      }
    }
    int nsup;
    const int pos = block_exclusive_scan(sup, scan_scratch, &nsup);
    if (sup) s_list[pos] = slot;
    __syncthreads();
    for (int lb = 0; lb < nsup; lb += kPvPages) {
      const int np = min(kPvPages, nsup - lb);
      if (tid < np) {
        int nv;
        const int sl = s_list[lb + tid];
        s_slot[tid] = sl;
        s_phys[tid] = slot_page(a, unit, b, sl, P, L, &nv);
        s_nv[tid] = s_phys[tid] >= 0 ? nv : 0;
      }
      __syncthreads();
      constexpr int CPR = D * sizeof(T) / 16;
      for (int i = tid; i < np * S * CPR; i += blockDim.x) {
        const int tp = i / (S * CPR), r = (i / CPR) % S, c = i % CPR;
        if (r < s_nv[tp]) {
          const uint4* src = reinterpret_cast<const uint4*>(
              static_cast<const T*>(a.v_pool) + ((static_cast<size_t>(s_phys[tp]) * a.Hkv + kvh) * S + r) * D) + c;
          *reinterpret_cast<uint4*>(vtile + (tp * S + r) * D + c * (16 / sizeof(T))) = __ldcs(src);
        }
      }
      for (int i = tid; i < np * G * S; i += blockDim.x) {
        const int tp = i / (G * S), g = (i / S) % G, t = i % S;
        float p = 0.f;
        if (t < s_nv[tp]) {
          const float u = a.am1 * a.ws.zbuf[(static_cast<size_t>(unit) * G + g) * zrow +
                                            static_cast<size_t>(s_slot[tp]) * S + t];
          const float w = u - s_tau[g];
          if (w > 0.f) p = pow_beta(w, a.beta, a.ibeta);
        }
        p_s[(tp * G + g) * S + t] = p;
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < IPT; ++k) {
        const int pair = tid + k * 256;
        if (pair < NPAIR) {
          const int g = pair / (D / 2), j = 2 * (pair % (D / 2));
          for (int tp = 0; tp < np; ++tp) {
            const int nv = s_nv[tp];
            const float* pr = p_s + (tp * G + g) * S;
            const T* vr = vtile + tp * S * D + j;
            for (int t = 0; t < nv; ++t) {
              const float p = pr[t];
              float v0, v1;
              if (sizeof(T) == 2) {
                const uint32_t w = *reinterpret_cast<const uint32_t*>(vr + t * D);
                v0 = __uint_as_float(w << 16);
                v1 = __uint_as_float(w & 0xffff0000u);
              } else {
                const float2 f = *reinterpret_cast<const float2*>(vr + t * D);
                v0 = f.x;
                v1 = f.y;
              }
              acc[k] = ffma2(make_float2(p, p), make_float2(v0, v1), acc[k]);
            }
          }
        }
      }
      __syncthreads();
    }
  }

  // partial outputs, then the last split of the unit reduces them in order
  float* part = a.ws.part + (static_cast<size_t>(unit) * a.nsplit + split) * G * D;
#pragma unroll
  for (int k = 0; k < IPT; ++k) {
    const int pair = tid + k * 256;
    if (pair < NPAIR) *reinterpret_cast<float2*>(part + 2 * pair) = acc[k];
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int ticket = atomicAdd(&a.ws.counter[unit], 1);
    s_last = ticket == a.nsplit - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* part0 = a.ws.part + static_cast<size_t>(unit) * a.nsplit * G * D;
  for (int e = tid; e < G * D; e += blockDim.x) {
    float s = 0.f;
    for (int sp = 0; sp < a.nsplit; ++sp) s += __ldcg(part0 + static_cast<size_t>(sp) * G * D + e);
    const int g = e / D, j = e % D;
    a.out[(static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G + g) * D + j] = s;
  }
  if (tid == 0) a.ws.counter[unit] = 0;
}

template <typename T, int D, int G>
cudaError_t run_decode(DecodeArgs& a, int U, cudaStream_t st) {
  constexpr int PAD = 16 / sizeof(T);
  const size_t row_bytes = static_cast<size_t>(D + PAD) * sizeof(T);
  const size_t q_bytes = static_cast<size_t>(G) * D * sizeof(float);
  int tp = 256 / (G * a.S);
  tp = tp < 1 ? 1 : (tp > 8 ? 8 : tp);
  while (tp > 1 && q_bytes + static_cast<size_t>(tp) * a.S * row_bytes > 48 * 1024) tp >>= 1;
  a.tp = tp;
  const size_t qk_smem = q_bytes + static_cast<size_t>(tp) * a.S * row_bytes;
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(U));
  if (qk_smem > 48 * 1024)
    cudaFuncSetAttribute(qk_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(qk_smem));
  qk_kernel<T, D, G><<<grid, 256, qk_smem, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_max = a.cap * a.S;
  if (n_max <= 8 * kTauThreads)
    tau_kernel<8><<<U * G, kTauThreads, 0, st>>>(a, G);
  else if (n_max <= 32 * kTauThreads)
    tau_kernel<32><<<U * G, kTauThreads, 0, st>>>(a, G);
  else
    tau_kernel<0><<<U * G, kTauThreads, 0, st>>>(a, G);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t pv_smem = static_cast<size_t>(kPvPages) * a.S * D * sizeof(T) +
                         static_cast<size_t>(kPvPages) * G * a.S * sizeof(float);
  if (pv_smem > 48 * 1024)
    cudaFuncSetAttribute(pv_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(pv_smem));
  pv_kernel<T, D, G><<<grid, 256, pv_smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                          float scale, float alpha, const int32_t* sel, const int32_t* n_sel,
                          int cap, int dense_v, float* out, float* tau, int32_t* support_count,
                          uint32_t* support_bits, const DecodeWs& ws, int nsplit, cudaStream_t st) {
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
  a.Hkv = c.num_kv_heads;
  a.Hq = Hq;
  a.S = c.page_size;
  a.num_phys = c.num_phys_pages;
  a.max_pages = s.max_pages;
  a.cap = cap;
  a.nsplit = nsplit;
  a.sps = (cap + nsplit - 1) / nsplit;
  a.dense_v = dense_v;
  a.words = (cap * c.page_size + 31) / 32;
  const int G = Hq / c.num_kv_heads, U = s.batch * c.num_kv_heads;
#define EKV_DEC_CASE(TT, DD, GG) \
  if (c.head_dim == DD && G == GG) return run_decode<TT, DD, GG>(a, U, st);
  if (c.dtype == EKV_BF16) {
    EKV_DEC_CASE(bf16, 128, 1) EKV_DEC_CASE(bf16, 128, 2) EKV_DEC_CASE(bf16, 128, 4)
    EKV_DEC_CASE(bf16, 128, 8) EKV_DEC_CASE(bf16, 128, 16)
    EKV_DEC_CASE(bf16, 64, 1) EKV_DEC_CASE(bf16, 64, 2) EKV_DEC_CASE(bf16, 64, 4)
    EKV_DEC_CASE(bf16, 64, 8) EKV_DEC_CASE(bf16, 64, 16)
  } else {
    EKV_DEC_CASE(float, 128, 1) EKV_DEC_CASE(float, 128, 2) EKV_DEC_CASE(float, 128, 4)
    EKV_DEC_CASE(float, 128, 8) EKV_DEC_CASE(float, 128, 16)
    EKV_DEC_CASE(float, 64, 1) EKV_DEC_CASE(float, 64, 2) EKV_DEC_CASE(float, 64, 4)
    EKV_DEC_CASE(float, 64, 8) EKV_DEC_CASE(float, 64, 16)
  }
#undef EKV_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ekv
