// Arguments and per-slot helpers shared by the decode kernels (decode.cu: the
// three-kernel path; decode_fused.cu: the one-cluster-per-unit path).
#pragma once

#include "kernels.cuh"

namespace ekv {

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
  int ibeta;  // β when it is 1 or 2 (closed-form τ on the support), else 0
  int ipow;   // β when it is an integer 1..4 (powers by multiplication), else 0
  int Hkv, Hq, S, num_phys, max_pages, cap, spp_pv, dense_v, words;
};

template <class A>
__device__ __forceinline__ int unit_slots(const A& a, int unit, int P) {
  if (a.sel == nullptr) return min(P, a.cap);
  const int n = a.n_sel[unit];
  return max(0, min(n, a.cap));
}

// Logical page of a selected slot → (physical page, valid tokens); −1 when bad.
template <class A>
__device__ __forceinline__ int slot_page(const A& a, int unit, int b, int slot, int P, int L, int* nv) {
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

// w^β for w > 0: multiplications for integer β ≤ 4, powf otherwise.
__device__ __forceinline__ float pow_beta(float w, float beta, int ipow) {
  switch (ipow) {
    case 1: return w;
    case 2: return w * w;
    case 3: return w * w * w;
    case 4: { const float w2 = w * w; return w2 * w2; }
    default: return powf(w, beta);
  }
}
// The same with a fast base-2 exp/log for non-integer β (relative error near
// 1e-6, far inside the bf16 output tolerance): a few instructions instead of
// an inlined powf, for code that runs once per CTA.
// Newton step toward the root of Σ_i (u_i − τ)_+^β = 1, taken on
// h(τ) = (Σ_i (u_i − τ)_+^β)^(1/β), the ℓ_β norm of (u − τ)_+: convex and
// decreasing, so steps from the left never pass the root, and close to linear
// far from it (Newton on the sum itself closes only a fraction 1/β of the gap
// there).  With F = 1 + f the sum and s = Σ_i (u_i − τ)_+^(β−1), the step
// (h − 1)/(−h') is F^(1−1/β)·(F^(1/β) − 1)/s, formed from f without
// cancellation near the root; for β = 1 it is Newton's step f/s.
template <typename V>
__device__ __forceinline__ V norm_newton_step(V f, V s, V beta) {
  if constexpr (sizeof(V) == 8) {
    const double l = log1p(f);
    return exp((1.0 - 1.0 / beta) * l) * expm1(l / beta) / s;
  } else {
    const float l = log1pf(f);
    return expf((1.0f - 1.0f / beta) * l) * expm1f(l / beta) / s;
  }
}

__device__ __forceinline__ float pow_beta_fast(float w, float beta, int ipow) {
  switch (ipow) {
    case 1: return w;
    case 2: return w * w;
    case 3: return w * w * w;
    case 4: { const float w2 = w * w; return w2 * w2; }
    default: return exp2f(beta * __log2f(w));
  }
}

// B fragments of the m16n8k16 score MMA: the G queries of KV head kvh of
// sequence b, under the k permutation that lets lane (g, t) feed its A
// fragments from one 16-byte load per row and 32-column chunk: chunk c,
// k-step 2c takes columns 32c + 8t + {0..3}, k-step 2c+1 columns 32c + 8t +
// {4..7} (so every row uses the same column order).
template <int D, int G, class A>
__device__ __forceinline__ void load_q_frags(const A& a, int b, int kvh, int g, int t,
                                             uint32_t (&bfrag)[D / 16][(G + 7) / 8][2]) {
  constexpr int KS = D / 16, NT = (G + 7) / 8;
  const bf16* qb = static_cast<const bf16*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(kvh) * G) * D;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int col = nt * 8 + g;
      const int k0 = 32 * (ks >> 1) + 8 * t + 4 * (ks & 1);
      if (col < G) {
        const uint2 w = *reinterpret_cast<const uint2*>(qb + col * D + k0);
        bfrag[ks][nt][0] = w.x;
        bfrag[ks][nt][1] = w.y;
      } else {
        bfrag[ks][nt][0] = bfrag[ks][nt][1] = 0u;
      }
    }
}

// One m16 tile of scores: rows (g, g+8) of the tile as uint4 chunks va / vb
// (chunk c = columns 32c + 8t .. +7), times the query fragments.
template <int D, int G>
__device__ __forceinline__ void score_mtile(const uint4 (&va)[D / 32], const uint4 (&vb)[D / 32],
                                            const uint32_t (&bfrag)[D / 16][(G + 7) / 8][2],
                                            float (&acc)[(G + 7) / 8][4]) {
  constexpr int KP = D / 32, NT = (G + 7) / 8;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int c = 0; c < KP; ++c) {
    const uint32_t f0[4] = {va[c].x, vb[c].x, va[c].y, vb[c].y};
    const uint32_t f1[4] = {va[c].z, vb[c].z, va[c].w, vb[c].w};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mma_bf16(acc[nt], f0, bfrag[2 * c][nt][0], bfrag[2 * c][nt][1]);
      mma_bf16(acc[nt], f1, bfrag[2 * c + 1][nt][0], bfrag[2 * c + 1][nt][1]);
    }
  }
}

// Launch of the two-launch split decode (decode_split.cu): false when the
// configuration does not fit it.
template <int D, int G>
bool split_decode_fits(int cap, int S);
template <int D, int G>
cudaError_t run_split_decode(DecodeArgs& a, int units, cudaStream_t st);
// The three-kernel decode's V pass alone (decode.cu), over the scores and τ
// the split decode left in the workspace: its dense-V variant.
template <int D, int G>
cudaError_t run_dense_v_pass(DecodeArgs& a, int units, cudaStream_t st);

// Launch of the fused path: false when the configuration does not fit it
// (the caller then runs the three-kernel path).
template <int D, int G>
bool fused_decode_fits(int units, int cap, int S);
// CTAs per unit of the fused path's cluster (0: it does not fit).
template <int D, int G>
int fused_decode_cluster(int units, int cap, int S);

// The decode path of a bf16 selection: the one-cluster-per-unit kernel when
// at least kFusedMinCluster CTAs can work on each unit at once (few units),
// else the split decode when the selection fits it (many units, or the full
// cache: two launches, a third for dense V), else whichever fits, else the
// three-kernel path.
constexpr int kFusedMinCluster = 4;
enum class DecodePath { kFused, kSplit, kThree };
template <int D, int G>
DecodePath choose_decode_path(int units, int cap, int S, int dense_v) {
  if (units > 65535) return DecodePath::kThree;
  const int C = fused_decode_cluster<D, G>(units, cap, S);
  const bool split = split_decode_fits<D, G>(cap, S);
  if (C >= kFusedMinCluster) return DecodePath::kFused;
  if (split) return DecodePath::kSplit;
  return C > 0 ? DecodePath::kFused : DecodePath::kThree;
}
template <int D, int G>
cudaError_t run_fused_decode(DecodeArgs& a, int units, cudaStream_t st);

}  // namespace ekv
