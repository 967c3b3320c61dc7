// Shared device helpers of libekv (sm_100a).  Nothing here is shared with the
// float64 oracle; both only read the same stored cache bytes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/ekv.h"

namespace ekv {

using bf16 = __nv_bfloat16;

// Sticky device error word (EKV_EFLAG_* bits), read by ekv_get_error().
extern __device__ unsigned int g_error_flags;

__device__ __forceinline__ void raise_flag(unsigned int bit) { atomicOr(&g_error_flags, bit); }

// A hint that brings the 128-byte line holding p into L2.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ------------------------------------------------------------------ launches
// Every kernel is launched with programmatic stream serialization: its CTAs
// may be dispatched while the previous kernel on the stream drains.  Each
// kernel therefore opens with grid_dep_enter(): it waits until the previous
// kernel has completed and its memory is visible (griddepcontrol.wait; a
// no-op when launched without the attribute), then lets the next kernel be
// dispatched early.  No global memory is read or written before the wait
// (the fused decode only hints L2 prefetches of its page-table row there,
// which no kernel writes).
__device__ __forceinline__ void grid_dep_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ loads
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

// Eight consecutive elements (16 B for bf16, 32 B for fp32) widened to fp32.
__device__ __forceinline__ void load8(const bf16* p, float* v) {
  uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(ws[i] << 16);
    v[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float* v) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// Four consecutive elements widened to fp32.
__device__ __forceinline__ void load4(const bf16* p, float* v) {
  uint2 w = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(w.x << 16);
  v[1] = __uint_as_float(w.x & 0xffff0000u);
  v[2] = __uint_as_float(w.y << 16);
  v[3] = __uint_as_float(w.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* p, float* v) {
  float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

// ------------------------------------------------------------------ rounding
// float64 → bfloat16 bits, round to nearest, ties to even, written from the
// IEEE-754 binary64 / bfloat16 encodings: bfloat16 keeps the sign, fp32's
// 8-bit exponent and 7 explicit mantissa bits.
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  const unsigned int sign = static_cast<unsigned int>(u >> 63) << 15;
  const unsigned long long a = u & 0x7fffffffffffffffull;
  if (a == 0) return static_cast<uint16_t>(sign);
  if (a >= 0x7ff0000000000000ull)  // inf / nan
    return static_cast<uint16_t>(sign | 0x7f80u | (a > 0x7ff0000000000000ull ? 0x40u : 0u));
  const int e = static_cast<int>(a >> 52);
  if (e >= 1023 - 126) {
    // normal bfloat16 range: drop 45 of binary64's 52 mantissa bits, RNE
    const unsigned long long lsb = (a >> 45) & 1ull;
    const unsigned long long r = (a + 0x0fffffffffffull + lsb) >> 45;
    const int eb = static_cast<int>(r >> 7) - 1023 + 127;
    if (eb >= 255) return static_cast<uint16_t>(sign | 0x7f80u);
    return static_cast<uint16_t>(sign | (static_cast<unsigned int>(eb) << 7) |
                                 static_cast<unsigned int>(r & 0x7fu));
  }
  // subnormal bfloat16: a multiple of 2^-133; the scaling by 2^133 is exact
  const double k = rint(fabs(x) * 0x1p133);
  return static_cast<uint16_t>(sign | static_cast<unsigned int>(k));
}

template <typename T>
__device__ __forceinline__ T round_store(double x);
template <>
__device__ __forceinline__ float round_store<float>(double x) { return __double2float_rn(x); }
template <>
__device__ __forceinline__ bf16 round_store<bf16>(double x) {
  return __ushort_as_bfloat16(f64_to_bf16_bits(x));
}

// ------------------------------------------------------------------ keys
// Order-preserving map fp32 → uint32 (larger float ⇒ larger key); −0 → +0.
__device__ __forceinline__ uint32_t float_key(float x) {
  uint32_t b = __float_as_uint(x + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// ------------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Reduce N per-lane values across independent groups of W lanes (W a power
// of two ≤ 32, N ≤ W) with N−1+log2(W/N) shuffles: each halving step trades
// half of the values with the partner lane.  On return vals[0] of lane l
// holds the group total of value index transpose_index<N, W>(l); lanes of a
// group that differ only in their low bits hold the same total.
template <int N, int W>
__device__ __forceinline__ void warp_transpose_sum(float* vals, int lane) {
  static_assert(N <= W && W <= 32, "N must fit in the lane group");
  int count = N;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) {
    if (count > 1) {
      const bool upper = (lane & o) != 0;
      const int half = count >> 1;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < half) {
          const float send = upper ? vals[i] : vals[i + half];
          const float keep = upper ? vals[i + half] : vals[i];
          vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      count = half;
    } else {
      vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], o);
    }
  }
}
// Index of the value a lane holds after warp_transpose_sum<N, W>.
template <int N, int W>
__device__ __forceinline__ int transpose_index(int lane) {
  int idx = 0, count = N;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) {
    if (count > 1) {
      count >>= 1;
      if (lane & o) idx += count;
    }
  }
  return idx;
}
// True on exactly one lane per (group, value index) after the transpose.
template <int N, int W>
__device__ __forceinline__ bool transpose_owner(int lane) {
  constexpr int low = W / N;  // lanes holding the same value are the low log2(W/N) bits
  return (lane & (low - 1)) == 0;
}

// Packed fp32 FMA of sm_100 (two lanes of fp32 per instruction).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// ------------------------------------------------------------------ tensor cores
// Warp-level bf16 MMA (m16n8k16, fp32 accumulate) and its fragment loads.
// A (16×16, row-major): a0 = (row g, k 2t..2t+1), a1 = (row g+8, same k),
// a2 = (row g, k 2t+8..), a3 = (row g+8, k 2t+8..); B (16×8, k-major per
// column): b0 = (k 2t..2t+1, col g), b1 = (k 2t+8..2t+9, col g); C/D:
// c0,c1 = (row g, cols 2t, 2t+1), c2,c3 = (row g+8, cols 2t, 2t+1);
// g = lane / 4, t = lane % 4.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two bf16 values (given as fp32 holding bf16-representable numbers) → bf16x2.
__device__ __forceinline__ uint32_t pack_bf16_exact(float lo, float hi) {
  return (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xffff0000u);
}
// x ≈ hi + lo with hi, lo bf16 (hi = nearest bf16 of x, lo = nearest of the rest).
__device__ __forceinline__ void split_bf16(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = __bfloat162float(__float2bfloat16_rn(x - hi));
}

// Block-wide reductions through shared memory (blockDim.x multiple of 32).
template <typename V, typename Op>
__device__ __forceinline__ V block_reduce(V v, V* scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  V r = scratch[0];
  for (int w = 1; w < nw; ++w) r = op(r, scratch[w]);
  return r;
}

// Exclusive prefix sum of an int over the block; *total receives the sum.
// Warp scans, then one warp scans the warp totals (blockDim.x ≤ 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) scratch[lane] = w;  // inclusive warp-total prefix
  }
  __syncthreads();
  *total = scratch[nw - 1];
  return (warp > 0 ? scratch[warp - 1] : 0) + x - v;
}

// ------------------------------------------------------------------ async copies
// Bulk global→shared copies completed on an mbarrier (the TMA engine's 1-D
// form), and bounded waits: a wait that gives up raises EKV_EFLAG_TIMEOUT and
// returns false instead of spinning forever.
constexpr unsigned int kSpinLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned int bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned int parity) {
  unsigned int done;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0u;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned int parity,
                                          unsigned int limit = kSpinLimit) {
  for (unsigned int i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  raise_flag(EKV_EFLAG_TIMEOUT);
  return false;
}
// bytes: a multiple of 16; both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned int bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Orders this thread's earlier generic-proxy accesses of shared memory before
// its later async-proxy ones (a bulk copy into a slot that was read).
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Sequence geometry with device-side checks (no trap: clamp and flag).
__device__ __forceinline__ int seq_pages(const int32_t* seq_lens, int b, int S, int max_pages,
                                         int* len_out) {
  int L = seq_lens[b];
  if (L < 1 || L > max_pages * S) {
    raise_flag(EKV_EFLAG_BAD_LEN);
    L = L < 1 ? 0 : max_pages * S;
  }
  *len_out = L;
  return (L + S - 1) / S;
}
__device__ __forceinline__ bool phys_ok(int phys, int num_phys) {
  if (phys < 0 || phys >= num_phys) {
    raise_flag(EKV_EFLAG_BAD_PAGE);
    return false;
  }
  return true;
}

}  // namespace ekv
