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
// [mean | var] — which is the whole per-step HBM traffic of selection, and
// both are a skinny contraction [rows × 2d]·[2d × n] with n a few columns
// per query head.
//
// Persistent, warp-specialised design: kCtasPerSm CTAs per SM take equal slices of
// the flattened (sequence, KV head, page) rows.  A producer warp gathers the
// slice's rows through the page table with bulk async copies (one copy per
// row, 512 B for bf16 d = 128) into a kStages-deep ring of 16-row stages,
// each completed on an mbarrier; rows sit at a 16 B-padded pitch so ldmatrix
// reads them without bank conflicts.  A consumer warp takes each 16-row stage
// through bf16 tensor-core MMAs (m16n8k16, fp32 accumulation): the
// rows are the A operand, the query coefficients a register-resident B
// operand.  bf16·bf16 products are exact in fp32.  The Gaussian variance
// columns carry q² split into two bf16 parts (hi + lo, relative error 2⁻¹⁷).
// fp32 caches (and 16-head Gaussian groups) use a CUDA-core consumer instead.
// Every mbarrier wait is bounded.
#include <type_traits>

#include "kernels.cuh"

namespace ekv {

namespace {

// Small CTAs, several per SM: one 512 B bulk copy per row is issued at a
// limited rate per CTA (about one every 55 cycles on B200, measured), so the
// row-request rate, and with it the bandwidth, scales with CTAs per SM.
constexpr int kRows = 16;        // rows per stage (one tensor-core m-tile)
constexpr int kStages = 6;       // stages in flight per CTA
constexpr int kConsumers = 1;    // consumer warps (16 rows each)
constexpr int kIdAhead = 8;      // stages of page ids fetched ahead of the row copies
constexpr int kCtasPerSm = 4;
constexpr int kStreamThreads = 32 * (kConsumers + 1);

struct StreamArgs {
  const void* rows;          // box or mom pool
  const int32_t* page_table;
  const int32_t* seq_lens;
  const void* q;
  float* ub;                 // score: [U, max_pages]
  GaussWs gws;               // Gaussian statistics outputs
  float scale, am1;
  int Hkv, Hq, S, num_phys, max_pages, batch;
  // 1: the preceding kernel on the stream is the cache append, whose writes
  // reach only the last page of every sequence; the bf16 kernel then waits
  // for it just before the tiles holding those pages (see meta_direct_kernel)
  int defer_wait;
};

// Walks a CTA's slice [f0, f1) of the flattened rows as ≤ kRows-row stages
// that never cross a (sequence, KV head) boundary.
struct StageIter {
  const int* prefix;  // [batch+1] rows before each sequence (pages·Hkv)
  int batch, Hkv, rows;
  long long f, f1;
  int b = 0, h = 0, p = 0, pe = 0;
  __device__ bool next(int& ob, int& oh, int& op0, int& on) {
    while (p >= pe) {
      if (f >= f1) return false;
      int lo = 0, hi = batch;  // largest b with prefix[b] <= f
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= f) lo = mid; else hi = mid;
      }
      b = lo;
      const int Pb = (prefix[b + 1] - prefix[b]) / Hkv;
      const long long r = f - prefix[b];
      h = static_cast<int>(r / Pb);
      p = static_cast<int>(r % Pb);
      const long long seg_end =
          min(f1, static_cast<long long>(prefix[b]) + static_cast<long long>(h + 1) * Pb);
      pe = p + static_cast<int>(seg_end - f);
      f = seg_end;
    }
    ob = b;
    oh = h;
    op0 = p;
    on = min(rows, pe - p);
    p += on;
    return true;
  }
};

template <typename T, int G, bool GAUSS>
struct UseMma {
  static constexpr bool value = std::is_same<T, bf16>::value && (!GAUSS || G <= 8);
};

// Columns of the B operand per tile group: score n = G heads; Gaussian n = G
// mean columns + 2G variance columns (q² hi, q² lo).
template <int G, bool GAUSS>
struct Cols {
  static constexpr int n = GAUSS ? 3 * G : G;
  static constexpr int tiles = (n + 7) / 8;
};

// Rows per stage.
template <int ROWP>
struct StageRows {
  static constexpr int value = kRows;
};

template <typename T, int D, int G, bool GAUSS>
__global__ void __launch_bounds__(kStreamThreads, kCtasPerSm) meta_stream_kernel(StreamArgs a) {
  grid_dep_enter();
  constexpr int ROW = 2 * D * static_cast<int>(sizeof(T));  // bytes per metadata row
  constexpr int ROWP = ROW + 16;                             // padded pitch in shared memory
  constexpr bool MMA = UseMma<T, G, GAUSS>::value;
  constexpr int kRows = StageRows<ROWP>::value;
  static_assert(!MMA || kRows == 16 * kConsumers, "tensor-core consumers take 16 rows each");

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* stage_buf = smem;                                             // [kStages][kRows][ROWP]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kRows * ROWP);  // [kStages]
  uint64_t* empty = full + kStages;                                             // [kStages]
  signed char* ok = reinterpret_cast<signed char*>(empty + kStages);            // [kStages][kRows]
  float* ctile = reinterpret_cast<float*>(ok + kStages * kRows);                // [kConsumers][16][24]
  int* pid = reinterpret_cast<int*>(ctile + kConsumers * 16 * 24);              // [kIdAhead][kRows]
  int4* sdesc = reinterpret_cast<int4*>(pid + kIdAhead * kRows);                // [kIdAhead]
  int* prefix = reinterpret_cast<int*>(sdesc + kIdAhead);                       // [batch+1]
  __shared__ int scan_scratch[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // rows before each sequence: ⌈L_b/S⌉ pages × Hkv heads
  int carry = 0;
  for (int base = 0; base < a.batch; base += blockDim.x) {
    const int b = base + tid;
    int L, rows = 0;
    if (b < a.batch) rows = seq_pages(a.seq_lens, b, a.S, a.max_pages, &L) * a.Hkv;
    int total;
    const int ex = block_exclusive_scan(rows, scan_scratch, &total);
    if (b < a.batch) prefix[b] = carry + ex;
    carry += total;
  }
  if (tid == 0) {
    prefix[a.batch] = carry;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const long long total_rows = prefix[a.batch];
  StageIter it{prefix, a.batch, a.Hkv, kRows, total_rows * blockIdx.x / gridDim.x,
               total_rows * (blockIdx.x + 1) / gridDim.x};

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    // Page ids run kIdAhead stages ahead of the row copies: each stage's ids
    // are fetched with asynchronous 4 B copies into a shared ring (one commit
    // group per stage), so no global-load latency sits on the copy path.
    int stage = 0;
    unsigned int phase = 0;
    StageIter ahead = it;
    auto prefetch = [&](int slot) {
      int bb, hh, pp, nn;
      const bool have = ahead.next(bb, hh, pp, nn);
      if (lane == 0) sdesc[slot] = have ? make_int4(bb, hh, pp, nn) : make_int4(0, 0, 0, -1);
      if (have) {
        const int32_t* pt = a.page_table + static_cast<size_t>(bb) * a.max_pages + pp;
        for (int i = lane; i < nn; i += 32)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(&pid[slot * kRows + i])),
                       "l"(pt + i)
                       : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    for (int j = 0; j < kIdAhead; ++j) prefetch(j);
    for (int s_i = 0;; ++s_i) {
      const int slot = s_i % kIdAhead;
      asm volatile("cp.async.wait_group %0;" ::"n"(kIdAhead - 1) : "memory");
      __syncwarp();
      const int4 dsc = sdesc[slot];
      const int h = dsc.y, n = dsc.w;
      if (n < 0) break;
      int ids[2];
      ids[0] = lane < n ? pid[slot * kRows + lane] : -1;
      ids[1] = (kRows > 32 && lane + 32 < n) ? pid[slot * kRows + (kRows > 32 ? lane + 32 : 0)] : -1;
      __syncwarp();
      prefetch(slot);  // refill this slot with the stage kIdAhead further on
      if (!mbar_wait(&empty[stage], phase ^ 1u)) break;
      int bytes = 0;
      const void* src[2];
      for (int k = 0; k < 2; ++k) {
        const int i = lane + 32 * k;
        src[k] = nullptr;
        if (i < n) {
          const bool good = phys_ok(ids[k], a.num_phys);
          ok[stage * kRows + i] = good ? 1 : 0;
          if (good) {
            src[k] = static_cast<const unsigned char*>(a.rows) + (static_cast<size_t>(h) * a.num_phys + ids[k]) * ROW;
            bytes += ROW;
          }
        }
      }
      bytes = warp_sum(bytes);
      __syncwarp();  // the validity flags above are ordered before the arrive
      if (lane == 0) mbar_arrive_expect_tx(&full[stage], static_cast<unsigned int>(bytes));
      __syncwarp();  // copies are issued after the expected bytes are registered
      for (int k = 0; k < 2; ++k)
        if (src[k] != nullptr)
          bulk_g2s(stage_buf + (stage * kRows + lane + 32 * k) * ROWP, src[k], ROW, &full[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // drain: let every issued copy land before the CTA exits
    for (int s = 0; s < kStages; ++s) mbar_wait(&full[s], s < stage ? phase : phase ^ 1u);
    return;
  }

  // ---------------------------------------------------------------- consumers
  int stage = 0;
  unsigned int phase = 0;
  int b, h, p0, n, cur_unit = -1, L = 0;

  if constexpr (MMA) {
    constexpr int KS = 2 * D / 16;  // k-steps over the [first | second] row
    constexpr int NT = Cols<G, GAUSS>::tiles;
    const int g = lane >> 2, t = lane & 3;
    uint32_t bfrag[KS][NT][2];
    const uint32_t warp_rows = smem_addr(stage_buf) + (warp * 16 + (lane & 15)) * ROWP + (lane >> 4) * 16;
    float* my_tile = ctile + warp * 16 * 24;
    while (it.next(b, h, p0, n)) {
      const int unit = b * a.Hkv + h;
      if (unit != cur_unit) {
        cur_unit = unit;
        seq_pages(a.seq_lens, b, a.S, a.max_pages, &L);
        const bf16* qb = static_cast<const bf16*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(h) * G) * D;
        // coefficient of column c at row-position k (k < D: first half, else second)
        auto coef = [&](int c, int k) -> float {
          const bool lo_half = k < D;
          const int j = lo_half ? k : k - D;
          if constexpr (!GAUSS) {
            if (c >= G) return 0.f;
            const float v = __bfloat162float(qb[c * D + j]);
            return lo_half ? fmaxf(v, 0.f) : fminf(v, 0.f);
          } else {
            if (c < G) return lo_half ? __bfloat162float(qb[c * D + j]) : 0.f;
            if (c >= 3 * G || lo_half) return 0.f;
            const int hh = (c - G) >> 1;
            const float v = __bfloat162float(qb[hh * D + j]);
            float hi, lo;
            split_bf16(v * v, hi, lo);
            return ((c - G) & 1) ? lo : hi;
          }
        };
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int c = nt * 8 + g, k0 = kk * 16 + 2 * t;
            bfrag[kk][nt][0] = pack_bf16_exact(coef(c, k0), coef(c, k0 + 1));
            bfrag[kk][nt][1] = pack_bf16_exact(coef(c, k0 + 8), coef(c, k0 + 9));
          }
      }
      if (!mbar_wait(&full[stage], phase)) break;
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      if (warp * 16 < n) {
        const uint32_t base = warp_rows + stage * kRows * ROWP;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          uint32_t af[4];
          ldsm_x4(base + kk * 32, af);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], af, bfrag[kk][nt][0], bfrag[kk][nt][1]);
        }
      }
      const int r_lo = warp * 16 + g, r_hi = r_lo + 8;
      const bool live_lo = r_lo < n && ok[stage * kRows + r_lo];
      const bool live_hi = r_hi < n && ok[stage * kRows + r_hi];
      if constexpr (!GAUSS) {
        float m_lo = -INFINITY, m_hi = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int c0 = nt * 8 + 2 * t;
          if (c0 < G) { m_lo = fmaxf(m_lo, acc[nt][0]); m_hi = fmaxf(m_hi, acc[nt][2]); }
          if (c0 + 1 < G) { m_lo = fmaxf(m_lo, acc[nt][1]); m_hi = fmaxf(m_hi, acc[nt][3]); }
        }
        m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 1));
        m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 1));
        m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 2));
        m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 2));
        if (t == 0) {
          float* urow = a.ub + static_cast<size_t>(cur_unit) * a.max_pages + p0;
          if (r_lo < n) urow[r_lo] = live_lo ? a.scale * m_lo : -INFINITY;
          if (r_hi < n) urow[r_hi] = live_hi ? a.scale * m_hi : -INFINITY;
        }
      } else {
        constexpr int TW = 24;  // tile width in floats
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int c0 = nt * 8 + 2 * t;
          my_tile[g * TW + c0] = acc[nt][0];
          my_tile[g * TW + c0 + 1] = acc[nt][1];
          my_tile[(g + 8) * TW + c0] = acc[nt][2];
          my_tile[(g + 8) * TW + c0 + 1] = acc[nt][3];
        }
        __syncwarp();
        for (int pr = lane; pr < 16 * G; pr += 32) {
          const int r = pr / G, hh = pr % G, rr = warp * 16 + r;
          if (rr < n) {
            const int p = p0 + rr;
            const bool live = ok[stage * kRows + rr] != 0;
            const float m = a.scale * my_tile[r * TW + hh];
            const float s2 = my_tile[r * TW + G + 2 * hh] + my_tile[r * TW + G + 2 * hh + 1];
            const float sd = a.scale * sqrtf(fmaxf(s2, 0.f));
            const float nv = static_cast<float>(min(a.S, L - p * a.S));
            float mu = a.am1 * m, sg = a.am1 * sd, hat = a.am1 * (m + sd * sqrtf(2.f * logf(nv)));
            if (!live) mu = hat = -INFINITY, sg = 0.f;
            const size_t o = (static_cast<size_t>(cur_unit) * G + hh) * a.max_pages + p;
            a.gws.mu[o] = mu;
            a.gws.sig[o] = sg;
            a.gws.hat[o] = hat;
          }
        }
        __syncwarp();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
  } else {
    // CUDA-core consumer: each lane owns one 8-element chunk of a row
    constexpr int LPP = D / 4;       // lanes per row
    constexpr int PPW = 32 / LPP;    // rows per warp step
    constexpr int HALF = LPP / 2;
    constexpr int CH = sizeof(T) / 2;  // uint4 per lane chunk
    const int ps = lane / LPP, wl = lane % LPP;
    const int e0 = wl * 8;
    const bool first = e0 < D;
    const int j0 = first ? e0 : e0 - D;
    float2 coef[G][4];
    while (it.next(b, h, p0, n)) {
      const int unit = b * a.Hkv + h;
      if (unit != cur_unit) {
        cur_unit = unit;
        seq_pages(a.seq_lens, b, a.S, a.max_pages, &L);
        const T* qb = static_cast<const T*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(h) * G) * D + j0;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          float v[8];
          load8(qb + static_cast<size_t>(gg) * D, v);
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
            coef[gg][i] = make_float2(c0, c1);
          }
        }
      }
      if (!mbar_wait(&full[stage], phase)) break;
      for (int r0 = warp * PPW; r0 < n; r0 += kConsumers * PPW) {
        const int r = r0 + ps;
        const bool live = r < n && ok[stage * kRows + r];
        const uint4* chunk = reinterpret_cast<const uint4*>(stage_buf + (stage * kRows + (r < n ? r : 0)) * ROWP) + wl * CH;
        float acc[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          float2 a2 = make_float2(0.f, 0.f);
          if (live) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 v = chunk[(i >> 1) * (CH - 1)];
              float2 pr;
              if constexpr (sizeof(T) == 2) {
                const uint32_t w = i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
                pr = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
              } else {
                pr = (i & 1) ? make_float2(__uint_as_float(v.z), __uint_as_float(v.w))
                             : make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
              }
              a2 = ffma2(coef[gg][i], pr, a2);
            }
          }
          acc[gg] = a2.x + a2.y;
        }
        const int p = p0 + r;
        if constexpr (!GAUSS) {
          warp_transpose_sum<G, LPP>(acc, lane);
          float m = acc[0];
#pragma unroll
          for (int o = LPP / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (wl == 0 && r < n)
            a.ub[static_cast<size_t>(unit) * a.max_pages + p] = live ? a.scale * m : -INFINITY;
        } else {
          warp_transpose_sum<G, HALF>(acc, lane);
          const float s2 = __shfl_xor_sync(0xffffffffu, acc[0], HALF);
          if (first && transpose_owner<G, HALF>(lane) && r < n) {
            const int gg = transpose_index<G, HALF>(lane);
            const size_t o = (static_cast<size_t>(unit) * G + gg) * a.max_pages + p;
            const float nv = static_cast<float>(min(a.S, L - p * a.S));
            const float m = a.scale * acc[0];
            const float sd = a.scale * sqrtf(fmaxf(s2, 0.f));
            float mu = a.am1 * m, sg = a.am1 * sd, hat = a.am1 * (m + sd * sqrtf(2.f * logf(nv)));
            if (!live) mu = hat = -INFINITY, sg = 0.f;
            a.gws.mu[o] = mu;
            a.gws.sig[o] = sg;
            a.gws.hat[o] = hat;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
  }
}

// ---------------------------------------------------------------------------
// bf16 path: every warp streams 16-row tiles straight from global memory into
// tensor-core A fragments.  Lane (g, t) = (lane / 4, lane % 4) loads, per
// 32-element chunk c of its rows g and g + 8, the 16 B at columns
// 32c + 8t … 32c + 8t + 7; those four bf16 pairs are the A fragments of two
// k-steps under a fixed permutation of k (columns 8t+4e+{0,1} and
// 8t+4e+{2,3} of step e take the places of k 2t, 2t+1 and 2t+8, 2t+9).  The B
// fragments use the same permutation, so every product pairs the right
// coefficient with the right element.  A warp keeps one 16-row tile (8 KB for
// bf16, d = 128) of 16 B loads in flight and the SM runs 16 such warps, about
// the 128 KB per SM that saturates HBM at its loaded latency.  Each warp owns
// a contiguous range of tiles, so its query coefficients change only at unit
// boundaries, and the next tile's page ids load while the current tile's
// rows are in flight.
constexpr int kDirectWarps = 4;
constexpr int kTile = 16;

// 8-column tiles of B per k-step in the direct kernel.  The score takes the
// G heads' q⁺ over the kmax half of a row and q⁻ over the kmin half, in the
// same columns.  The Gaussian statistics take q over the mean half (G
// columns) and q² hi, lo over the variance half (2G columns): each k-step
// lies in one half, so it multiplies only that half's columns.
template <int G, bool GAUSS>
struct DirectTiles {
  static constexpr int value = ((GAUSS ? 2 * G : G) + 7) / 8;
};

// CTAs per SM: 4 (16 warps) while the B fragments are one 8-column tile, 2
// with more (G = 8 Gaussian statistics).
template <int D, int G, bool GAUSS>
struct DirectOcc {
  static constexpr int value = DirectTiles<G, GAUSS>::value > 1 ? 2 : 4;
};

template <int D, int G, bool GAUSS>
__global__ void __launch_bounds__(32 * kDirectWarps, DirectOcc<D, G, GAUSS>::value)
    meta_direct_kernel(StreamArgs a) {
  // With defer_wait the kernel overlaps the append that precedes it: tiles
  // without a sequence's last page never read what the append writes, so
  // only a warp about to load such a tile waits for the append to finish.
  if (a.defer_wait) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  } else {
    grid_dep_enter();
  }
  bool waited = a.defer_wait == 0;
  constexpr int KP = 2 * D / 32;                 // 32-element chunks per row
  constexpr int NT = DirectTiles<G, GAUSS>::value; // 8-column tiles of B per k-step
  constexpr int ROW = 2 * D * 2;              // bytes per metadata row
  extern __shared__ __align__(16) int dyn[];
  float* ctile = reinterpret_cast<float*>(dyn);                // [kDirectWarps][16][24]
  int* prefix = dyn + kDirectWarps * 16 * 24;                  // [batch + 1] tiles before each sequence
  __shared__ int scan_scratch[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;

  int carry = 0;
  for (int base = 0; base < a.batch; base += blockDim.x) {
    const int b = base + tid;
    int L, tiles = 0;
    if (b < a.batch) tiles = (seq_pages(a.seq_lens, b, a.S, a.max_pages, &L) + kTile - 1) / kTile * a.Hkv;
    int total;
    const int ex = block_exclusive_scan(tiles, scan_scratch, &total);
    if (b < a.batch) prefix[b] = carry + ex;
    carry += total;
  }
  if (tid == 0) prefix[a.batch] = carry;
  __syncthreads();
  const long long total = prefix[a.batch];
  const long long nw = static_cast<long long>(gridDim.x) * kDirectWarps;
  const long long gw = static_cast<long long>(blockIdx.x) * kDirectWarps + warp;
  const long long t0 = total * gw / nw, t1 = total * (gw + 1) / nw;
  if (t0 >= t1) return;

  // Tile cursor: tiles of a sequence run KV head by KV head, 16 pages each;
  // the first tile is found by search, later ones by stepping (no division
  // per tile).
  struct Cursor {
    int b, h, p0, P, L;
  };
  auto seek = [&](long long ti, Cursor& c) {
    int lo = 0, hi = a.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= ti) lo = mid; else hi = mid;
    }
    c.b = lo;
    c.P = seq_pages(a.seq_lens, c.b, a.S, a.max_pages, &c.L);
    const int tpu = (c.P + kTile - 1) / kTile;
    const int r = static_cast<int>(ti - prefix[c.b]);
    c.h = r / tpu;
    c.p0 = (r - c.h * tpu) * kTile;
  };
  auto step = [&](Cursor& c) {
    c.p0 += kTile;
    if (c.p0 >= c.P) {
      c.p0 = 0;
      if (++c.h == a.Hkv) {
        c.h = 0;
        do {
          ++c.b;
          c.P = c.b < a.batch ? seq_pages(a.seq_lens, c.b, a.S, a.max_pages, &c.L) : 1;
        } while (c.P == 0);
      }
    }
  };
  auto load_ids = [&](const Cursor& c) -> int {
    const int n = min(kTile, c.P - c.p0);
    return lane < n ? a.page_table[static_cast<size_t>(c.b) * a.max_pages + c.p0 + lane] : -1;
  };

  uint32_t bfrag[2 * KP][NT][2];
  int cur_unit = -1;
  float* my_tile = ctile + warp * 16 * 24;
  Cursor cur;
  seek(t0, cur);
  int ids = load_ids(cur);
  for (long long ti = t0; ti < t1; ++ti) {
    const int b = cur.b, h = cur.h, p0 = cur.p0, L = cur.L;
    const int n = min(kTile, cur.P - p0);
    const int unit = b * a.Hkv + h;
    if (!waited && p0 + n == cur.P) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      waited = true;
    }
    const int id_lo = __shfl_sync(0xffffffffu, ids, g), id_hi = __shfl_sync(0xffffffffu, ids, g + 8);
    const bool ok_lo = g < n && id_lo >= 0 && id_lo < a.num_phys;
    const bool ok_hi = g + 8 < n && id_hi >= 0 && id_hi < a.num_phys;
    if ((g < n && !ok_lo) || (g + 8 < n && !ok_hi)) raise_flag(EKV_EFLAG_BAD_PAGE);
    // bit r: row r of the tile exists and has a valid page
    const unsigned int live_mask = __ballot_sync(0xffffffffu, lane < n && ids >= 0 && ids < a.num_phys);
    const unsigned char* hrows = static_cast<const unsigned char*>(a.rows) + static_cast<size_t>(h) * a.num_phys * ROW;
    const uint4* row_lo = reinterpret_cast<const uint4*>(hrows + static_cast<size_t>(ok_lo ? id_lo : 0) * ROW) + t;
    const uint4* row_hi = reinterpret_cast<const uint4*>(hrows + static_cast<size_t>(ok_hi ? id_hi : 0) * ROW) + t;
    uint4 va[KP], vb[KP];
#pragma unroll
    for (int c = 0; c < KP; ++c) {
      va[c] = ok_lo ? __ldcs(row_lo + 4 * c) : make_uint4(0, 0, 0, 0);
      vb[c] = ok_hi ? __ldcs(row_hi + 4 * c) : make_uint4(0, 0, 0, 0);
    }
    // next tile's page ids travel while this tile's rows do
    if (ti + 1 < t1) {
      step(cur);
      ids = load_ids(cur);
    }
    if (unit != cur_unit) {
      cur_unit = unit;
      const bf16* qb = static_cast<const bf16*>(a.q) + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(h) * G) * D;
      auto coef = [&](int col, int k) -> float {
        const bool lo_half = k < D;
        const int j = lo_half ? k : k - D;
        if constexpr (!GAUSS) {
          if (col >= G) return 0.f;
          const float v = __bfloat162float(qb[col * D + j]);
          return lo_half ? fmaxf(v, 0.f) : fminf(v, 0.f);
        } else {
          if (lo_half) return col < G ? __bfloat162float(qb[col * D + j]) : 0.f;
          if (col >= 2 * G) return 0.f;
          const float v = __bfloat162float(qb[(col >> 1) * D + j]);
          float hi, lo;
          split_bf16(v * v, hi, lo);
          return (col & 1) ? lo : hi;
        }
      };
#pragma unroll
      for (int ks = 0; ks < 2 * KP; ++ks)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int col = nt * 8 + g;
          const int k0 = 32 * (ks >> 1) + 8 * t + 4 * (ks & 1);
          bfrag[ks][nt][0] = pack_bf16_exact(coef(col, k0), coef(col, k0 + 1));
          bfrag[ks][nt][1] = pack_bf16_exact(coef(col, k0 + 2), coef(col, k0 + 3));
        }
    }
    // acc: the score, or the Gaussian means; acv: the Gaussian variances
    float acc[NT][4], acv[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = acv[nt][e] = 0.f;
#pragma unroll
    for (int c = 0; c < KP; ++c) {
      const uint32_t f0[4] = {va[c].x, vb[c].x, va[c].y, vb[c].y};
      const uint32_t f1[4] = {va[c].z, vb[c].z, va[c].w, vb[c].w};
      const bool var_half = GAUSS && c >= KP / 2;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (var_half) {
          mma_bf16(acv[nt], f0, bfrag[2 * c][nt][0], bfrag[2 * c][nt][1]);
          mma_bf16(acv[nt], f1, bfrag[2 * c + 1][nt][0], bfrag[2 * c + 1][nt][1]);
        } else if (!GAUSS || nt * 8 < G) {  // a Gaussian mean tile holds G ≤ 8 columns
          mma_bf16(acc[nt], f0, bfrag[2 * c][nt][0], bfrag[2 * c][nt][1]);
          mma_bf16(acc[nt], f1, bfrag[2 * c + 1][nt][0], bfrag[2 * c + 1][nt][1]);
        }
      }
    }
    if constexpr (!GAUSS) {
      float m_lo = -INFINITY, m_hi = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int c0 = nt * 8 + 2 * t;
        if (c0 < G) { m_lo = fmaxf(m_lo, acc[nt][0]); m_hi = fmaxf(m_hi, acc[nt][2]); }
        if (c0 + 1 < G) { m_lo = fmaxf(m_lo, acc[nt][1]); m_hi = fmaxf(m_hi, acc[nt][3]); }
      }
      m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 1));
      m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 1));
      m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, 2));
      m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, 2));
      if (t == 0) {
        float* urow = a.ub + static_cast<size_t>(unit) * a.max_pages + p0;
        if (g < n) urow[g] = ok_lo ? a.scale * m_lo : -INFINITY;
        if (g + 8 < n) urow[g + 8] = ok_hi ? a.scale * m_hi : -INFINITY;
      }
    } else {
      // per row: 8 mean columns (G ≤ 8 used), then 16 variance columns
      constexpr int TW = 24, VOFF = 8;
      static_assert(G <= 8 && VOFF + 8 * NT <= TW, "tile columns");
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int c0 = nt * 8 + 2 * t;
        if (nt == 0) {
          my_tile[g * TW + c0] = acc[0][0];
          my_tile[g * TW + c0 + 1] = acc[0][1];
          my_tile[(g + 8) * TW + c0] = acc[0][2];
          my_tile[(g + 8) * TW + c0 + 1] = acc[0][3];
        }
        my_tile[g * TW + VOFF + c0] = acv[nt][0];
        my_tile[g * TW + VOFF + c0 + 1] = acv[nt][1];
        my_tile[(g + 8) * TW + VOFF + c0] = acv[nt][2];
        my_tile[(g + 8) * TW + VOFF + c0 + 1] = acv[nt][3];
      }
      __syncwarp();
      for (int pr = lane; pr < 16 * G; pr += 32) {
        const int r = pr / G, hh = pr % G;
        if (r < n) {
          const int p = p0 + r;
          const float m = a.scale * my_tile[r * TW + hh];
          const float s2 = my_tile[r * TW + VOFF + 2 * hh] + my_tile[r * TW + VOFF + 2 * hh + 1];
          const float sd = a.scale * sqrtf(fmaxf(s2, 0.f));
          const float nv = static_cast<float>(min(a.S, L - p * a.S));
          float mu = a.am1 * m, sg = a.am1 * sd, hat = a.am1 * (m + sd * sqrtf(2.f * logf(nv)));
          if (!((live_mask >> r) & 1u)) mu = hat = -INFINITY, sg = 0.f;
          const size_t o = (static_cast<size_t>(unit) * G + hh) * a.max_pages + p;
          a.gws.mu[o] = mu;
          a.gws.sig[o] = sg;
          a.gws.hat[o] = hat;
        }
      }
      __syncwarp();
    }
  }
}


template <typename T, int D, int G, bool GAUSS>
cudaError_t launch_stream(const StreamArgs& a, cudaStream_t st) {
  if constexpr (UseMma<T, G, GAUSS>::value) {
    const size_t smem = kDirectWarps * 16 * 24 * sizeof(float) + (static_cast<size_t>(a.batch) + 1) * sizeof(int);
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(meta_direct_kernel<D, G, GAUSS>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    const cudaError_t le_ = launch_k(meta_direct_kernel<D, G, GAUSS>, sm_count() * DirectOcc<D, G, GAUSS>::value,
                                     32 * kDirectWarps, smem, st, a);
    if (le_ != cudaSuccess) return le_;
    return cudaGetLastError();
  }
  constexpr int ROWP = 2 * D * static_cast<int>(sizeof(T)) + 16;
  constexpr int rows = StageRows<ROWP>::value;
  const size_t smem = static_cast<size_t>(kStages) * rows * ROWP + 2 * kStages * sizeof(uint64_t) +
                      kStages * rows + kConsumers * 16 * 24 * sizeof(float) +
                      kIdAhead * rows * sizeof(int) + kIdAhead * sizeof(int4) +
                      (static_cast<size_t>(a.batch) + 1) * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(meta_stream_kernel<T, D, G, GAUSS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le_ = launch_k(meta_stream_kernel<T, D, G, GAUSS>, sm_count() * kCtasPerSm, kStreamThreads, smem, st, a);
    if (le_ != cudaSuccess) return le_;
  }
  return cudaGetLastError();
}

template <typename T, bool GAUSS>
cudaError_t dispatch_stream(const ekv_cache& c, const StreamArgs& a, int G, cudaStream_t st) {
#define EKV_STREAM_CASE(DD, GG) \
  if (c.head_dim == DD && G == GG) return launch_stream<T, DD, GG, GAUSS>(a, st);
  EKV_STREAM_CASE(128, 1) EKV_STREAM_CASE(128, 2) EKV_STREAM_CASE(128, 4)
  EKV_STREAM_CASE(128, 8) EKV_STREAM_CASE(128, 16)
  EKV_STREAM_CASE(64, 1) EKV_STREAM_CASE(64, 2) EKV_STREAM_CASE(64, 4) EKV_STREAM_CASE(64, 8)
#undef EKV_STREAM_CASE
  if constexpr (!GAUSS) {
    if (c.head_dim == 64 && G == 16) return launch_stream<T, 64, 16, false>(a, st);
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
  a.batch = s.batch;
  return a;
}

}  // namespace

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t launch_score(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq, float scale,
                         float* ub, cudaStream_t st, int after_append) {
  StreamArgs a = base_args(c, s, q, Hq, scale);
  a.defer_wait = after_append;
  a.rows = c.box;
  a.ub = ub;
  const int G = Hq / c.num_kv_heads;
  return c.dtype == EKV_BF16 ? dispatch_stream<bf16, false>(c, a, G, st)
                             : dispatch_stream<float, false>(c, a, G, st);
}

cudaError_t launch_gauss_stats(const ekv_cache& c, const ekv_seqs& s, const void* q, int Hq,
                               float scale, float alpha, const GaussWs& ws, cudaStream_t st,
                               int after_append) {
  StreamArgs a = base_args(c, s, q, Hq, scale);
  a.defer_wait = after_append;
  a.rows = c.mom;
  a.gws = ws;
  a.am1 = alpha - 1.0f;
  const int G = Hq / c.num_kv_heads;
  return c.dtype == EKV_BF16 ? dispatch_stream<bf16, true>(c, a, G, st)
                             : dispatch_stream<float, true>(c, a, G, st);
}

}  // namespace ekv
