// Block-denoise attention (one denoiser layer).
//
// "Architecture" / "Generation Process" of the gist.science summary: every
// block query attends to the frozen context tower's K/V of the same layer and
// to the block's own S keys, with no mask inside the block.  One softmax
// runs over [block keys ; context keys] per query row (the order of keys does
// not change a softmax).
//
// Work units and schedule.  A unit is a KV head g of sequence b and a query
// tile of up to 256 rows (block positions x the G query heads sharing g,
// packed so one K/V tile feeds every row).  Its keys form tiles of 128: tile
// 0 holds the block's own S keys, tiles 1.. the context keys.  All units'
// tiles are laid end to end (attn_plan_kernel writes the prefix sums from the
// device-side context lengths) and cut into one contiguous range per CTA of a
// persistent grid (one CTA per SM), so every SM streams the same number of
// K/V tiles whatever the batch and the lengths.  A CTA walks its range as
// segments, one per unit it touches, and writes per segment the unnormalised
// O and the row maxima and sums; the CTA that completes a unit (a per-unit
// counter) merges the unit's segments into the bf16 output.
//
// Inside a CTA the unit's rows form two 128-row halves, each an M=128
// tcgen05 tile with its own TMEM columns.  Per 128-key tile i and half h:
//   S_h  = Q_h . K(i)^T       (TMEM, 128 fp32 columns; Q and K from smem)
//   P_h  = exp2(S_h*c - m)    (bf16 pairs, written back over S_h's columns)
//   O_h += P_h . V(i)         (TMEM accumulator; A = P_h read from TMEM)
// so P never goes through shared memory.  Roles (20 warps):
//   warp 0     TMA for Q and K (3-slot ring);
//   warp 1     TMEM owner; TMA for V (2-slot ring) and zeroing of the V rows
//              past the last valid key that a 16-key MMA step still reads;
//   warps 2, 3 MMA issue for half 0 / half 1: P_h(i).V(i) as soon as
//              softmax h has written P_h(i), then S_h(i+1) into the same
//              columns (tcgen05 MMAs of one thread execute in issue order);
//   warps 4-11 / 12-19  softmax of half 0 / half 1.  Warp w serves the 32
//              rows of its TMEM lane quarter (w % 4) and one 64-key column
//              half of every tile; the two warps of a row swap partial row
//              maxima through shared memory.  Thread = row: no shuffles.
// The two softmax groups take turns tile by tile, so the tensor core runs
// one half's MMAs during the other half's softmax.  An eighth of the
// exponentials run on the FMA pipe (exp2_poly) to offload the MUFU unit.
// The running max only moves (and O is rescaled in TMEM) when it grows by
// more than 2^8; the final O / l is exact for any stale max.
#include <math.h>

#include "tt_ptx.cuh"

// Timeline hooks for instrumented builds; empty in the library build.
#ifndef TT_TRACE_POINT
#define TT_TRACE_POINT(cond, slot, t)
#endif

namespace tt {

namespace {

constexpr int kKSlots = 3, kVSlots = 2;       // K and V ring depths
constexpr uint32_t kKVSub = kAttnBN * 128;    // 128 keys x 64 dh bf16 (128-byte rows) = 16 KB
constexpr uint32_t kQSub = 16384;             // 128 rows x 64 dh bf16
constexpr float kRescaleThreshold = 8.0f;     // log2 units
// Context K/V tiles this far ahead of the one being loaded into shared
// memory are prefetched into L2 (0: none), so that more of the stream is in
// flight than the rings hold.
#ifndef TT_ATTN_L2_AHEAD
#define TT_ATTN_L2_AHEAD 0
#endif
constexpr int kL2Ahead = TT_ATTN_L2_AHEAD;

struct AttnSmem {
  uint32_t q, k, v, bars, xchg, total;
};

__host__ __device__ inline AttnSmem attn_layout(int dh, int halves) {
  AttnSmem L;
  const uint32_t nsub = (uint32_t)dh / 64;
  L.q = 0;
  L.k = L.q + (uint32_t)halves * nsub * kQSub;
  L.v = L.k + kKSlots * nsub * kKVSub;
  L.bars = L.v + kVSlots * nsub * kKVSub;  // 28 mbarriers, then control words
  L.xchg = L.bars + 256;      // row-max exchange: [half][quarter][column half][lane] bf16
  L.total = L.xchg + 1024;
  return L;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// A unit's context length, clamped to [0, L_cap] (an out-of-range length is
// reported by the plan kernel).
__device__ __forceinline__ int unit_len(const AttnArgs& a, int b) {
  return min(max(a.ctx_len[b], 0), a.L_cap);
}

struct UnitInfo {
  int b, g, qt, L;
};
__device__ __forceinline__ UnitInfo unit_info(const AttnArgs& a, int u) {
  UnitInfo ui;
  const int pair = u / a.n_qtiles;
  ui.qt = u - pair * a.n_qtiles;
  ui.b = pair / a.Hkv;
  ui.g = pair - ui.b * a.Hkv;
  ui.L = unit_len(a, ui.b);
  return ui;
}

struct TileInfo {
  int is_blk, key0, nvalid;
};
// Local tile tl of a unit: 0 is the block's own S keys, tl >= 1 the context
// keys (tl-1)*128 .. min(tl*128, L) - 1.
__device__ __forceinline__ TileInfo tile_info(int tl, int L, int S) {
  TileInfo ti;
  if (tl == 0) {
    ti.is_blk = 1;
    ti.key0 = 0;
    ti.nvalid = S;
  } else {
    ti.is_blk = 0;
    ti.key0 = (tl - 1) * kAttnBN;
    ti.nvalid = min(kAttnBN, L - ti.key0);
  }
  return ti;
}

// The CTA's range [lo, hi) of the tile sequence and its segments, walked the
// same way by every role: segment = (unit u, local tiles [a, b)).
struct SegWalk {
  const int* start;
  int t, hi, u;
  __device__ __forceinline__ bool next(int& unit, int& a, int& b) {
    if (t >= hi) return false;
    const int s0 = start[u], s1 = start[u + 1];
    unit = u;
    a = t - s0;
    b = min(hi, s1) - s0;
    t = min(hi, s1);
    ++u;
    return true;
  }
};

// 2^x on the FMA pipe, to take part of the exponentials off the MUFU unit
// (Cody-Waite style range reduction): n = round(x) by the float trick of
// adding 1.5 * 2^23 (whose low mantissa bits then hold n), f = x - n in
// [-1/2, 1/2], 2^f by a cubic fitted for relative error over that interval
// (Chebyshev-node least squares with Lawson reweighting towards minimax; max
// relative error 7.5e-5, far below the bf16 rounding P goes through), and
// 2^n added to the exponent field with integer arithmetic - no conversion
// instructions, which would run at the MUFU rate.  x <= -126 gives 0.
__device__ __forceinline__ float exp2_poly(float x) {
  const float xc = fmaxf(x, -126.0f);
  const float t = xc + 12582912.0f;  // 1.5 * 2^23
  const float f = xc - (t - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(0.0551716685295105f, f, 0.2426111251115799f), f,
                            0.6932609677314758f),
                       f, 0.9999280571937561f);
  const int e = (__float_as_int(t) - 0x4B400000) << 23;
  const float r = __int_as_float(__float_as_int(p) + e);
  return x > -126.0f ? r : 0.f;
}

// TMEM load of 16 columns (32x32b shape: a thread's lane, consecutive columns).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// P for 16 score columns as 8 bf16 pairs, written in place: pair j/2 goes to
// sv[j] (the registers of S it came from are dead by then); the last pair
// on the FMA pipe.
__device__ __forceinline__ void exp_slice16(uint32_t (&sv)[16], float c, float m, float& s0,
                                            float& s1) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float x0 = fmaf(__uint_as_float(sv[j]), c, -m);
    const float x1 = fmaf(__uint_as_float(sv[j + 1]), c, -m);
    float p0, p1;
    if (j == 14) {
      p0 = exp2_poly(x0);
      p1 = exp2_poly(x1);
    } else {
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    s0 += p0;
    s1 += p1;
    sv[j] = pack_bf16x2(p0, p1);
  }
}
// TMEM store of the 8 pairs exp_slice16 left in the even registers.
__device__ __forceinline__ void tmem_st8_even(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[2]), "r"(r[4]), "r"(r[6]), "r"(r[8]), "r"(r[10]), "r"(r[12]),
               "r"(r[14])
               : "memory");
}

// Tiles per unit and their exclusive prefix sums (one CTA), then the first
// unit of every CTA of the attention's persistent grid.
__global__ void __launch_bounds__(1024) attn_plan_kernel(const AttnArgs a) {
  griddep_launch();
  griddep_wait();
  __shared__ int warp_tot[32];
  __shared__ int running;
  int* start = a.tile_start;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) running = 0;
  __syncthreads();
  for (int base = 0; base < a.units; base += blockDim.x) {
    const int u = base + tid;
    int n = 0;
    if (u < a.units) {
      const int b = u / (a.Hkv * a.n_qtiles);
      const int L = a.ctx_len[b];
      if ((L < 0 || L > a.L_cap) && (u % (a.Hkv * a.n_qtiles)) == 0)
        atomicCAS(a.err, 0, (int)TT_ERR_INVALID_ARG);
      n = 1 + (min(max(L, 0), a.L_cap) + kAttnBN - 1) / kAttnBN;
    }
    int incl = n;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
      before += w < warp ? warp_tot[w] : 0;
      total += warp_tot[w];
    }
    if (u < a.units) start[u] = running + before + incl - n;
    __syncthreads();
    if (tid == 0) running += total;
    __syncthreads();
  }
  if (tid == 0) start[a.units] = running;
  __syncthreads();
  // CTA c's range starts at lo(c) = c*T/P; the unit holding lo(c) is its
  // first.  Unit u holds [s0, s1), i.e. the CTAs ceil(s0*P/T) ..
  // ceil(s1*P/T) - 1.
  const long long T = running, P = a.n_ctas;
  for (int u = tid; u < a.units; u += blockDim.x) {
    const long long s0 = start[u], s1 = start[u + 1];
    const long long c0 = (s0 * P + T - 1) / T, c1 = (s1 * P + T - 1) / T;
    for (long long c = c0; c < c1 && c < P; ++c) a.first_unit[c] = u;
    // the fix-up's view: the CTAs holding the unit's first and last tiles,
    // and how many CTAs hold a tile of it (with fewer tiles than CTAs every
    // non-empty CTA holds one tile)
    const int cf = (int)(((s0 + 1) * P - 1) / T), cl = (int)((s1 * P - 1) / T);
    a.unit_ctas[u] = make_int4(cf, cl, T >= P ? cl - cf + 1 : (int)(s1 - s0), T >= P ? 1 : 0);
    a.unit_done[u] = 0;
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKb,
                const __grid_constant__ CUtensorMap tmVb, const AttnArgs a) {
  griddep_launch();
  griddep_wait();
  extern __shared__ uint8_t smem_raw[];
  if (a.active != nullptr && *a.active == 0) return;
  const int cta = blockIdx.x;
  // HBM is mostly idle while this kernel runs on an L2-resident context:
  // warm L2 with the head of the W rows the vocabulary GEMM's CTA `cta`
  // streams first.  Issued by the softmax warps (threads 128..), which
  // wait for the first S anyway, not by the producers.
  if (a.pf_bytes > 0 && threadIdx.x >= 128) {
    const int r1 = min(a.pf_rows, (cta + 1) * a.pf_tile);
    for (int r = cta * a.pf_tile + (int)threadIdx.x - 128; r < r1; r += (int)blockDim.x - 128)
      prefetch_l2_bulk(a.pf_base + (long long)r * a.pf_ld, (uint32_t)a.pf_bytes);
  }
  const long long T = a.tile_start[a.units];
  const int lo = (int)((long long)cta * T / a.n_ctas);
  const int hi = (int)((long long)(cta + 1) * T / a.n_ctas);
  const int u0 = a.first_unit[cta];
  if (lo >= hi) {
    // An empty range (fewer tiles than CTAs) lies inside the CTA range of at
    // most one unit, the one holding tile lo, and only when that unit starts
    // before lo: its slot gets an empty record (no keys, sum 0), so the
    // merges can take every CTA of a unit's range as present.
    if (!a.fixup && a.tile_start[u0] < lo)
      for (int i = threadIdx.x; i < 256; i += blockDim.x)
        *reinterpret_cast<float4*>(a.part_ml + ((size_t)(u0 + cta) * 256 + i) * 4) =
            make_float4(-INFINITY, 0.f, 0.f, 0.f);
    return;
  }
  const int dh = a.dh, nsub = dh / 64;
  const int halves = a.halves;

  const AttnSmem SL = attn_layout(dh, halves);
  uint8_t* base = align1024(smem_raw);
  uint8_t* sQ = base + SL.q;
  uint8_t* sK = base + SL.k;
  uint8_t* sV = base + SL.v;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SL.bars);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;        // one arrival per half: its last S of the segment done
  uint64_t* k_full = q_empty + 1;        // [kKSlots]
  uint64_t* k_empty = k_full + kKSlots;  // [kKSlots], one arrival per half
  uint64_t* v_full = k_empty + kKSlots;  // [kVSlots]
  uint64_t* v_empty = v_full + kVSlots;  // [kVSlots], one arrival per half
  uint64_t* v_ready = v_empty + kVSlots; // [kVSlots]: V landed and its padding rows cleared
  uint64_t* s_full = v_ready + kVSlots;  // [half]: S_h(i) ready (and P_h(i-1).V done)
  uint64_t* p_full = s_full + 2;         // [half]: P_h(i) written, O_h corrected
  uint64_t* o_full = p_full + 2;         // [half]: the segment's last P.V done
  uint64_t* xbar = o_full + 2;           // [half][quarter]: both column halves' values written
  uint64_t* seg_done = xbar + 8;         // every softmax thread has written its partial
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(seg_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* n_merge = abort_flag + 1;         // units this CTA completed (merged at the end)
  int* merge_list = a.merge_list + (size_t)cta * a.merge_cap;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // TMEM: S/P of half h at column h*128, then O of half h at halves*128 + h*dh.
  const uint32_t tmem_need = halves * (kAttnBN + dh);
  const uint32_t tmem_cols = tmem_need <= 128 ? 128u : tmem_need <= 256 ? 256u : 512u;
  const uint32_t tO0 = halves * kAttnBN;

  // Rows of a half that the Q box does not cover must be finite (they only
  // produce output rows that are discarded): clear Q once when the box is
  // short; the boxes of later segments rewrite only the covered rows.
  if (a.rows_per_half < 128) {
    uint4* q4 = reinterpret_cast<uint4*>(sQ);
    const int n4 = halves * nsub * (int)kQSub / 16;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) q4[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, halves);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], halves);
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], halves);
      mbar_init(&v_ready[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&s_full[h], 1);
      mbar_init(&p_full[h], 256);
      mbar_init(&o_full[h], 1);
    }
    for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], 64);
    mbar_init(seg_done, halves * 256);
    *abort_flag = 0;
    *n_merge = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  SegWalk walk{a.tile_start, lo, hi, u0};
  int su, sa, sb;  // current segment: unit, local tiles [sa, sb)

  if (warp == 0) {
    // ------------------------------------------------ TMA producer: Q, K
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKc);
      prefetch_tmap(&tmKb);
      if (kL2Ahead > 0) prefetch_tmap(&tmVc);
      const uint64_t pol_kv = a.kv_keep ? policy_evict_last() : policy_evict_first();
      int kt = 0, qi = 0;
      bool ok = true;
      while (ok && walk.next(su, sa, sb)) {
        const UnitInfo ui = unit_info(a, su);
        // Q of this segment's unit, once both halves' last S of the
        // previous segment has read the buffer
        if (qi > 0 && !mbar_wait(q_empty, (uint32_t)(qi - 1) & 1u, a.err, abort_flag,
                                 WHERE_ATTN_PRODUCER))
          break;
        const int pos0 = ui.qt * halves * a.s_per_half;
        mbar_arrive_expect_tx(q_full, (uint32_t)(halves * nsub * a.rows_per_half * 128));
        for (int h = 0; h < halves; ++h)
          for (int xh = 0; xh < nsub; ++xh)
            tma_load_3d(sQ + (h * nsub + xh) * kQSub, &tmQ, q_full, xh * 64, ui.g * a.G,
                        ui.b * a.S + pos0 + h * a.s_per_half);
        ++qi;
        const int row_base = (ui.b * a.Hkv + ui.g) * a.L_cap;
        for (int tl = sa; tl < sb; ++tl, ++kt) {
          const TileInfo ti = tile_info(tl, ui.L, a.S);
          const uint32_t bytes = ti.is_blk ? (uint32_t)(nsub * a.S * 128) : (uint32_t)(nsub * kKVSub);
          const int ks = kt % kKSlots;
          if (!mbar_wait(&k_empty[ks], ((uint32_t)(kt / kKSlots) & 1u) ^ 1u, a.err, abort_flag,
                         WHERE_ATTN_PRODUCER)) {
            ok = false;
            break;
          }
          if (kL2Ahead > 0 && tl + kL2Ahead < sb) {
            const TileInfo ta = tile_info(tl + kL2Ahead, ui.L, a.S);
            for (int xh = 0; xh < nsub; ++xh) {
              tma_prefetch_l2_2d(&tmKc, xh * 64, row_base + ta.key0);
              tma_prefetch_l2_2d(&tmVc, xh * 64, row_base + ta.key0);
            }
          }
          uint8_t* dk = sK + ks * nsub * kKVSub;
          mbar_arrive_expect_tx(&k_full[ks], bytes);
          for (int xh = 0; xh < nsub; ++xh) {
            if (ti.is_blk)
              tma_load_3d(dk + xh * kKVSub, &tmKb, &k_full[ks], xh * 64, ui.g, ui.b * a.S);
            else
              tma_load_2d_hint(dk + xh * kKVSub, &tmKc, &k_full[ks], xh * 64,
                               row_base + ti.key0, pol_kv);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- TMA producer: V; V padding
    // Lane 0 streams V (own loop, so K never waits for a V slot).  The P.V
    // MMA reads V rows up to the next multiple of 16 past the valid keys;
    // those rows hold whatever the cache holds beyond the context (or an
    // older tile's rows), and P is zero there but 0 * NaN is NaN, so the
    // warp zeroes them before either half's MMA may read the slot.  V(t) is
    // issued before V(t-1) is cleaned, keeping two loads in flight.
    if (lane == 0) {
      prefetch_tmap(&tmVc);
      prefetch_tmap(&tmVb);
    }
    const uint64_t pol_kv = a.kv_keep ? policy_evict_last() : policy_evict_first();
    int vt = 0, prev_nv = -1;
    bool ok = true;
    auto clean = [&](int t, int nvalid) -> bool {
      const int vs = t % kVSlots;
      const bool landed = mbar_wait(&v_full[vs], (uint32_t)(t / kVSlots) & 1u, a.err, abort_flag,
                                    WHERE_ATTN_MMA);
      if (!__all_sync(0xffffffffu, landed)) return false;
      const int pad = ((nvalid + 15) & ~15) - nvalid;
      if (pad > 0) {
        for (int xh = 0; xh < nsub; ++xh) {
          uint4* dst = reinterpret_cast<uint4*>(sV + (vs * nsub + xh) * kKVSub + nvalid * 128);
          for (int i = lane; i < pad * 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_ready[vs]);
      return true;
    };
    while (ok && walk.next(su, sa, sb)) {
      const UnitInfo ui = unit_info(a, su);
      const int row_base = (ui.b * a.Hkv + ui.g) * a.L_cap;
      for (int tl = sa; tl < sb; ++tl, ++vt) {
        const TileInfo ti = tile_info(tl, ui.L, a.S);
        int good = 1;
        if (lane == 0) {
          const uint32_t bytes =
              ti.is_blk ? (uint32_t)(nsub * a.S * 128) : (uint32_t)(nsub * kKVSub);
          const int vs = vt % kVSlots;
          good = mbar_wait(&v_empty[vs], ((uint32_t)(vt / kVSlots) & 1u) ^ 1u, a.err, abort_flag,
                           WHERE_ATTN_PRODUCER);
          if (good) {
            uint8_t* dv = sV + vs * nsub * kKVSub;
            mbar_arrive_expect_tx(&v_full[vs], bytes);
            for (int xh = 0; xh < nsub; ++xh) {
              if (ti.is_blk)
                tma_load_3d(dv + xh * kKVSub, &tmVb, &v_full[vs], xh * 64, ui.g, ui.b * a.S);
              else
                tma_load_2d_hint(dv + xh * kKVSub, &tmVc, &v_full[vs], xh * 64,
                                 row_base + ti.key0, pol_kv);
            }
          }
        }
        if (__shfl_sync(0xffffffffu, good, 0) == 0 || (vt > 0 && !clean(vt - 1, prev_nv))) {
          ok = false;
          break;
        }
        prev_nv = ti.nvalid;
      }
    }
    if (ok && vt > 0) clean(vt - 1, prev_nv);
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------- MMA issuer of half (warp-2)
    const int h = warp - 2;
    if (h < halves) {
      const uint32_t idS = idesc_bf16(128, kAttnBN, false, false);
      const uint32_t idO = idesc_bf16(128, dh, false, true);
      const uint32_t tS = tmem + h * kAttnBN, tOh = tmem + tO0 + h * dh;
      // Descriptor bases; each MMA adds a compile-time offset (the start
      // address field is address >> 4 in the low bits, and no smem address
      // carries out of it), so an issue costs a few instructions.
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ) + h * nsub * kQSub, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = sdesc_sw128(smem_u32(sV), kKVSub, 1024);
      int kt = 0, pt = 0, qi = 0;  // tiles, turns, segments
      bool ok = true;
      while (ok && walk.next(su, sa, sb)) {
        const UnitInfo ui = unit_info(a, su);
        const int n = sb - sa;
        // S_h = Q_h . K(local tile i)^T; the K slot is free once the MMA has
        // read it (both halves), Q once the segment's last S has.
        auto scores = [&](int i) -> bool {
          const int ks = (kt + i) % kKSlots;
          if (!mbar_wait(&k_full[ks], (uint32_t)((kt + i) / kKSlots) & 1u, a.err, abort_flag,
                         WHERE_ATTN_MMA))
            return false;
          tc_fence_after();
          if (lane == 0) {
            const uint64_t dK = dK0 + (uint64_t)((uint32_t)(ks * nsub) * (kKVSub >> 4));
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              if (kk < dh / 16)
                umma_bf16_ss(tS, dQ + (uint64_t)(((kk >> 2) * kQSub + (kk & 3) * 32) >> 4),
                             dK + (uint64_t)(((kk >> 2) * kKVSub + (kk & 3) * 32) >> 4), idS,
                             kk > 0);
            }
            umma_commit(&s_full[h]);
            umma_commit(&k_empty[ks]);
            if (i == n - 1) umma_commit(q_empty);
          }
          __syncwarp();
          return true;
        };
        ok = mbar_wait(q_full, (uint32_t)qi & 1u, a.err, abort_flag, WHERE_ATTN_MMA);
        if (ok) tc_fence_after();
        if (ok) ok = scores(0);
        for (int i = 0; ok && i < n; ++i, ++pt) {
          // O_h += P_h(i) . V(i), once warp 1 has cleared V(i)'s padding rows
          const int vs = (kt + i) % kVSlots;
          if (!mbar_wait(&p_full[h], (uint32_t)pt & 1u, a.err, abort_flag, WHERE_ATTN_MMA) ||
              !mbar_wait(&v_ready[vs], (uint32_t)((kt + i) / kVSlots) & 1u, a.err, abort_flag,
                         WHERE_ATTN_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int ksteps = (tile_info(sa + i, ui.L, a.S).nvalid + 15) >> 4;
          if (lane == 0) {
            // V as an MN-major operand: 64-wide dh blocks kKVSub apart, 8-key
            // groups 1 KB apart, 16 keys (2 KB) per MMA.  P of keys 0..63
            // sits in columns 0..31, of keys 64..127 in columns 64..95.
            const uint64_t dV = dV0 + (uint64_t)((uint32_t)(vs * nsub) * (kKVSub >> 4));
#pragma unroll
            for (int kk = 0; kk < kAttnBN / 16; ++kk) {
              if (kk < ksteps)
                umma_bf16_ts(tOh, tS + kk * 8 + (kk >= 4 ? 32 : 0),
                             dV + (uint64_t)(kk * (2048 >> 4)), idO, (i > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&v_empty[vs]);
          }
          __syncwarp();
          if (i + 1 < n) ok = scores(i + 1);
        }
        if (ok && lane == 0) umma_commit(&o_full[h]);
        __syncwarp();
        kt += n;
        ++qi;
      }
    }
  } else {
    // ---------------------------------------------------- softmax groups
    // Half wg is served by warps 4+8*wg .. 11+8*wg.  Warp w owns the rows of
    // its TMEM lane quarter q = w % 4 and one column half ch of every tile
    // (S columns ch*64..+63, the O columns ch*dh/2..+dh/2-1), so two warps
    // per SMSP share a row: they swap their partial row maxima through
    // shared memory (as bf16, rounded the same way on both sides, so both
    // use the identical stabiliser) and add their row sums at the end of
    // each segment.
    const int wg = (warp - 4) >> 3;
    const int ch = ((warp - 4) >> 2) & 1;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    if (wg < halves) {
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      const uint32_t tS = tmem + wg * kAttnBN + lane_off + ch * 64;
      const int dh2 = dh / 2;
      const uint32_t tO = tmem + tO0 + wg * dh + lane_off + ch * dh2;
      uint16_t* xch = reinterpret_cast<uint16_t*>(base + SL.xchg) + (wg * 4 + q) * 64;
      uint64_t* xb = &xbar[wg * 4 + q];
      const float c = a.scale_log2;
      int pt = 0, qi = 0, xp = 0, sdp = 0;  // turns, segments, exchanges, fix-ups
      bool ok = true;
      // The row's partial max of this warp's 64 columns -> the row max
      // (both column halves, rounded to bf16 the same way on both sides).
      auto exchange = [&](float part, float& mx) -> bool {
        xch[ch * 32 + lane] = bf16_bits(part);
        mbar_arrive(xb);
        if (!mbar_wait(xb, (uint32_t)xp & 1u, a.err, abort_flag, WHERE_ATTN_SOFTMAX)) return false;
        ++xp;
        mx = fmaxf(bf16_value(xch[lane]), bf16_value(xch[32 + lane]));
        return true;
      };
      // O_h to a new max before P_h(i).V adds to it (s_full also covered
      // P_h(i-1).V, so O_h is settled).
      auto rescale_o = [&](float alpha) {
#pragma unroll 1
        for (int c0 = 0; c0 < dh2; c0 += 16) {
          uint32_t o[16];
          tmem_ld16(tO + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st16(tO + c0, o);
        }
      };
      while (ok && walk.next(su, sa, sb)) {
        const int Lu = unit_len(a, (su / a.n_qtiles) / a.Hkv);
        float m = -INFINITY, l = 0.f;
        for (int i = sa; i < sb; ++i, ++pt) {
          // The two halves take turns (0 on tile t, then 1 on tile t, then 0
          // on t+1): the tensor core runs one half's P.V and next S while
          // the other half's softmax runs, instead of both halves contending
          // for MUFU and then both waiting for their MMAs.  p_full[other]
          // marks the other half's turn done.
          if (halves == 2 && (wg == 1 || pt > 0) &&
              !mbar_wait(&p_full[wg ^ 1], (uint32_t)(wg == 1 ? pt : pt - 1) & 1u, a.err,
                         abort_flag, WHERE_ATTN_SOFTMAX)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&s_full[wg], (uint32_t)pt & 1u, a.err, abort_flag,
                         WHERE_ATTN_SOFTMAX)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nvt = tile_info(i, Lu, a.S).nvalid;
          {
            // Columns past the valid keys (the block's own tile, or the last
            // tile of a unit) are overwritten with -inf (nothing to the max,
            // exp2 gives 0 on both exponential paths), then the row max, then
            // the exponentials.
            const int nv = nvt - ch * 64;
            if (nv < 64) {
#pragma unroll 1
              for (int c0 = max(nv, 0) & ~15; c0 < 64; c0 += 16) {
                uint32_t v[16];
                if (c0 < nv) {
                  tmem_ld16(tS + c0, v);
                  tmem_wait_ld();
#pragma unroll
                  for (int j = 0; j < 16; ++j) v[j] = c0 + j < nv ? v[j] : __float_as_uint(-INFINITY);
                } else {
#pragma unroll
                  for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(-INFINITY);
                }
                tmem_st16(tS + c0, v);
              }
              tmem_wait_st();
            }
            float mc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) mc[k] = -INFINITY;
            uint32_t sa32[32];
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
              tmem_ld32(tS + c0, sa32);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; j += 2)
                mc[(j >> 1) & 3] =
                    fmax3(mc[(j >> 1) & 3], __uint_as_float(sa32[j]), __uint_as_float(sa32[j + 1]));
            }
            uint32_t s_even[16], s_odd[16];
            tmem_ld16(tS, s_even);  // the first sub-slice is read while the maxima are swapped
            float mx;
            if (!exchange(fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]), mx)) {
              tmem_wait_ld();
              ok = false;
              break;
            }
            const float mxs = mx * c;
            const bool need = mxs > m + kRescaleThreshold;
            float alpha = 1.f;
            if (need) {
              alpha = ex2(m - mxs);
              m = mxs;
            }
            float e0 = 0.f, e1 = 0.f;
            tmem_wait_ld();
#pragma unroll 1
            for (int k = 0; k < 4; k += 2) {
              tmem_ld16(tS + 16 * (k + 1), s_odd);
              exp_slice16(s_even, c, m, e0, e1);
              tmem_st8_even(tS + 8 * k, s_even);
              tmem_wait_ld();
              if (k == 0) tmem_ld16(tS + 32, s_even);
              exp_slice16(s_odd, c, m, e0, e1);
              tmem_st8_even(tS + 8 * (k + 1), s_odd);
              if (k == 0) tmem_wait_ld();
            }
            l = l * alpha + (e0 + e1);
            // a segment's first P.V overwrites O, so its first tile needs none
            if (i > sa && __any_sync(0xffffffffu, need)) rescale_o(alpha);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&p_full[wg]);
        }
        if (!ok) break;
        // The segment's partial, each column half writing its own: its half
        // of the unnormalised O row (tile-major [slot][dh/4][256 rows][4],
        // so a warp's float4 store covers 32 consecutive rows, 512
        // contiguous bytes), the running max (log2 units, the same in both
        // halves) and its row sum: [slot][256 rows] x (m, l of column half
        // 0, l of column half 1, unused).
        if (!mbar_wait(&o_full[wg], (uint32_t)qi & 1u, a.err, abort_flag, WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int slot = su + cta;
        const bool valid = r < a.rows_per_half;
        const int r256 = wg * 128 + r;
        float* po = a.part_o + (size_t)slot * dh * 256 + (size_t)r256 * 4;
        for (int c0 = 0; c0 < dh2; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c0, o);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              *reinterpret_cast<float4*>(po + (size_t)((ch * dh2 + c0) / 4 + v) * 1024) =
                  make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                              __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
          }
        }
        if (valid) {
          float* ml = a.part_ml + ((size_t)slot * 256 + r256) * 4;
          if (ch == 0) {
            ml[0] = m;
            ml[1] = l;
          } else {
            ml[2] = l;
          }
        }
        ++qi;
        // With the fix-up, the CTA that completes a unit (the last of its
        // segments to finish, by a per-unit counter) merges it once its
        // whole range is done.
        if (!a.fixup) continue;
        __threadfence();
        mbar_arrive(seg_done);
        if (warp == 4 && lane == 0 &&
            mbar_wait(seg_done, (uint32_t)sdp & 1u, a.err, abort_flag, WHERE_ATTN_SOFTMAX) &&
            atomicAdd(a.unit_done + su, 1) == a.unit_ctas[su].z - 1) {
          a.unit_done[su] = 0;  // ready for the next launch
          merge_list[(*n_merge)++] = su;  // at most merge_cap: a unit's last tile is in range
        }
        ++sdp;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
  // Fix-up of the units this CTA completed: all threads, item = (query row,
  // 16-column chunk) with consecutive threads on consecutive rows (so the
  // tile-major partial reads are coalesced), o = sum_i 2^(m_i - m*) O_i /
  // sum_i 2^(m_i - m*) l_i over the unit's segments, two segments' loads in
  // flight, bf16 output.
  if (!a.fixup || *n_merge == 0 || *abort_flag) return;
  __threadfence();
  // With fewer tiles than CTAs (unit_ctas.w == 0) some CTAs of a unit's range
  // held no tile and wrote nothing.
  auto ran = [&](const int4& uc, int c) {
    return uc.w != 0 || (long long)c * T / a.n_ctas < (long long)(c + 1) * T / a.n_ctas;
  };
  const int nrows = halves * 128, items = nrows * (dh / 16);
  for (int mi = 0; mi < *n_merge; ++mi) {
    const int u = merge_list[mi];
    const int4 uc = a.unit_ctas[u];
    const UnitInfo ui = unit_info(a, u);
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
      const int r256 = it % nrows, c16 = (it / nrows) * 16;
      const int wg = r256 >> 7, r = r256 & 127;
      if (r >= a.rows_per_half) continue;
      float mrun = -INFINITY, den = 0.f;
      for (int cc = uc.x; cc <= uc.y; ++cc) {
        if (!ran(uc, cc)) continue;
        const float4 q4 = __ldcg(
            reinterpret_cast<const float4*>(a.part_ml + ((size_t)(u + cc) * 256 + r256) * 4));
        const float li = q4.y + q4.z;
        if (!(li > 0.f)) continue;
        if (q4.x > mrun) {
          den = mrun == -INFINITY ? 0.f : den * ex2(mrun - q4.x);
          mrun = q4.x;
        }
        den += li * ex2(q4.x - mrun);
      }
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.f;
      for (int cc = uc.x; cc <= uc.y; cc += 2) {
        float4 o4[2][4];
        float w[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int c = cc + k;
          w[k] = 0.f;
          if (c <= uc.y && ran(uc, c)) {
            const size_t sl = (size_t)(u + c);
            const float msl = __ldcg(a.part_ml + (sl * 256 + r256) * 4);
            w[k] = msl > -INFINITY ? ex2(msl - mrun) : 0.f;
            const float* pos = a.part_o + sl * dh * 256 + (size_t)r256 * 4;
#pragma unroll
            for (int v = 0; v < 4; ++v)
              o4[k][v] = __ldcg(reinterpret_cast<const float4*>(pos + (size_t)(c16 / 4 + v) * 1024));
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v) o4[k][v] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            acc[4 * v] += w[k] * o4[k][v].x;
            acc[4 * v + 1] += w[k] * o4[k][v].y;
            acc[4 * v + 2] += w[k] * o4[k][v].z;
            acc[4 * v + 3] += w[k] * o4[k][v].w;
          }
        }
      }
      const float inv = 1.f / den;
      const int s = ui.qt * halves * a.s_per_half + wg * a.s_per_half + r / a.G;
      const int head = ui.g * a.G + r % a.G;
      uint16_t* dst = a.out + (size_t)(ui.b * a.S + s) * a.ldo + head * dh + c16;
      uint4 w0, w1;
      w0.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      w0.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      w0.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      w0.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      w1.x = pack_bf16x2(acc[8] * inv, acc[9] * inv);
      w1.y = pack_bf16x2(acc[10] * inv, acc[11] * inv);
      w1.z = pack_bf16x2(acc[12] * inv, acc[13] * inv);
      w1.w = pack_bf16x2(acc[14] * inv, acc[15] * inv);
      reinterpret_cast<uint4*>(dst)[0] = w0;
      reinterpret_cast<uint4*>(dst)[1] = w1;
    }
  }
}

// Thread per (unit, query row, 4-column group): combine the unit's segment
// partials,
//   O = sum_i 2^(m_i - m*) O_i / sum_i 2^(m_i - m*) l_i,
// in one pass (running max, rescaled sums), four segments' loads in flight
// before any is used.  Consecutive threads take consecutive rows, so the
// tile-major partial reads are coalesced.
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnArgs a) {
  griddep_launch();
  griddep_wait();
  if (a.active != nullptr && *a.active == 0) return;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int ngrp = a.dh / 4;
  const int row256 = (int)(i & 255);
  const int grp = (int)((i >> 8) % ngrp);
  const int u = (int)((i >> 8) / ngrp);
  if (u >= a.units) return;
  const int h = row256 >> 7, r = row256 & 127;
  if (h >= a.halves || r >= a.rows_per_half) return;
  const int qt = u % a.n_qtiles, pair = u / a.n_qtiles;
  const int b = pair / a.Hkv, g = pair % a.Hkv;
  const int4 uc = a.unit_ctas[u];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f, mrun = -INFINITY;
  for (int c0 = uc.x; c0 <= uc.y; c0 += 4) {
    float2 ml[4];
    float4 o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool in = c0 + k <= uc.y;
      const size_t slot = (size_t)u + c0 + k;
      if (in) {
        const float4 q4 = *reinterpret_cast<const float4*>(a.part_ml + (slot * 256 + row256) * 4);
        ml[k] = make_float2(q4.x, q4.y + q4.z);
      } else {
        ml[k] = make_float2(-INFINITY, 0.f);
      }
      o[k] = in ? *reinterpret_cast<const float4*>(a.part_o + ((slot * ngrp + grp) * 256 + row256) * 4)
                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!(ml[k].y > 0.f)) continue;
      if (ml[k].x > mrun) {
        const float sc = mrun == -INFINITY ? 0.f : ex2(mrun - ml[k].x);
        den *= sc;
        acc.x *= sc;
        acc.y *= sc;
        acc.z *= sc;
        acc.w *= sc;
        mrun = ml[k].x;
      }
      const float w = ex2(ml[k].x - mrun);
      den += w * ml[k].y;
      acc.x += w * o[k].x;
      acc.y += w * o[k].y;
      acc.z += w * o[k].z;
      acc.w += w * o[k].w;
    }
  }
  const float inv = 1.f / den;
  const int s = qt * a.halves * a.s_per_half + h * a.s_per_half + r / a.G;
  const int head = g * a.G + r % a.G;
  uint16_t* dst = a.out + (size_t)(b * a.S + s) * a.ldo + head * a.dh + grp * 4;
  uint2 wv;
  wv.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  wv.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(dst) = wv;
}

}  // namespace

size_t attn_smem_bytes(int dh, int halves) { return attn_layout(dh, halves).total + 1024; }

cudaError_t launch_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKc, const CUtensorMap& tmVc,
                        const CUtensorMap& tmKb, const CUtensorMap& tmVb, const AttnArgs& a,
                        cudaStream_t st) {
  const size_t smem = attn_smem_bytes(a.dh, a.halves);
  cudaError_t e =
      cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(attn_kernel, dim3(a.n_ctas), dim3(kAttnThreads), smem, st, tmQ, tmKc, tmVc, tmKb,
                  tmVb, a);
}

cudaError_t launch_attn_plan(const AttnArgs& a, cudaStream_t st) {
  return launch_k(attn_plan_kernel, dim3(1), dim3(1024), 0, st, a);
}

cudaError_t launch_attn_merge(const AttnArgs& a, cudaStream_t st) {
  const long long threads = (long long)a.units * 256 * (a.dh / 4);
  const int blocks = (int)((threads + 255) / 256);
  return launch_k(attn_merge_kernel, dim3(blocks), dim3(256), 0, st, a);
}

}  // namespace tt
