// Block-denoise attention (one denoiser layer), split over context keys.
//
// "Architecture" / "Generation Process" of the gist.science summary: every
// block query attends to the frozen context tower's K/V of the same layer and
// to the block's own S keys, with no mask inside the block.  This kernel runs
// one softmax over [context keys ; block keys] per query row.
//
// Work unit (one CTA): a KV head g of sequence b, a query tile of up to 256
// rows (block positions x the G query heads sharing g, packed so one K/V
// tile feeds every row) and a contiguous split of the context keys; split 0
// also owns the block's own S keys.  The rows form two 128-row halves, each
// an M=128 tcgen05 tile with its own TMEM columns.  Per 128-key tile i and
// half h:
//   S_h  = Q_h . K(i)^T       (TMEM, 128 fp32 columns; Q and K from smem)
//   P_h  = exp2(S_h*c - m)    (bf16 pairs, written back into S_h's columns)
//   O_h += P_h . V(i)         (TMEM accumulator; A = P_h read from TMEM)
// so P never goes through shared memory.  Roles (20 warps):
//   warp 0     TMA for Q and K (3-slot ring);
//   warps 1, 2 MMA issue for half 0 / half 1: P_h(i).V(i) as soon as
//              softmax h has written P_h(i), then S_h(i+1) into the same
//              columns (tcgen05 MMAs of one thread execute in issue order);
//   warp 3     TMEM owner; TMA for V (2-slot ring) and zeroing of the V rows
//              past the last valid key that a 16-key MMA step still reads;
//   warps 4-11 / 12-19  softmax of half 0 / half 1.  Warp w serves the 32
//              rows of its TMEM lane quarter (w % 4) and one 64-key column
//              half of every tile; the two warps of a row swap partial row
//              maxima through shared memory.  Thread = row: no shuffles.
// The two softmax groups take turns tile by tile, so the tensor core runs
// one half's MMAs during the other half's softmax.  An eighth of the
// exponentials run on the FMA pipe (exp2_poly) to offload the MUFU unit.
// The running max only moves (and O is rescaled in TMEM) when it grows by
// more than 2^8; the final O / l is exact for any stale max.  With one split
// the CTA writes the bf16 output; otherwise (unnormalised O, max, sum)
// partials for a merge kernel.
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

struct AttnSmem {
  uint32_t q, k, v, bars, xchg, total;
};

__host__ __device__ inline AttnSmem attn_layout(int dh, int halves) {
  AttnSmem L;
  const uint32_t nsub = (uint32_t)dh / 64;
  L.q = 0;
  L.k = L.q + (uint32_t)halves * nsub * kQSub;
  L.v = L.k + kKSlots * nsub * kKVSub;
  L.bars = L.v + kVSlots * nsub * kKVSub;
  L.xchg = L.bars + 256;      // row-max exchange: [half][quarter][column half][lane] bf16
  L.total = L.xchg + 1024;
  return L;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

struct TileInfo {
  int is_blk, key0, nvalid;
};
__device__ __forceinline__ TileInfo tile_info(int t, int has_blk, int k0, int k1, int S) {
  TileInfo ti;
  if (has_blk && t == 0) {
    ti.is_blk = 1;
    ti.key0 = 0;
    ti.nvalid = S;
  } else {
    ti.is_blk = 0;
    ti.key0 = k0 + (t - has_blk) * kAttnBN;
    ti.nvalid = min(kAttnBN, k1 - ti.key0);
  }
  return ti;
}

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
// TMEM store of 8 columns, same shape.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}
// P for 16 score columns as 8 bf16 pairs; the last pair on the FMA pipe.
__device__ __forceinline__ void exp_slice16(const uint32_t (&sv)[16], float c, float m, float& s0,
                                            float& s1, uint32_t (&pk)[8]) {
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
    pk[j >> 1] = pack_bf16x2(p0, p1);
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
  const int split = blockIdx.x, qt = blockIdx.y, pair = blockIdx.z;
  const int b = pair / a.Hkv, g = pair % a.Hkv;
  int L = a.ctx_len[b];
  if (L < 0 || L > a.L_cap) {
    if (threadIdx.x == 0) atomicCAS(a.err, 0, (int)TT_ERR_INVALID_ARG);
    L = min(max(L, 0), a.L_cap);
  }
  const int k0 = split == 0 ? 0 : a.first + (split - 1) * a.chunk;
  const int k1 = min(split == 0 ? a.first : k0 + a.chunk, L);
  const int n_ctx_tiles = k1 > k0 ? (k1 - k0 + kAttnBN - 1) / kAttnBN : 0;
  const int has_blk = split == 0 ? 1 : 0;
  const int n_tiles = has_blk + n_ctx_tiles;
  const int unit = (pair * a.n_qtiles + qt) * a.n_splits + split;
  const int dh = a.dh, nsub = dh / 64;
  const int halves = a.halves;

  if (n_tiles == 0) {  // an empty split (only split > 0): contributes nothing
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
      a.part_ml[((size_t)unit * 256 + i) * 2 + 0] = -INFINITY;
      a.part_ml[((size_t)unit * 256 + i) * 2 + 1] = 0.f;
    }
    return;
  }

  const AttnSmem SL = attn_layout(dh, halves);
  uint8_t* base = align1024(smem_raw);
  uint8_t* sQ = base + SL.q;
  uint8_t* sK = base + SL.k;
  uint8_t* sV = base + SL.v;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SL.bars);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;         // [kKSlots]
  uint64_t* k_empty = k_full + kKSlots;  // [kKSlots], one arrival per half
  uint64_t* v_full = k_empty + kKSlots;  // [kVSlots]
  uint64_t* v_empty = v_full + kVSlots;  // [kVSlots], one arrival per half
  uint64_t* v_ready = v_empty + kVSlots; // [kVSlots]: V landed and its padding rows cleared
  uint64_t* s_full = v_ready + kVSlots;  // [half]: S_h(i) ready (and P_h(i-1).V done)
  uint64_t* p_full = s_full + 2;         // [half]: P_h(i) written, O_h corrected
  uint64_t* o_full = p_full + 2;         // [half]
  uint64_t* xbar = o_full + 2;           // [half][quarter]: both column halves' row maxima written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 8);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // TMEM: S/P of half h at column h*128, then O of half h at halves*128 + h*dh.
  const uint32_t tmem_need = halves * (kAttnBN + dh);
  const uint32_t tmem_cols = tmem_need <= 128 ? 128u : tmem_need <= 256 ? 256u : 512u;
  const uint32_t tO0 = halves * kAttnBN;

  // Rows of a half that the Q box does not cover must be finite (they only
  // produce output rows that are discarded): clear Q when the box is short.
  if (a.rows_per_half < 128) {
    uint4* q4 = reinterpret_cast<uint4*>(sQ);
    const int n4 = halves * nsub * (int)kQSub / 16;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) q4[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
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
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 3) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int pos0 = qt * halves * a.s_per_half;  // first block position of this query tile

  if (warp < 4) {
    if (warp == 0) {
      // ------------------------------------------------ TMA producer: Q, K
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmKc);
        const uint64_t pol_kv = a.kv_keep ? policy_evict_last() : policy_evict_first();
        mbar_arrive_expect_tx(q_full, (uint32_t)(halves * nsub * a.rows_per_half * 128));
        for (int h = 0; h < halves; ++h)
          for (int xh = 0; xh < nsub; ++xh)
            tma_load_3d(sQ + (h * nsub + xh) * kQSub, &tmQ, q_full, xh * 64, g * a.G,
                        b * a.S + pos0 + h * a.s_per_half);
        const int row_base = (b * a.Hkv + g) * a.L_cap;
        for (int t = 0; t < n_tiles; ++t) {
          const TileInfo ti = tile_info(t, has_blk, k0, k1, a.S);
          const uint32_t bytes = ti.is_blk ? (uint32_t)(nsub * a.S * 128) : (uint32_t)(nsub * kKVSub);
          const int ks = t % kKSlots;
          if (!mbar_wait(&k_empty[ks], ((uint32_t)(t / kKSlots) & 1u) ^ 1u, a.err, abort_flag,
                         WHERE_ATTN_PRODUCER))
            break;
          TT_TRACE_POINT(true, 0, t);
          uint8_t* dk = sK + ks * nsub * kKVSub;
          mbar_arrive_expect_tx(&k_full[ks], bytes);
          for (int xh = 0; xh < nsub; ++xh) {
            if (ti.is_blk)
              tma_load_3d(dk + xh * kKVSub, &tmKb, &k_full[ks], xh * 64, g, b * a.S);
            else
              tma_load_2d_hint(dk + xh * kKVSub, &tmKc, &k_full[ks], xh * 64, row_base + ti.key0,
                               pol_kv);
          }
        }
      }
    } else if (warp == 1 || warp == 2) {
      // ------------------------------------------- MMA issuer of half (warp-1)
      const int h = warp - 1;
      if (h < halves) {
        const uint32_t idS = idesc_bf16(128, kAttnBN, false, false);
        const uint32_t idO = idesc_bf16(128, dh, false, true);
        const uint32_t tS = tmem + h * kAttnBN, tOh = tmem + tO0 + h * dh;
        // Descriptor bases; each MMA adds a compile-time offset (the start
        // address field is address >> 4 in the low bits, and no smem address
        // carries out of it), so an issue costs a few instructions: the
        // issuing warp shares its SMSP with busy softmax warps.
        const uint64_t dQ = sdesc_sw128(smem_u32(sQ) + h * nsub * kQSub, 16, 1024);
        const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t dV0 = sdesc_sw128(smem_u32(sV), kKVSub, 1024);
        // S_h(t) = Q_h . K(t)^T
        auto scores = [&](int t) -> bool {
          const int ks = t % kKSlots;
          if (!mbar_wait(&k_full[ks], (uint32_t)(t / kKSlots) & 1u, a.err, abort_flag,
                         WHERE_ATTN_MMA))
            return false;
          if (h == 0) TT_TRACE_POINT(lane == 0, 1, t);
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
          }
          __syncwarp();
          if (h == 0) TT_TRACE_POINT(lane == 0, 2, t);
          return true;
        };
        // O_h += P_h(t) . V(t), once warp 3 has cleared V(t)'s padding rows
        auto pv = [&](int t) -> bool {
          if (!mbar_wait(&p_full[h], (uint32_t)t & 1u, a.err, abort_flag, WHERE_ATTN_MMA))
            return false;
          TT_TRACE_POINT(lane == 0, 3 + h, t);
          const int vs = t % kVSlots;
          const int ksteps = (tile_info(t, has_blk, k0, k1, a.S).nvalid + 15) >> 4;
          if (!mbar_wait(&v_ready[vs], (uint32_t)(t / kVSlots) & 1u, a.err, abort_flag,
                         WHERE_ATTN_MMA))
            return false;
          tc_fence_after();
          if (lane == 0) {
            // V as an MN-major operand: 64-wide dh blocks kKVSub apart, 8-key
            // groups 1 KB apart, 16 keys (2 KB) per MMA.  P of keys 0..63
            // sits in columns 0..31, of keys 64..127 in columns 64..95.
            const uint64_t dV = dV0 + (uint64_t)((uint32_t)(vs * nsub) * (kKVSub >> 4));
#pragma unroll
            for (int kk = 0; kk < kAttnBN / 16; ++kk) {
              if (kk < ksteps)
                umma_bf16_ts(tOh, tS + kk * 8 + (kk >= 4 ? 32 : 0), dV + (uint64_t)(kk * (2048 >> 4)),
                             idO, (t > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&v_empty[vs]);
          }
          __syncwarp();
          return true;
        };
        bool ok = mbar_wait(q_full, 0, a.err, abort_flag, WHERE_ATTN_MMA);
        if (ok) tc_fence_after();
        if (ok) ok = scores(0);
        for (int t = 0; ok && t < n_tiles; ++t) {
          ok = pv(t);
          if (ok && t + 1 < n_tiles) ok = scores(t + 1);
        }
        if (lane == 0) umma_commit(&o_full[h]);
        __syncwarp();
      }
    } else {
      // ------------------------------------------- TMA producer: V; V padding
      // Lane 0 streams V (own loop, so K never waits for a V slot).  The
      // P.V MMA reads V rows up to the next multiple of 16 past the valid
      // keys; those rows hold whatever the cache holds beyond the context (or
      // an older tile's rows), and P is zero there but 0 * NaN is NaN, so the
      // warp zeroes them before either half's MMA may read the slot.  V(t) is
      // issued before V(t-1) is cleaned, keeping two loads in flight.
      if (lane == 0) prefetch_tmap(&tmVc);
      const uint64_t pol_kv = a.kv_keep ? policy_evict_last() : policy_evict_first();
      const int row_base = (b * a.Hkv + g) * a.L_cap;
      for (int t = 0; t <= n_tiles; ++t) {
        if (t < n_tiles) {
          int good = 1;
          if (lane == 0) {
            const TileInfo ti = tile_info(t, has_blk, k0, k1, a.S);
            const uint32_t bytes =
                ti.is_blk ? (uint32_t)(nsub * a.S * 128) : (uint32_t)(nsub * kKVSub);
            const int vs = t % kVSlots;
            good = mbar_wait(&v_empty[vs], ((uint32_t)(t / kVSlots) & 1u) ^ 1u, a.err,
                             abort_flag, WHERE_ATTN_PRODUCER);
            if (good) {
              uint8_t* dv = sV + vs * nsub * kKVSub;
              mbar_arrive_expect_tx(&v_full[vs], bytes);
              for (int xh = 0; xh < nsub; ++xh) {
                if (ti.is_blk)
                  tma_load_3d(dv + xh * kKVSub, &tmVb, &v_full[vs], xh * 64, g, b * a.S);
                else
                  tma_load_2d_hint(dv + xh * kKVSub, &tmVc, &v_full[vs], xh * 64,
                                   row_base + ti.key0, pol_kv);
              }
            }
          }
          if (__shfl_sync(0xffffffffu, good, 0) == 0) break;
        }
        if (t >= 1) {
          const int tc = t - 1, vs = tc % kVSlots;
          const bool landed = mbar_wait(&v_full[vs], (uint32_t)(tc / kVSlots) & 1u, a.err,
                                        abort_flag, WHERE_ATTN_MMA);
          if (!__all_sync(0xffffffffu, landed)) break;
          const int nvalid = tile_info(tc, has_blk, k0, k1, a.S).nvalid;
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
        }
      }
    }
  } else {
    // ---------------------------------------------------- softmax groups
    // Half wg is served by warps 4+8*wg .. 11+8*wg.  Warp w owns the rows of
    // its TMEM lane quarter q = w % 4 and one column half ch of every tile
    // (S columns ch*64..+63, the O columns ch*dh/2..+dh/2-1), so two warps
    // per SMSP share a row: they swap their partial row maxima through
    // shared memory (as bf16, rounded the same way on both sides, so both
    // use the identical stabiliser) and add their row sums at the end.
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
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        // The two halves take turns (0 on tile t, then 1 on tile t, then 0
        // on t+1): the tensor core runs one half's P.V and next S while the
        // other half's softmax runs, instead of both halves contending for
        // MUFU and then both waiting for their MMAs.  p_full[other] marks
        // the other half's tile done.
        if (halves == 2 && (wg == 1 || t > 0) &&
            !mbar_wait(&p_full[wg ^ 1], (uint32_t)(wg == 1 ? t : t - 1) & 1u, a.err, abort_flag,
                       WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&s_full[wg], (uint32_t)t & 1u, a.err, abort_flag, WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        TT_TRACE_POINT(lane == 0 && q == 0 && ch == 0, 5 + 5 * wg, t);
        tc_fence_after();
        // Columns past the valid keys (the block's own tile, or the last
        // tile of a split) are overwritten with -inf: nothing to the max,
        // exp2 gives 0 on both exponential paths.
        const int nv = tile_info(t, has_blk, k0, k1, a.S).nvalid - ch * 64;
        if (nv < 64) {
          for (int c0 = max(nv, 0) & ~31; c0 < 64; c0 += 32) {
            uint32_t v[32];
            if (c0 < nv) {
              tmem_ld32(tS + c0, v);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = c0 + j < nv ? v[j] : __float_as_uint(-INFINITY);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(-INFINITY);
            }
            tmem_st32(tS + c0, v);
          }
          tmem_wait_st();
        }
        float mc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) mc[k] = -INFINITY;
        uint32_t sa[32];
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          tmem_ld32(tS + c0, sa);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 2)
            mc[(j >> 1) & 3] = fmax3(mc[(j >> 1) & 3], __uint_as_float(sa[j]), __uint_as_float(sa[j + 1]));
        }
        const float part = fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
        // The first exponential sub-slice is read while the maxima are swapped.
        uint32_t s_even[16], s_odd[16];  // sub-slices 0, 2 and 1, 3
        tmem_ld16(tS, s_even);
        // One buffer suffices: a warp writes tile t+1's value only after
        // S(t+1), which needs its partner's P(t), written after the read.
        xch[ch * 32 + lane] = bf16_bits(part);
        mbar_arrive(xb);
        if (!mbar_wait(xb, (uint32_t)t & 1u, a.err, abort_flag, WHERE_ATTN_SOFTMAX)) {
          tmem_wait_ld();
          ok = false;
          break;
        }
        const float mx = fmaxf(bf16_value(xch[lane]), bf16_value(xch[32 + lane]));
        TT_TRACE_POINT(lane == 0 && q == 0 && ch == 0, 6 + 5 * wg, t);
        const float mxs = mx * c;
        const bool need = mxs > m + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2(m - mxs);
          m = mxs;
        }
        l *= alpha;
        TT_TRACE_POINT(lane == 0 && q == 0 && ch == 0, 7 + 5 * wg, t);
        // P = exp2(S*c - m) as bf16 pairs, written into this warp's own S
        // columns (slice i's 16 pair columns over slice i's first half, read
        // already); one pair in eight on the FMA pipe.
        float s0 = 0.f, s1 = 0.f;
        tmem_wait_ld();
        // Four 16-column sub-slices; the next one's load is in flight while
        // this one's exponentials run.  P of sub-slice k goes to columns
        // [8k, 8k+8), which sub-slices already read cover.
#pragma unroll 1
        for (int k = 0; k < 4; k += 2) {
          uint32_t pk[8];
          tmem_ld16(tS + 16 * (k + 1), s_odd);
          exp_slice16(s_even, c, m, s0, s1, pk);
          tmem_st8(tS + 8 * k, pk);
          tmem_wait_ld();
          if (k == 0) tmem_ld16(tS + 32, s_even);
          exp_slice16(s_odd, c, m, s0, s1, pk);
          tmem_st8(tS + 8 * (k + 1), pk);
          if (k == 0) tmem_wait_ld();
        }
        l += s0 + s1;
        // O_h to the new max before P_h(t).V adds to it (s_full also
        // covered P_h(t-1).V, so O_h is settled).
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          for (int c0 = 0; c0 < dh2; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st32(tO + c0, o);
          }
        }
        TT_TRACE_POINT(lane == 0 && q == 0 && ch == 0, 8 + 5 * wg, t);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[wg]);
        TT_TRACE_POINT(lane == 0 && q == 0 && ch == 0, 9 + 5 * wg, t);
      }
      // Column half 1 hands its row sum to column half 0, which writes the
      // whole row.  o_full (the last P.V done) implies both warps have read
      // the last tile's maxima, so the buffer is free.
      if (ok) ok = mbar_wait(&o_full[wg], 0, a.err, abort_flag, WHERE_ATTN_SOFTMAX);
      if (ok) {
        if (ch == 1) {
          const uint32_t lb = __float_as_uint(l);
          xch[lane] = (uint16_t)(lb & 0xffffu);
          xch[32 + lane] = (uint16_t)(lb >> 16);
        }
        mbar_arrive(xb);
        ok = mbar_wait(xb, (uint32_t)n_tiles & 1u, a.err, abort_flag, WHERE_ATTN_SOFTMAX);
      }
      if (ok && ch == 0) {
        l += __uint_as_float((uint32_t)xch[lane] | ((uint32_t)xch[32 + lane] << 16));
        tc_fence_after();
        const uint32_t tOr = tmem + tO0 + wg * dh + lane_off;  // the whole O row
        const bool valid = r < a.rows_per_half;
        const int s = pos0 + wg * a.s_per_half + r / a.G;
        const int head = g * a.G + r % a.G;
        if (a.n_splits == 1) {
          const float inv = 1.f / l;
          uint16_t* dst = a.out + (size_t)(b * a.S + s) * a.ldo + head * dh;
          for (int c0 = 0; c0 < dh; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tOr + c0, o);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                *reinterpret_cast<uint4*>(dst + c0 + 8 * v) = w;
              }
            }
          }
        } else {
          // Partial O is tile-major, [unit][dh/4][256 rows][4]: a warp's
          // float4 store covers 32 consecutive rows, 512 contiguous bytes.
          const int r256 = wg * 128 + r;
          const size_t prow_i = (size_t)unit * 256 + r256;
          float* po = a.part_o + (size_t)unit * dh * 256 + (size_t)r256 * 4;
          for (int c0 = 0; c0 < dh; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tOr + c0, o);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                *reinterpret_cast<float4*>(po + (size_t)(c0 / 4 + v) * 1024) =
                    make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
            }
          }
          if (valid) {
            a.part_ml[prow_i * 2 + 0] = m;
            a.part_ml[prow_i * 2 + 1] = l;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Thread per (query row, 4-column group): combine the splits' partials,
//   O = sum_i 2^(m_i - m*) O_i / sum_i 2^(m_i - m*) l_i,
// in one pass over the splits (running max, rescaled sums), four splits'
// loads in flight before any is used.  Consecutive threads take consecutive
// rows, so the tile-major partial reads are coalesced.  An empty split
// (l = 0, O never written) is skipped by selection.
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnArgs a) {
  griddep_launch();
  griddep_wait();
  if (a.active != nullptr && *a.active == 0) return;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int ngrp = a.dh / 4;
  const int row256 = (int)(i & 255);
  const int grp = (int)((i >> 8) % ngrp);
  const int pq = (int)((i >> 8) / ngrp);  // pair * n_qtiles + qt
  if (pq >= a.B * a.Hkv * a.n_qtiles) return;
  const int h = row256 >> 7, r = row256 & 127;
  if (h >= a.halves || r >= a.rows_per_half) return;
  const int pair = pq / a.n_qtiles, qt = pq % a.n_qtiles;
  const int b = pair / a.Hkv, g = pair % a.Hkv;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f, mrun = -INFINITY;
  for (int sp0 = 0; sp0 < a.n_splits; sp0 += 4) {
    float2 ml[4];
    float4 o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t pt = (size_t)pq * a.n_splits + sp0 + k;
      const bool in = sp0 + k < a.n_splits;
      ml[k] = in ? *reinterpret_cast<const float2*>(a.part_ml + (pt * 256 + row256) * 2)
                 : make_float2(-INFINITY, 0.f);
      o[k] = in ? *reinterpret_cast<const float4*>(a.part_o + ((pt * ngrp + grp) * 256 + row256) * 4)
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
  dim3 grid(a.n_splits, a.n_qtiles, a.B * a.Hkv);
  return launch_k(attn_kernel, grid, dim3(kAttnThreads), smem, st, tmQ, tmKc, tmVc, tmKb, tmVb, a);
}

cudaError_t launch_attn_merge(const AttnArgs& a, cudaStream_t st) {
  const long long threads = (long long)a.B * a.Hkv * a.n_qtiles * 256 * (a.dh / 4);
  const int blocks = (int)((threads + 255) / 256);
  return launch_k(attn_merge_kernel, dim3(blocks), dim3(256), 0, st, a);
}

}  // namespace tt
