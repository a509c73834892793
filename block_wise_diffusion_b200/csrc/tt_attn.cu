// Block-denoise attention (one denoiser layer), split over context keys.
//
// "Architecture" / "Generation Process" of the gist.science summary: every
// block query attends to the frozen context tower's K/V of the same layer and
// to the block's own S keys, with no mask inside the block.  This kernel runs
// one softmax over [context keys ; block keys] per query row.
//
// Work unit (one CTA): a KV head g of sequence b, a query tile of up to 256
// rows (block positions x the G query heads sharing g, packed so one K/V tile
// feeds every row), and a contiguous split of the context keys.  Split 0 also
// owns the block's own S keys.  Rows are split into two 128-row halves, each
// an M=128 tcgen05 tile with its own TMEM accumulators:
//   S_h  = Q_h . K^T   (TMEM, 64 fp32 columns)    P_h = exp2(S_h*c - m) (smem, bf16)
//   O_h += P_h . V     (TMEM, dh fp32 columns)
// Warp 0 streams 64-key K/V tiles by TMA (4-stage ring), warp 1 issues the
// MMAs in the order S0 S1 | PV0 S0' | PV1 S1' ... so each softmax warpgroup
// works while the tensor core serves the other half.  Warps 2-5 and 6-9 are
// the softmax warpgroups: one thread per row (TMEM lane), so row max and row
// sum need no shuffles.  The running max is only moved (and O rescaled in
// TMEM) when it grows by more than 2^8, which keeps exp2 in range while
// skipping most rescales; the final O / l is exact for any stale max.
// Partials (unnormalised O, max, sum) are merged by attn_merge_kernel when a
// head is split; with one split the CTA writes the bf16 result itself.
#include <math.h>

#include "tt_ptx.cuh"

// Timeline hooks for instrumented builds; empty in the library build.
#ifndef TT_TRACE_POINT
#define TT_TRACE_POINT(cond, slot, t)
#endif

namespace tt {

namespace {

constexpr uint32_t kSub = 8192;     // one 64-key x 64-dh bf16 sub-tile (128-byte rows)
constexpr uint32_t kQSub = 16384;   // one 128-row x 64-dh bf16 sub-tile
constexpr uint32_t kPHalf = 16384;  // 128 rows x 64 keys bf16
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnSmem {
  uint32_t q, k, v, p, bars, total;
};

__host__ __device__ inline AttnSmem attn_layout(int dh, int halves) {
  AttnSmem L;
  const uint32_t nsub = (uint32_t)dh / 64;
  L.q = 0;
  L.k = L.q + (uint32_t)halves * nsub * kQSub;
  L.v = L.k + kAttnStages * nsub * kSub;
  L.p = L.v + kAttnStages * nsub * kSub;
  L.bars = L.p + 2 * kPHalf;
  L.total = L.bars + 256;
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

// Row max over the valid columns of a 64-key score tile (thread = row).
template <bool kFull>
__device__ __forceinline__ float row_max(const uint32_t (&sr)[64], int nvalid) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 64; j += 4) {
    const float v0 = __uint_as_float(sr[j]), v1 = __uint_as_float(sr[j + 1]);
    const float v2 = __uint_as_float(sr[j + 2]), v3 = __uint_as_float(sr[j + 3]);
    if (kFull) {
      m0 = fmaxf(m0, v0);
      m1 = fmaxf(m1, v1);
      m2 = fmaxf(m2, v2);
      m3 = fmaxf(m3, v3);
    } else {
      m0 = (j < nvalid) ? fmaxf(m0, v0) : m0;
      m1 = (j + 1 < nvalid) ? fmaxf(m1, v1) : m1;
      m2 = (j + 2 < nvalid) ? fmaxf(m2, v2) : m2;
      m3 = (j + 3 < nvalid) ? fmaxf(m3, v3) : m3;
    }
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// p = exp2(s*c - m) for the valid columns (0 elsewhere), packed to bf16
// pairs; returns the row sum of p.
template <bool kFull>
__device__ __forceinline__ float exp_pack(const uint32_t (&sr)[64], int nvalid, float c, float m,
                                          uint32_t (&pk)[32]) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int j = 0; j < 64; j += 2) {
    float p0 = ex2(fmaf(__uint_as_float(sr[j]), c, -m));
    float p1 = ex2(fmaf(__uint_as_float(sr[j + 1]), c, -m));
    if (!kFull) {
      p0 = (j < nvalid) ? p0 : 0.f;
      p1 = (j + 1 < nvalid) ? p1 : 0.f;
    }
    s0 += p0;
    s1 += p1;
    pk[j >> 1] = pack_bf16x2(p0, p1);
  }
  return s0 + s1;
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
  const int k0 = split * a.chunk;
  const int k1 = min(k0 + a.chunk, L);
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
  uint8_t* sP = base + SL.p;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + SL.bars);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kAttnStages;
  uint64_t* s_full = kv_empty + kAttnStages;  // [half][buffer]
  uint64_t* p_full = s_full + 4;              // [half]: P written (and O corrected)
  uint64_t* pv_done = p_full + 2;             // [half]: last P.V of the half finished
  uint64_t* o_full = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // TMEM: S[half][buffer] (64 fp32 columns each, double-buffered so the next
  // tile's scores are computed while this tile's softmax runs), then O[half].
  const uint32_t tmem_need = halves * (2 * kAttnBN + dh);
  const uint32_t tmem_cols = tmem_need <= 128 ? 128u : tmem_need <= 256 ? 256u : 512u;
  const uint32_t tO0 = halves * 2 * kAttnBN;

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
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&s_full[i], 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&p_full[h], 128);
      mbar_init(&pv_done[h], 1);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
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
  const int pos0 = qt * halves * a.s_per_half;  // first block position of this query tile

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKc);
      prefetch_tmap(&tmVc);
      const uint64_t pol_kv = policy_evict_first();
      mbar_arrive_expect_tx(q_full, (uint32_t)(halves * nsub * a.rows_per_half * 128));
      for (int h = 0; h < halves; ++h)
        for (int xh = 0; xh < nsub; ++xh)
          tma_load_3d(sQ + (h * nsub + xh) * kQSub, &tmQ, q_full, xh * 64, g * a.G,
                      b * a.S + pos0 + h * a.s_per_half);
      const int row_base = (b * a.Hkv + g) * a.L_cap;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % kAttnStages;
        const uint32_t ph = (uint32_t)(t / kAttnStages) & 1u;
        if (!mbar_wait(&kv_empty[st], ph ^ 1u, a.err, abort_flag, WHERE_ATTN_PRODUCER)) break;
        TT_TRACE_POINT(true, 0, t);
        const TileInfo ti = tile_info(t, has_blk, k0, k1, a.S);
        uint8_t* dk = sK + st * nsub * kSub;
        uint8_t* dv = sV + st * nsub * kSub;
        if (ti.is_blk) {
          mbar_arrive_expect_tx(&kv_full[st], (uint32_t)(2 * nsub * a.S * 128));
          for (int xh = 0; xh < nsub; ++xh) {
            tma_load_3d(dk + xh * kSub, &tmKb, &kv_full[st], xh * 64, g, b * a.S);
            tma_load_3d(dv + xh * kSub, &tmVb, &kv_full[st], xh * 64, g, b * a.S);
          }
        } else {
          mbar_arrive_expect_tx(&kv_full[st], (uint32_t)(2 * nsub * kSub));
          for (int xh = 0; xh < nsub; ++xh) {
            tma_load_2d_hint(dk + xh * kSub, &tmKc, &kv_full[st], xh * 64, row_base + ti.key0,
                             pol_kv);
            tma_load_2d_hint(dv + xh * kSub, &tmVc, &kv_full[st], xh * 64, row_base + ti.key0,
                             pol_kv);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t idS = idesc_bf16(128, kAttnBN, false, false);
    const uint32_t idO = idesc_bf16(128, dh, false, true);
    const uint32_t q0 = smem_u32(sQ), k0s = smem_u32(sK), v0s = smem_u32(sV), p0s = smem_u32(sP);
    auto issue_S = [&](int h, int st, int buf) {
      for (int kk = 0; kk < dh / 16; ++kk) {
        const int xh = kk >> 2;
        const uint32_t off = (uint32_t)(kk & 3) * 32;
        const uint64_t ad = sdesc_sw128(q0 + (h * nsub + xh) * kQSub + off, 16, 1024);
        const uint64_t bd = sdesc_sw128(k0s + (st * nsub + xh) * kSub + off, 16, 1024);
        umma_bf16_ss(tmem + (h * 2 + buf) * kAttnBN, ad, bd, idS, kk > 0);
      }
    };
    auto issue_PV = [&](int h, int st, bool acc) {
      for (int kk = 0; kk < kAttnBN / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(p0s + h * kPHalf + kk * 32, 16, 1024);
        // V as an MN-major operand: 64-wide dh blocks kSub apart, 8-key groups 1 KB apart.
        const uint64_t bd = sdesc_sw128(v0s + st * nsub * kSub + kk * 2048, kSub, 1024);
        umma_bf16_ss(tmem + tO0 + h * dh, ad, bd, idO, (acc || kk > 0) ? 1u : 0u);
      }
    };
    // V rows past the valid keys of a tile may hold anything (other
    // sequences' cache rows, stale stages); P is zero there, but 0 * NaN is
    // NaN, so clear them before the PV product reads the stage.
    auto prep = [&](int t, int st) {
      const TileInfo ti = tile_info(t, has_blk, k0, k1, a.S);
      if (ti.nvalid < kAttnBN) {
        const int rows = kAttnBN - ti.nvalid;
        for (int xh = 0; xh < nsub; ++xh) {
          uint4* dst = reinterpret_cast<uint4*>(sV + (st * nsub + xh) * kSub + ti.nvalid * 128);
          for (int i = lane; i < rows * 8; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
    };
    // Issue order: scores run two tiles ahead (S(0), S(1) up front), and in
    // each iteration P(t).V is issued for each half the moment its softmax
    // has written P, before S(t+2) - so a P.V never queues behind the next
    // tile's score MMAs and the softmax never waits for its P buffer.
    // S(t+2) reuses the buffer of tile t, which the softmax released with P(t).
    auto issue_scores = [&](int tt) -> bool {
      const int stt = tt % kAttnStages;
      if (!mbar_wait(&kv_full[stt], (uint32_t)(tt / kAttnStages) & 1u, a.err, abort_flag,
                     WHERE_ATTN_MMA))
        return false;
      TT_TRACE_POINT(lane == 0, 1, tt);
      tc_fence_after();
      prep(tt, stt);
      if (lane == 0) {
        for (int h = 0; h < halves; ++h) {
          issue_S(h, stt, tt & 1);
          umma_commit(&s_full[h * 2 + (tt & 1)]);
        }
      }
      __syncwarp();
      TT_TRACE_POINT(lane == 0, 2, tt);
      return true;
    };
    bool ok = mbar_wait(q_full, 0, a.err, abort_flag, WHERE_ATTN_MMA);
    for (int tt = 0; ok && tt < 2 && tt < n_tiles; ++tt) ok = issue_scores(tt);
    for (int t = 0; ok && t < n_tiles; ++t) {
      const int st = t % kAttnStages;
      for (int h = 0; h < halves; ++h) {
        if (!mbar_wait(&p_full[h], (uint32_t)t & 1u, a.err, abort_flag, WHERE_ATTN_MMA)) {
          ok = false;
          break;
        }
        TT_TRACE_POINT(lane == 0, 3 + h, t);
        tc_fence_after();
        if (lane == 0) {
          issue_PV(h, st, t > 0);
          umma_commit(&pv_done[h]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&kv_empty[st]);
      __syncwarp();
      if (t + 2 < n_tiles) ok = issue_scores(t + 2);
    }
    if (lane == 0) umma_commit(o_full);
    __syncwarp();
  } else {
    // ---------------------------------------------------- softmax groups
    const int wg = (warp - 2) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    if (wg < halves) {
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      const uint32_t tS = tmem + wg * 2 * kAttnBN + lane_off;
      const uint32_t tO = tmem + tO0 + wg * dh + lane_off;
      uint8_t* prow = sP + wg * kPHalf + r * 128;
      const float c = a.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        const int buf = t & 1;
        if (!mbar_wait(&s_full[wg * 2 + buf], (uint32_t)(t >> 1) & 1u, a.err, abort_flag,
                       WHERE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        TT_TRACE_POINT(lane == 0 && q == 0, 5 + 5 * wg, t);
        tc_fence_after();
        const int nvalid = tile_info(t, has_blk, k0, k1, a.S).nvalid;
        uint32_t sr[64];
        tmem_ld32(tS + buf * kAttnBN, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + buf * kAttnBN + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        TT_TRACE_POINT(lane == 0 && q == 0, 6 + 5 * wg, t);
        const bool full = nvalid == kAttnBN;
        float mx = full ? row_max<true>(sr, nvalid) : row_max<false>(sr, nvalid);
        const float mxs = mx * c;
        const bool need = mxs > m + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2(m - mxs);
          m = mxs;
        }
        l *= alpha;
        // P(t-1).V must have finished before O is rescaled or P rewritten.
        if (t > 0) {
          if (!mbar_wait(&pv_done[wg], (uint32_t)(t - 1) & 1u, a.err, abort_flag,
                         WHERE_ATTN_SOFTMAX)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
            for (int c0 = 0; c0 < dh; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st32(tO + c0, o);
            }
            tmem_wait_st();
          }
        }
        TT_TRACE_POINT(lane == 0 && q == 0, 7 + 5 * wg, t);
        uint32_t pk[32];
        l += full ? exp_pack<true>(sr, nvalid, c, m, pk) : exp_pack<false>(sr, nvalid, c, m, pk);
        TT_TRACE_POINT(lane == 0 && q == 0, 8 + 5 * wg, t);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int phys = j ^ (r & 7);
          *reinterpret_cast<uint4*>(prow + phys * 16) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[wg]);
        TT_TRACE_POINT(lane == 0 && q == 0, 9 + 5 * wg, t);
      }
      if (ok && mbar_wait(o_full, 0, a.err, abort_flag, WHERE_ATTN_SOFTMAX)) {
        tc_fence_after();
        const bool valid = r < a.rows_per_half;
        const int s = pos0 + wg * a.s_per_half + r / a.G;
        const int head = g * a.G + r % a.G;
        if (a.n_splits == 1) {
          const float inv = 1.f / l;
          uint16_t* dst = a.out + (size_t)(b * a.S + s) * a.ldo + head * dh;
          for (int c0 = 0; c0 < dh; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
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
          const size_t prow_i = (size_t)unit * 256 + wg * 128 + r;
          float* po = a.part_o + prow_i * dh;
          for (int c0 = 0; c0 < dh; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                *reinterpret_cast<float4*>(po + c0 + 4 * v) =
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// One warp per query row: combine the splits' partials,
//   O = sum_i 2^(m_i - m*) O_i / sum_i 2^(m_i - m*) l_i.
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnArgs a) {
  griddep_launch();
  griddep_wait();
  if (a.active != nullptr && *a.active == 0) return;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int total = a.B * a.Hkv * a.n_qtiles * 256;
  if (gw >= total) return;
  const int row256 = gw & 255;
  const int pq = gw >> 8;  // pair * n_qtiles + qt
  const int h = row256 >> 7, r = row256 & 127;
  if (h >= a.halves || r >= a.rows_per_half) return;
  const int pair = pq / a.n_qtiles, qt = pq % a.n_qtiles;
  const int b = pair / a.Hkv, g = pair % a.Hkv;
  float mstar = -INFINITY;
  for (int sp = 0; sp < a.n_splits; ++sp) {
    const size_t i = ((size_t)(pq * a.n_splits + sp) * 256 + row256) * 2;
    if (a.part_ml[i + 1] > 0.f) mstar = fmaxf(mstar, a.part_ml[i]);
  }
  const int d0 = lane * 4;
  const bool act = d0 < a.dh;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  for (int sp = 0; sp < a.n_splits; ++sp) {
    const size_t prow = (size_t)(pq * a.n_splits + sp) * 256 + row256;
    const float ms = a.part_ml[prow * 2], ls = a.part_ml[prow * 2 + 1];
    if (!(ls > 0.f)) continue;
    const float w = ex2(ms - mstar);
    den += w * ls;
    if (act) {
      const float4 o = *reinterpret_cast<const float4*>(a.part_o + prow * a.dh + d0);
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
    }
  }
  if (act) {
    const float inv = 1.f / den;
    const int s = qt * a.halves * a.s_per_half + h * a.s_per_half + r / a.G;
    const int head = g * a.G + r % a.G;
    uint16_t* dst = a.out + (size_t)(b * a.S + s) * a.ldo + head * a.dh + d0;
    uint2 wv;
    wv.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    wv.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(dst) = wv;
  }
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
  const long long warps = (long long)a.B * a.Hkv * a.n_qtiles * 256;
  const int blocks = (int)((warps * 32 + 255) / 256);
  return launch_k(attn_merge_kernel, dim3(blocks), dim3(256), 0, st, a);
}

}  // namespace tt
