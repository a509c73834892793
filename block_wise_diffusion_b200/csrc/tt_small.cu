// The light kernels of the denoise step: step planning (masked-row list and
// timesteps), adaLN-single modulation, row gathers, block re-embedding and
// the confidence commit.  All are bandwidth- or latency-bound and tiny next
// to the attention and the vocabulary GEMM.
#include <math.h>

#include "tt_ptx.cuh"

namespace tt {

namespace {

// ------------------------------------------------------------------ plan
// Compact list of masked rows (b*S + s) in row order, the per-sequence
// timestep t_b = masked count / S, and the step's control words, computed by
// one CTA of any size (a multiple of 32 threads).  `masked` is read through
// volatile loads: in the commit kernel it was just written by other CTAs.
__device__ void plan_block(const PlanArgs& a) {
  __shared__ int warp_tot[32];
  __shared__ int running;
  const volatile uint8_t* masked = a.masked;
  const int n = a.B * a.S;
  const int nt = blockDim.x, nw = nt >> 5;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) running = 0;
  __syncthreads();
  for (int base = 0; base < n; base += nt) {
    const int i = base + tid;
    const int f = (i < n && masked[i] != 0) ? 1 : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    const int before_in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    int before_warps = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
      const int c = warp_tot[w];
      before_warps += (w < warp) ? c : 0;
      total += c;
    }
    if (f) {
      a.rowlist[running + before_warps + before_in_warp] = i;
      a.rowlist[n + i] = running + before_warps + before_in_warp;
    }
    __syncthreads();
    if (tid == 0) running += total;
    __syncthreads();
  }
  for (int b = tid; b < a.B; b += nt) {
    int c = 0;
    for (int s = 0; s < a.S; ++s) c += masked[b * a.S + s] != 0;
    a.t[b] = (float)c / (float)a.S;
  }
  if (tid == 0) {
    const int M = running;
    a.ctrl[CTRL_M] = M;
    a.ctrl[CTRL_REMAINING] = M;
    a.ctrl[CTRL_ACTIVE] = M > 0 ? 1 : 0;
  }
}

__global__ void __launch_bounds__(1024) plan_kernel(const PlanArgs a) {
  griddep_launch();
  griddep_wait();
  plan_block(a);
}

// ----------------------------------------------------------------- adaLN
// One CTA per output row.  y = LN(x) * (1 + E1 + cos(t w)) + E0 + sin(t w),
// w_i = 10000^(-i/H): the adaLN-single reading of this library.
constexpr int kAdaThreads = 512;
constexpr int kAdaMaxVec = 2;  // H <= 512 threads * 2 vectors * 8 = 8192

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < kAdaThreads / 32; ++w) s += red[w];
  return s;
}

// LayerNorm of the row held in v (8 values per vector, vectors threadIdx.x +
// k*kAdaThreads) followed by the time modulation; writes the bf16 row yr.
__device__ __forceinline__ void adaln_finish(float (&v)[kAdaMaxVec][8], float s, int H, float tb,
                                             const uint16_t* __restrict__ ss,
                                             uint16_t* __restrict__ yrow, float* red) {
  const int nvec = H / 8;
  // shift/scale loads are issued before the two reductions
  uint4 a0[kAdaMaxVec], a1[kAdaMaxVec];
  const uint4* e0 = reinterpret_cast<const uint4*>(ss);
  const uint4* e1 = reinterpret_cast<const uint4*>(ss + H);
#pragma unroll
  for (int k = 0; k < kAdaMaxVec; ++k) {
    const int vi = threadIdx.x + k * kAdaThreads;
    if (vi < nvec) {
      a0[k] = e0[vi];
      a1[k] = e1[vi];
    }
  }
  const float mean = block_sum(s, red) / (float)H;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < kAdaMaxVec; ++k) {
    const int vi = threadIdx.x + k * kAdaThreads;
    if (vi < nvec) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[k][e] - mean;
        q += d * d;
      }
    }
  }
  const float var = block_sum(q, red) / (float)H;
  const float rstd = rsqrtf(var + 1e-6f);
  const float lw = -13.287712379549449f / (float)H;  // -log2(10000) / H
  uint4* yr = reinterpret_cast<uint4*>(yrow);
#pragma unroll
  for (int k = 0; k < kAdaMaxVec; ++k) {
    const int vi = threadIdx.x + k * kAdaThreads;
    if (vi < nvec) {
      const uint32_t sh[4] = {a0[k].x, a0[k].y, a0[k].z, a0[k].w};
      const uint32_t sc[4] = {a1[k].x, a1[k].y, a1[k].z, a1[k].w};
      float out[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = vi * 8 + e;
        const float w = ex2((float)i * lw);
        float sn, cs;
        __sincosf(tb * w, &sn, &cs);  // |t w| <= 1: abs error ~1e-6, far below bf16 output
        const uint32_t hs = (e & 1) ? (sh[e >> 1] & 0xffff0000u) : (sh[e >> 1] << 16);
        const uint32_t hc = (e & 1) ? (sc[e >> 1] & 0xffff0000u) : (sc[e >> 1] << 16);
        const float shift = __uint_as_float(hs) + sn;
        const float scale = __uint_as_float(hc) + cs;
        out[e] = (v[k][e] - mean) * rstd * (1.f + scale) + shift;
      }
      uint4 o;
      o.x = pack_bf16x2(out[0], out[1]);
      o.y = pack_bf16x2(out[2], out[3]);
      o.z = pack_bf16x2(out[4], out[5]);
      o.w = pack_bf16x2(out[6], out[7]);
      yr[vi] = o;
    }
  }
}

// As adaln_finish, for rows held as 4-column groups: group k of this thread
// covers columns i0[k]..i0[k]+3 (gin[k] false: no group).
template <int KG>
__device__ __forceinline__ void adaln_finish_groups(float (&v)[KG][4], const bool (&gin)[KG],
                                                    const int (&i0)[KG], float s, int H, float tb,
                                                    const uint16_t* __restrict__ ss,
                                                    uint16_t* __restrict__ yrow, float* red) {
  uint2 a0[KG], a1[KG];  // shift/scale loads are issued before the reductions
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    if (gin[k]) {
      a0[k] = *reinterpret_cast<const uint2*>(ss + i0[k]);
      a1[k] = *reinterpret_cast<const uint2*>(ss + H + i0[k]);
    }
  }
  const float mean = block_sum(s, red) / (float)H;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    if (gin[k]) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d = v[k][e] - mean;
        q += d * d;
      }
    }
  }
  const float var = block_sum(q, red) / (float)H;
  const float rstd = rsqrtf(var + 1e-6f);
  const float lw = -13.287712379549449f / (float)H;  // -log2(10000) / H
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    if (!gin[k]) continue;
    const uint32_t sh[2] = {a0[k].x, a0[k].y};
    const uint32_t sc[2] = {a1[k].x, a1[k].y};
    float out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0[k] + e;
      const float w = ex2((float)i * lw);
      float sn, cs;
      __sincosf(tb * w, &sn, &cs);  // |t w| <= 1: abs error ~1e-6, far below bf16 output
      const uint32_t hs = (e & 1) ? (sh[e >> 1] & 0xffff0000u) : (sh[e >> 1] << 16);
      const uint32_t hc = (e & 1) ? (sc[e >> 1] & 0xffff0000u) : (sc[e >> 1] << 16);
      out[e] = (v[k][e] - mean) * rstd * (1.f + __uint_as_float(hc) + cs) + __uint_as_float(hs) + sn;
    }
    uint2 o;
    o.x = pack_bf16x2(out[0], out[1]);
    o.y = pack_bf16x2(out[2], out[3]);
    *reinterpret_cast<uint2*>(yrow + i0[k]) = o;
  }
}

// Block loop, one CTA per block row (all B*S rows are launched): decides
// whether this CTA's row is still masked and, if so, its index j in the
// compact list of masked rows (masked rows before it) and its sequence's
// time t_b = masked count / S.  The CTA of the first masked row publishes the
// row count (ctrl[CTRL_M]); every CTA records rowlist[j] = row for the commit.
// Returns false (uniformly) for a committed row.
__device__ bool loop_row(const uint8_t* __restrict__ masked, int rows, int S, int row,
                         int* __restrict__ rowlist, int* __restrict__ ctrl, int* j_out,
                         float* tb_out) {
  __shared__ int cnt[3][kAdaThreads / 32];
  // rowlist == nullptr: every row (a denoiser layer before the last), at its
  // own index, with nothing recorded
  const bool all_rows = rowlist == nullptr;
  if (!all_rows && masked[row] == 0) return false;
  const int b0 = (row / S) * S;
  int before = 0, total = 0, seq = 0;
  for (int i = threadIdx.x; i < rows; i += blockDim.x) {
    const int f = masked[i] != 0;
    total += f;
    before += (i < row) ? f : 0;
    seq += (i >= b0 && i < b0 + S) ? f : 0;
  }
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
    seq += __shfl_xor_sync(0xffffffffu, seq, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    cnt[0][warp] = before;
    cnt[1][warp] = total;
    cnt[2][warp] = seq;
  }
  __syncthreads();
  before = total = seq = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    before += cnt[0][w];
    total += cnt[1][w];
    seq += cnt[2][w];
  }
  if (threadIdx.x == 0 && !all_rows) {
    rowlist[before] = row;
    rowlist[rows + row] = before;
    if (before == 0) ctrl[CTRL_M] = total;
  }
  *j_out = all_rows ? row : before;
  *tb_out = (float)seq / (float)S;
  return true;
}

__global__ void __launch_bounds__(kAdaThreads)
    adaln_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ ss,
                 const float* __restrict__ t, uint16_t* __restrict__ y, int rows, int S, int H,
                 const uint8_t* __restrict__ masked, int* __restrict__ rowlist, int* ctrl,
                 const int* active) {
  griddep_launch();
  griddep_wait();
  __shared__ float red[kAdaThreads / 32];
  if (active != nullptr && *active == 0) return;
  // masked == nullptr: every row, t per sequence from `t`; otherwise the block
  // loop's rows (the masked ones compacted, or all of them for an earlier
  // denoiser layer).
  int j = blockIdx.x, src = blockIdx.x;
  float tb;
  if (masked == nullptr) {
    tb = t[src / S];
  } else if (!loop_row(masked, rows, S, src, rowlist, ctrl, &j, &tb)) {
    return;
  }
  const int nvec = H / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)src * H);
  float v[kAdaMaxVec][8];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kAdaMaxVec; ++k) {
    const int vi = threadIdx.x + k * kAdaThreads;
    if (vi < nvec) {
      const uint4 u = xr[vi];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[k][2 * e] = __uint_as_float(w[e] << 16);
        v[k][2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) s += v[k][e];
    }
  }
  adaln_finish(v, s, H, tb, ss, y + (size_t)j * H, red);
}

// The CTAs of a unit's range: [c_first, c_last] (one with an empty range
// wrote an empty record for the unit).
struct SegRange {
  int c_first, c_last;
};

// Attention merge fused with adaLN (block loop; used when the attention's
// units span many CTAs, see AttnArgs::fixup): one CTA per block row (b, s),
// returning at once for a committed row unless every row is wanted.  For
// each query head the unit's segment partials are combined,
//   o = sum_i 2^(m_i - m*) O_i / sum_i 2^(m_i - m*) l_i,
// rounded to bf16 (the attention output's storage precision), and the whole
// row then goes through adaln_finish.
// KG four-column groups per thread (H <= KG * 4 * kAdaThreads); NB segments'
// loads in flight per round.
template <int KG, int NB>
__global__ void __launch_bounds__(kAdaThreads)
    merge_adaln_kernel(const AttnArgs a, const uint16_t* __restrict__ ss,
                       uint16_t* __restrict__ y, const uint8_t* __restrict__ masked,
                       int* __restrict__ rowlist, int* ctrl) {
  griddep_launch();
  griddep_wait();
  __shared__ float red[kAdaThreads / 32];
  if (a.active != nullptr && *a.active == 0) return;
  const int row = blockIdx.x;
  int j;
  float tb;
  if (!loop_row(masked, a.B * a.S, a.S, row, rowlist, ctrl, &j, &tb)) return;
  const int b = row / a.S, s = row % a.S;
  const int H = a.Hq * a.dh;
  const int sq = a.halves * a.s_per_half;
  const int qt = s / sq, within = s % sq;
  const int hh = within / a.s_per_half, sl = within % a.s_per_half;
  // Each thread merges up to KG four-column groups of the row in one pass
  // over the segments (running max, rescaled sums), loading NB segments'
  // data for all its groups before using any.  Group gi covers head
  // gi % Hq, columns 4*(gi / Hq)..+3: consecutive threads take consecutive
  // heads, i.e. consecutive rows of the tile-major partials (coalesced).
  constexpr int kG = KG;
  const int ngrp = a.dh / 4, ng = a.Hq * ngrp;
  int unit[kG], n_seg[kG], r256[kG], grp[kG], i0[kG];
  SegRange sr[kG];
  bool gin[kG];
  float mrun[kG], den[kG], v[kG][4];
  int max_seg = 0;
#pragma unroll
  for (int k = 0; k < kG; ++k) {
    const int gi = (int)threadIdx.x + k * kAdaThreads;
    gin[k] = gi < ng;
    const int gc = min(gi, ng - 1);
    const int head = gc % a.Hq;
    grp[k] = gc / a.Hq;
    i0[k] = head * a.dh + grp[k] * 4;
    const int g = head / a.G, jh = head % a.G;
    unit[k] = (b * a.Hkv + g) * a.n_qtiles + qt;
    const int4 uc = a.unit_ctas[unit[k]];
    sr[k] = SegRange{uc.x, uc.y};
    n_seg[k] = gin[k] ? sr[k].c_last - sr[k].c_first + 1 : 0;
    max_seg = max(max_seg, n_seg[k]);
    r256[k] = hh * 128 + sl * a.G + jh;
    mrun[k] = -INFINITY;
    den[k] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) v[k][e] = 0.f;
  }
  for (int sp0 = 0; sp0 < max_seg; sp0 += NB) {
    float2 ml[NB][kG];
    float4 x[NB][kG];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
#pragma unroll
      for (int k = 0; k < kG; ++k) {
        if (sp0 + i < n_seg[k]) {
          const size_t slot = (size_t)unit[k] + sr[k].c_first + sp0 + i;
          const float4 q4 =
              *reinterpret_cast<const float4*>(a.part_ml + (slot * 256 + r256[k]) * 4);
          ml[i][k] = make_float2(q4.x, q4.y + q4.z);
          x[i][k] = *reinterpret_cast<const float4*>(
              a.part_o + ((slot * ngrp + grp[k]) * 256 + r256[k]) * 4);
        } else {
          ml[i][k] = make_float2(-INFINITY, 0.f);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
#pragma unroll
      for (int k = 0; k < kG; ++k) {
        if (!(ml[i][k].y > 0.f)) continue;
        if (ml[i][k].x > mrun[k]) {
          const float sc = mrun[k] == -INFINITY ? 0.f : ex2(mrun[k] - ml[i][k].x);
          den[k] *= sc;
#pragma unroll
          for (int e = 0; e < 4; ++e) v[k][e] *= sc;
          mrun[k] = ml[i][k].x;
        }
        const float w = ex2(ml[i][k].x - mrun[k]);
        den[k] += w * ml[i][k].y;
        v[k][0] += w * x[i][k].x;
        v[k][1] += w * x[i][k].y;
        v[k][2] += w * x[i][k].z;
        v[k][3] += w * x[i][k].w;
      }
    }
  }
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < kG; ++k) {
    if (!gin[k]) continue;
    const float inv = 1.f / den[k];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // the attention output is bf16 in the unfused path: round the same way
      v[k][e] = __uint_as_float(pack_bf16x2(v[k][e] * inv, 0.f) << 16);
      sum += v[k][e];
    }
  }
  adaln_finish_groups<kG>(v, gin, i0, sum, H, tb, ss, y + (size_t)j * H, red);
}

// ---------------------------------------------------------------- gathers
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint16_t* __restrict__ src, int ld_src, uint16_t* __restrict__ dst,
                       int H, const int* __restrict__ rowlist, const int* M_dev, int max_rows,
                       const int* active) {
  griddep_launch();
  griddep_wait();
  if (active != nullptr && *active == 0) return;
  const int M = M_dev != nullptr ? min(*M_dev, max_rows) : max_rows;
  const int j = blockIdx.x;
  if (j >= M) return;
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)rowlist[j] * ld_src);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)j * H);
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) d[i] = s[i];
}

// e[row] = masked ? e_mask : Emb[token]; an out-of-range token of a committed
// position is reported (TT_ERR_INTERNAL) and embedded as e_mask.
__global__ void __launch_bounds__(256)
    embed_kernel(const int* __restrict__ tokens, const uint8_t* __restrict__ masked,
                 const uint16_t* __restrict__ emb, const uint16_t* __restrict__ e_mask,
                 uint16_t* __restrict__ dst, int rows, int H, int V, const int* active,
                 int* err) {
  griddep_launch();
  griddep_wait();
  if (active != nullptr && *active == 0) return;
  const int row = blockIdx.x;
  if (row >= rows) return;
  const uint16_t* src = e_mask;
  if (masked[row] == 0) {
    const int tok = tokens[row];
    if (tok >= 0 && tok < V) {
      src = emb + (size_t)tok * H;
    } else if (threadIdx.x == 0) {
      atomicCAS(err, 0, (int)TT_ERR_INTERNAL);
      atomicCAS(err + 1, 0, (int)WHERE_GATHER_TOKEN);
    }
  }
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)row * H);
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) d[i] = s[i];
}

// ---------------------------------------------------------------- commit
// Merge of one tile-statistics entry into a running (best tile maximum v*,
// its tile and token, Z = sum_t z_t 2^(c (v_t - v*))); a strictly greater
// maximum wins, equal maxima keep the lower tile (hence the lowest id).
struct RowBest {
  float v, Z;
  int t, tok;
};
__device__ __forceinline__ void rb_merge(RowBest& x, const RowBest& y, float c) {
  if (y.Z == 0.f && y.v == -INFINITY) return;
  const float nv = fmaxf(x.v, y.v);
  x.Z = (x.v == nv ? x.Z : x.Z * ex2((x.v - nv) * c)) + (y.v == nv ? y.Z : y.Z * ex2((y.v - nv) * c));
  if (y.v > x.v || (y.v == x.v && y.t < x.t)) {
    x.v = y.v;
    x.t = y.t;
    x.tok = y.tok;
  }
}

// One CTA per block row.  A masked position's ceil(V/224) tile statistics
// are merged by all kCommitThreads threads (every load of the row in flight
// at once) into its confidence
//   conf = 1 / sum_t z_t 2^(c*(v_t - v*)),  token = argmax column of the
// tile with the largest v_t (lowest tile on ties, hence lowest id).
// The last CTA of a sequence to finish then applies the commit rule
// across the sequence's S positions.
__global__ void __launch_bounds__(kCommitThreads) commit_kernel(const CommitArgs a) {
  griddep_launch();
  griddep_wait();
  constexpr int kWarps = kCommitThreads / 32;
  __shared__ int s_last;
  __shared__ int s_tok[kCommitThreads];
  __shared__ int s_com[kCommitThreads];
  __shared__ float s_bc[kWarps];
  __shared__ int s_bs[kWarps];
  __shared__ RowBest s_rb[kWarps];
  if (a.active != nullptr && *a.active == 0) return;
  const int S = a.S;
  const int row = blockIdx.x, b = row / S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M_dev != nullptr ? *a.M_dev : a.B * S;
  const float c = a.scale_log2;
  if (a.masked[row] != 0) {
    const int j = a.rowlist[a.B * S + row];  // this row's compact index
    RowBest rb{-INFINITY, 0.f, 0x7fffffff, -1};
    if (j >= 0 && j < M) {
      // thread i reads tiles i, i + kCommitThreads, ...: all loads first
      const float4* st = a.stats + (size_t)j * a.n_vt;
      constexpr int kPer = 4;  // up to kPer * kCommitThreads tiles in one round
      for (int t0 = threadIdx.x; t0 < a.n_vt; t0 += kPer * kCommitThreads) {
        float4 q[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int t = t0 + i * kCommitThreads;
          q[i] = t < a.n_vt ? st[t] : make_float4(-INFINITY, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i)
          if (q[i].x > -INFINITY)
            rb_merge(rb, RowBest{q[i].x, q[i].y, t0 + i * kCommitThreads, __float_as_int(q[i].z)},
                     c);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      RowBest y;
      y.v = __shfl_xor_sync(0xffffffffu, rb.v, o);
      y.Z = __shfl_xor_sync(0xffffffffu, rb.Z, o);
      y.t = __shfl_xor_sync(0xffffffffu, rb.t, o);
      y.tok = __shfl_xor_sync(0xffffffffu, rb.tok, o);
      rb_merge(rb, y, c);
    }
    if (lane == 0) s_rb[warp] = rb;
    __syncthreads();
    if (threadIdx.x == 0) {
      RowBest x = s_rb[0];
      for (int w = 1; w < kWarps; ++w) rb_merge(x, s_rb[w], c);
      const bool found = j >= 0 && j < M && x.t < a.n_vt;
      a.rowres[row] = make_float2(found ? 1.f / x.Z : -1.f, __int_as_float(found ? x.tok : -1));
    }
  } else if (threadIdx.x == 0) {
    a.rowres[row] = make_float2(-1.f, __int_as_float(-1));
  }
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.seqcnt + b, 1) == S - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  {
    // One thread per position of sequence b (S <= kCommitThreads).
    const int s = threadIdx.x;
    const bool in = s < S;
    const int r = b * S + min(s, S - 1);
    const int is_m = in ? a.masked[r] != 0 : 0;
    const float2 rr = in ? __ldcg(a.rowres + r) : make_float2(-1.f, __int_as_float(-1));
    float cf = rr.x;
    const int tk = __float_as_int(rr.y);
    const bool bad = is_m && !(cf >= 0.f && cf <= 1.0001f);  // NaN or impossible value
    if (__syncthreads_or(bad) && threadIdx.x == 0) {
      atomicCAS(a.ctrl + CTRL_ERR, 0, (int)TT_ERR_INTERNAL);
      atomicCAS(a.ctrl + CTRL_ERR_WHERE, 0, (int)WHERE_COMMIT_NAN);
    }
    if (bad) cf = -1.f;
    const bool qual = is_m && cf >= a.gamma && tk >= 0;
    const int nqual = __syncthreads_count(qual);
    const int nmask = __syncthreads_count(is_m != 0);
    bool commit = qual;
    if (nqual == 0 && nmask != 0) {  // uniform over the CTA
      // fallback: the most confident masked position, lowest s on ties
      float bc = is_m ? cf : -INFINITY;
      int bs = is_m ? s : 0x7fffffff;
      for (int o = 16; o > 0; o >>= 1) {
        const float oc = __shfl_xor_sync(0xffffffffu, bc, o);
        const int os = __shfl_xor_sync(0xffffffffu, bs, o);
        if (oc > bc || (oc == bc && os < bs)) {
          bc = oc;
          bs = os;
        }
      }
      if (lane == 0) {
        s_bc[warp] = bc;
        s_bs[warp] = bs;
      }
      __syncthreads();
      for (int w = 0; w < kWarps; ++w) {
        if (s_bc[w] > bc || (s_bc[w] == bc && s_bs[w] < bs)) {
          bc = s_bc[w];
          bs = s_bs[w];
        }
      }
      commit = is_m && s == bs;
    }
    s_com[s] = (in && commit) ? 1 : 0;
    s_tok[s] = tk >= 0 ? tk : 0;
    if (in) {
      if (commit) {
        a.tokens[r] = s_tok[s];
        a.masked[r] = 0;
        if (a.commit_step != nullptr) a.commit_step[r] = a.step;
      }
      if (a.conf_out != nullptr) a.conf_out[r] = is_m ? rr.x : -1.f;
      if (a.argmax_out != nullptr) a.argmax_out[r] = is_m ? tk : -1;
    }
    const int ncom = __syncthreads_count(in && commit);
    if (threadIdx.x == 0) {
      a.seqcnt[b] = 0;  // ready for the next call
      if (a.n_committed != nullptr) a.n_committed[b] = ncom;
      if (a.steps_taken != nullptr && nmask != 0) a.steps_taken[b] = a.step + 1;
      if (a.plan_next) {
        // Loop: the remaining-masked counter is also the next step's active flag.
        if (ncom) atomicSub(a.ctrl + CTRL_REMAINING, ncom);
        if (b == 0) atomicAdd(a.ctrl + CTRL_STEPS_RUN, 1);
      }
    }
  }
  __syncthreads();
  // Loop only: a newly committed position's next embedding is Emb[token].
  // All threads copy the committed rows together, eight 16-byte loads in
  // flight per thread before any store.
  if (a.egath != nullptr) {
    const int nv = a.H / 8;  // 16-byte vectors per row
    int nc = 0;
    for (int s = 0; s < S; ++s) nc += s_com[s];
    const long long total = (long long)nc * nv;
    for (long long v0 = threadIdx.x; v0 < total; v0 += 8 * kCommitThreads) {
      uint4 buf[8];
      uint4* dst[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const long long v = v0 + (long long)k * kCommitThreads;
        dst[k] = nullptr;
        if (v < total) {
          int cc = (int)(v / nv), s = 0;
          for (;; ++s) {  // the cc-th committed position
            if (s_com[s] && cc-- == 0) break;
          }
          const int i = (int)(v % nv);
          buf[k] = __ldg(reinterpret_cast<const uint4*>(a.emb + (size_t)s_tok[s] * a.H) + i);
          dst[k] = reinterpret_cast<uint4*>(a.egath + (size_t)(b * S + s) * a.H) + i;
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (dst[k] != nullptr) *dst[k] = buf[k];
    }
  }
}

// Failure-detection self test: wait on an mbarrier that nothing will ever
// complete, with a short limit, so the bounded-wait path records
// TT_ERR_TIMEOUT in the control block and the kernel returns normally.
__global__ void selftest_wait_kernel(int* ctrl, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait_slow(&bar, 0, ctrl, &abort_flag, WHERE_SELFTEST, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag == 0) atomicCAS(ctrl, 0, (int)TT_ERR_INTERNAL);
}

__global__ void loop_init_kernel(int B, int S, int* steps_taken, int* commit_step) {
  griddep_launch();
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) steps_taken[i] = 0;
  if (i < B * S) commit_step[i] = -1;
}

// A committed block joins the context: CTA b copies the block's projected
// rows kv [B*S, ld] (k of head g at columns g*dh.., v at Hkv*dh + g*dh..) to
// context positions ctx_len[b] .. ctx_len[b] + S - 1 of every KV head, then
// advances ctx_len[b].  A sequence without room records TT_ERR_INVALID_ARG
// and is left unchanged.
__global__ void __launch_bounds__(256)
    append_kv_kernel(const uint16_t* __restrict__ kv, int ld, uint16_t* __restrict__ k_ctx,
                     uint16_t* __restrict__ v_ctx, int* __restrict__ ctx_len, int S, int Hkv,
                     int dh, int L_cap, int* err) {
  griddep_launch();
  griddep_wait();
  const int b = blockIdx.x;
  const int L = ctx_len[b];
  if (L < 0 || L + S > L_cap) {
    if (threadIdx.x == 0) atomicCAS(err, 0, (int)TT_ERR_INVALID_ARG);
    return;
  }
  const int nv = dh / 8;  // 16-byte vectors per head row
  const int total = S * Hkv * nv;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int c = i % nv, g = (i / nv) % Hkv, s = i / (nv * Hkv);
    const uint4* src = reinterpret_cast<const uint4*>(kv + (size_t)(b * S + s) * ld + g * dh);
    const size_t dst = ((size_t)(b * Hkv + g) * L_cap + L + s) * dh;
    reinterpret_cast<uint4*>(k_ctx + dst)[c] = src[c];
    reinterpret_cast<uint4*>(v_ctx + dst)[c] = src[(Hkv * dh) / 8 + c];
  }
  __syncthreads();
  if (threadIdx.x == 0) ctx_len[b] = L + S;
}

}  // namespace

cudaError_t launch_append_kv(const uint16_t* kv, int ld, uint16_t* k_ctx, uint16_t* v_ctx,
                             int* ctx_len, int B, int S, int Hkv, int dh, int L_cap, int* err,
                             cudaStream_t st) {
  return launch_k(append_kv_kernel, dim3(B), dim3(256), 0, st, kv, ld, k_ctx, v_ctx, ctx_len, S,
                  Hkv, dh, L_cap, err);
}

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t st) {
  return launch_k(plan_kernel, dim3(1), dim3(1024), 0, st, a);
}

cudaError_t launch_adaln(const uint16_t* x, const uint16_t* shift_scale, const float* t,
                         uint16_t* y, int rows, int S, int H, const uint8_t* masked,
                         int* rowlist, int* ctrl, const int* active, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(adaln_kernel, dim3(rows), dim3(kAdaThreads), 0, st, x, shift_scale, t, y, rows,
                  S, H, masked, rowlist, ctrl, active);
}

cudaError_t launch_merge_adaln(const AttnArgs& a, const uint16_t* shift_scale, uint16_t* y,
                               const uint8_t* masked, int* rowlist, int* ctrl, cudaStream_t st) {
  const int rows = a.B * a.S;
  if (a.Hq * a.dh <= 2 * 4 * kAdaThreads)
    return launch_k(merge_adaln_kernel<2, 4>, dim3(rows), dim3(kAdaThreads), 0, st, a, shift_scale,
                    y, masked, rowlist, ctrl);
  return launch_k(merge_adaln_kernel<4, 2>, dim3(rows), dim3(kAdaThreads), 0, st, a, shift_scale, y,
                  masked, rowlist, ctrl);
}

cudaError_t launch_gather_rows(const uint16_t* src, int ld_src, uint16_t* dst, int H,
                               const int* rowlist, const int* M_dev, int max_rows,
                               const int* active, cudaStream_t st) {
  if (max_rows <= 0) return cudaSuccess;
  return launch_k(gather_rows_kernel, dim3(max_rows), dim3(256), 0, st, src, ld_src, dst, H,
                  rowlist, M_dev, max_rows, active);
}

cudaError_t launch_embed(const int* tokens, const uint8_t* masked, const uint16_t* emb,
                         const uint16_t* e_mask, uint16_t* dst, int rows, int H, int V,
                         const int* active, int* err, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(embed_kernel, dim3(rows), dim3(256), 0, st, tokens, masked, emb, e_mask, dst,
                  rows, H, V, active, err);
}

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st) {
  return launch_k(commit_kernel, dim3(a.B * a.S), dim3(kCommitThreads), 0, st, a);
}

cudaError_t launch_selftest_wait(int* ctrl, unsigned long long limit_ns, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(ctrl, limit_ns);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_loop_init(int B, int S, int* steps_taken, int* commit_step, int* ctrl,
                             cudaStream_t st) {
  (void)ctrl;
  const int n = B * S;
  return launch_k(loop_init_kernel, dim3((n + 255) / 256), dim3(256), 0, st, B, S, steps_taken,
                  commit_step);
}

}  // namespace tt
