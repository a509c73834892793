// Persistent tcgen05 GEMM for the two dense contractions of the denoise step:
//
//  * the vocabulary projection (logits = y . W^T, W stored [V, H]) with an
//    epilogue that reduces each 256-wide logit tile of each row to
//    (max, sum of exp relative to that max, argmax) straight out of TMEM, so
//    logits never reach memory ("Training and Conditioning", Sampling: all
//    masked positions are predicted in parallel and ranked by confidence);
//  * the linear update [q|k|v] = e . U of the block loop, plain bf16 store.
//
// Layout: A [M, K] and B [N, K] are K-major bf16, loaded by TMA in 128-byte
// swizzled 64-column boxes (A: 128 rows, B: BN rows per stage; BN = 224 for
// the vocabulary, 128 for the linear update).  One CTA per SM walks tiles
// m-fastest, so the CTAs that share a W tile run together and W crosses HBM
// once.  Warp 0 issues TMA, warp 1 issues tcgen05.mma (M=128, N=BN, K=16)
// into one of two BN-column TMEM accumulators, warps 2..5 drain the other
// accumulator (TMEM lane = tile row).  With few rows the linear update is
// split over K so every SM streams part of U; the fp32 partial tiles are
// summed by splitk_reduce_kernel.
#include <math.h>

#include "tt_ptx.cuh"

namespace tt {

namespace {

constexpr uint32_t kStageA = kGemmBM * kGemmBK * 2;  // 16 KB

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// EPI 0: vocabulary statistics, 1: bf16 store.  BN: tile width (N of the
// MMA, a multiple of 16 up to 256); STAGES: depth of the TMA ring.
template <int EPI, int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs a) {
  griddep_launch();
  griddep_wait();
  extern __shared__ uint8_t smem_raw[];
  if (a.active != nullptr && *a.active == 0) return;
  const int M = a.M_dev != nullptr ? min(*a.M_dev, a.M_alloc) : a.M_alloc;
  if (M <= 0) return;
  const int num_m = (M + kGemmBM - 1) / kGemmBM;
  constexpr uint32_t kStageB = BN * kGemmBK * 2;
  const int num_n = (a.N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  const int ksplit = (EPI == 1 && a.ksplit > 1) ? a.ksplit : 1;
  const int units = tiles * ksplit;  // work unit = (tile, K range)
  if ((int)blockIdx.x >= units) return;
  const int kb_per = (a.K / kGemmBK) / ksplit;

  uint8_t* base = align1024(smem_raw);
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * kStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * kStageB);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const int tile = u / ksplit;
        const int m = tile % num_m, n = tile / num_m;
        const int kb0 = (u - tile * ksplit) * kb_per;
        for (int kb = kb0; kb < kb0 + kb_per; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, a.err, abort_flag, WHERE_GEMM_PRODUCER)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageA + kStageB);
          tma_load_2d_hint(sA + stage * kStageA, &tmA, &full[stage], kb * kGemmBK, m * kGemmBM,
                           pol_a);
          tma_load_2d_hint(sB + stage * kStageB, &tmB, &full[stage], kb * kGemmBK, n * BN,
                           (a.b_keep || num_m > 1 || n < a.b_keep_tiles) ? pol_a : pol_b);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16(kGemmBM, BN, false, false);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
      if (!mbar_wait(&acce[acc], acc_phase ^ 1, a.err, abort_flag, WHERE_GEMM_MMA)) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * BN;
      for (int kb = 0; kb < kb_per; ++kb) {
        if (!mbar_wait(&full[stage], phase, a.err, abort_flag, WHERE_GEMM_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + stage * kStageA);
          const uint32_t b0 = smem_u32(sB + stage * kStageB);
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k) {
            umma_bf16_ss(d, sdesc_sw128(a0 + k * 32, 16, 1024), sdesc_sw128(b0 + k * 32, 16, 1024),
                         idesc, (kb | k) != 0);
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&accf[acc]);
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int tile = u / ksplit;
      const int m = tile % num_m, n = tile / num_m;
      if (!mbar_wait(&accf[acc], acc_phase, a.err, abort_flag, WHERE_GEMM_EPI)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + acc * BN + ((uint32_t)(q * 32) << 16);
      const int row = m * kGemmBM + q * 32 + lane;
      const int ncols = min(BN, a.N - n * BN);
      const int nchunks = (ncols + 31) >> 5;
      if constexpr (EPI == 0) {
        const float c = a.scale_log2;
        float best = -INFINITY, z = 0.f, mu = -INFINITY;
        int bidx = 0;
        for (int ch = 0; ch < nchunks; ++ch) {
          uint32_t r[32];
          tmem_ld32(tbase + ch * 32, r);
          tmem_wait_ld();
          const int lim = ncols - ch * 32;
          float cm = -INFINITY;
          int ci = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float v = __uint_as_float(r[j]);
            if (j < lim && v > cm) {
              cm = v;
              ci = j;
            }
          }
          if (cm > best) {
            best = cm;
            bidx = ch * 32 + ci;
          }
          const float nmu = best * c;
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float e = ex2(fmaf(__uint_as_float(r[j]), c, -nmu));
            s += (j < lim) ? e : 0.f;
          }
          z = (mu == -INFINITY ? 0.f : z * ex2(mu - nmu)) + s;
          mu = nmu;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[acc]);
        if (row < M)
          a.stats[(size_t)row * num_n + n] =
              make_float4(best, z, __int_as_float(n * BN + bidx), 0.f);
      } else if (ksplit == 1) {
        for (int ch = 0; ch < nchunks; ++ch) {
          uint32_t r[32];
          tmem_ld32(tbase + ch * 32, r);
          tmem_wait_ld();
          if (row < M) {
            const int col0 = n * BN + ch * 32;
            uint16_t* dst = a.C + (size_t)row * a.ldc + col0;
            const int lim = ncols - ch * 32;  // multiple of 8 when < 32
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (v * 8 < lim) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                *reinterpret_cast<uint4*>(dst + 8 * v) = w;
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[acc]);
      } else {
        // split-K: store this K range's fp32 partial tile in tile-major
        // order [chunk][4-column group][row][4], so each warp store covers
        // 32 consecutive rows = 512 contiguous bytes.
        const int ks = u - tile * ksplit;
        float* ptile = a.partial + (((size_t)ks * num_m + m) * num_n + n) * (size_t)(BN * kGemmBM);
        const int r = q * 32 + lane;
        for (int ch = 0; ch < nchunks; ++ch) {
          uint32_t rr[32];
          tmem_ld32(tbase + ch * 32, rr);
          tmem_wait_ld();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            __stcg(reinterpret_cast<float4*>(ptile + ((size_t)(ch * 8 + v) * kGemmBM + r) * 4),
                   make_float4(__uint_as_float(rr[4 * v]), __uint_as_float(rr[4 * v + 1]),
                               __uint_as_float(rr[4 * v + 2]), __uint_as_float(rr[4 * v + 3])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[acc]);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Sum of the split-K partials (tile-major, as the split-K epilogue stores
// them) to bf16 C.  Thread = (tile, 32-column chunk, 8-column group, row):
// its reads are coalesced across the warp's consecutive rows.
template <int BN>
__global__ void __launch_bounds__(256)
    splitk_reduce_kernel(const float* __restrict__ partial, int ksplit, int rows, int N,
                         uint16_t* __restrict__ C, int ldc, const int* active) {
  griddep_launch();
  griddep_wait();
  if (active != nullptr && *active == 0) return;
  const int num_m = (rows + kGemmBM - 1) / kGemmBM, num_n = (N + BN - 1) / BN;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int r = (int)(i % kGemmBM);
  long long rest = i / kGemmBM;
  const int g8 = (int)(rest % (BN / 8));  // 8-column group within the tile
  rest /= BN / 8;
  const int n = (int)(rest % num_n), m = (int)(rest / num_n);
  if (m >= num_m) return;
  const int row = m * kGemmBM + r, col = n * BN + g8 * 8;
  if (row >= rows || col >= N) return;
  const size_t plane = (size_t)num_m * num_n * BN * kGemmBM;
  // columns g8*8 .. +7 are the 4-column groups 2*g8 and 2*g8+1 of the tile
  const float* p = partial + ((size_t)m * num_n + n) * (size_t)(BN * kGemmBM) +
                   ((size_t)(2 * g8) * kGemmBM + r) * 4;
  float4 x0 = __ldcg(reinterpret_cast<const float4*>(p));
  float4 x1 = __ldcg(reinterpret_cast<const float4*>(p + kGemmBM * 4));
  for (int k = 1; k < ksplit; ++k) {
    const float4 y0 = __ldcg(reinterpret_cast<const float4*>(p + k * plane));
    const float4 y1 = __ldcg(reinterpret_cast<const float4*>(p + k * plane + kGemmBM * 4));
    x0.x += y0.x; x0.y += y0.y; x0.z += y0.z; x0.w += y0.w;
    x1.x += y1.x; x1.y += y1.y; x1.z += y1.z; x1.w += y1.w;
  }
  uint4 w;
  w.x = pack_bf16x2(x0.x, x0.y);
  w.y = pack_bf16x2(x0.z, x0.w);
  w.z = pack_bf16x2(x1.x, x1.y);
  w.w = pack_bf16x2(x1.z, x1.w);
  *reinterpret_cast<uint4*>(C + (size_t)row * ldc + col) = w;
}

template <int EPI, int BN, int STAGES>
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                        int grid, cudaStream_t st) {
  constexpr size_t smem = gemm_smem_bytes(BN, STAGES);
  static_assert(smem <= 232448, "shared memory per CTA");
  static_assert(2 * BN <= 512, "two accumulators must fit TMEM");
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<EPI, BN, STAGES>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(gemm_kernel<EPI, BN, STAGES>, dim3(grid), dim3(kGemmThreads), smem, st, tmA,
                  tmB, a);
}

}  // namespace

cudaError_t launch_gemm_vocab(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                              int grid, cudaStream_t st) {
  return launch_gemm<0, kVocabBN, kVocabStages>(tmA, tmB, a, grid, st);
}
cudaError_t launch_gemm_bf16(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                             int grid, int bn, cudaStream_t st) {
  if (bn == kQkvBNSmall)
    return launch_gemm<1, kQkvBNSmall, kQkvStagesSmall>(tmA, tmB, a, grid, st);
  return launch_gemm<1, kQkvBN, kQkvStages>(tmA, tmB, a, grid, st);
}

template <int BN>
static cudaError_t launch_reduce(const float* partial, int ksplit, int rows, int N, uint16_t* C,
                                 int ldc, const int* active, cudaStream_t st) {
  const long long tiles = (long long)((rows + kGemmBM - 1) / kGemmBM) * ((N + BN - 1) / BN);
  const long long threads = tiles * (BN / 8) * kGemmBM;
  return launch_k(splitk_reduce_kernel<BN>, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0,
                  st, partial, ksplit, rows, N, C, ldc, active);
}
cudaError_t launch_splitk_reduce(const float* partial, int ksplit, int rows, int N, uint16_t* C,
                                 int ldc, const int* active, int bn, cudaStream_t st) {
  if (bn == kQkvBNSmall)
    return launch_reduce<kQkvBNSmall>(partial, ksplit, rows, N, C, ldc, active, st);
  return launch_reduce<kQkvBN>(partial, ksplit, rows, N, C, ldc, active, st);
}

}  // namespace tt
