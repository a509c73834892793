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
// swizzled 64-column boxes (A: 128 rows, B: 256 rows per stage).  One CTA per
// SM walks tiles m-fastest, so the CTAs that share a W tile run together and
// W crosses HBM once.  Warp 0 issues TMA, warp 1 issues tcgen05.mma
// (M=128, N=256, K=16) into one of two 256-column TMEM accumulators, warps
// 2..5 drain the other accumulator (TMEM lane = tile row).
#include <math.h>

#include "tt_ptx.cuh"

namespace tt {

namespace {

constexpr uint32_t kStageA = kGemmBM * kGemmBK * 2;  // 16 KB
constexpr uint32_t kStageB = kGemmBN * kGemmBK * 2;  // 32 KB

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int EPI>  // 0: vocabulary statistics, 1: bf16 store
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  if (a.active != nullptr && *a.active == 0) return;
  const int M = a.M_dev != nullptr ? min(*a.M_dev, a.M_alloc) : a.M_alloc;
  if (M <= 0) return;
  const int num_m = (M + kGemmBM - 1) / kGemmBM;
  const int num_n = (a.N + kGemmBN - 1) / kGemmBN;
  const int tiles = num_m * num_n;
  if ((int)blockIdx.x >= tiles) return;
  const int kb_n = a.K / kGemmBK;

  uint8_t* base = align1024(smem_raw);
  uint8_t* sA = base;
  uint8_t* sB = base + kGemmStages * kStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGemmStages * kStageB);
  uint64_t* empty = full + kGemmStages;
  uint64_t* accf = empty + kGemmStages;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
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
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
        const int m = tile % num_m, n = tile / num_m;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, a.err, abort_flag, WHERE_GEMM_PRODUCER)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageA + kStageB);
          tma_load_2d_hint(sA + stage * kStageA, &tmA, &full[stage], kb * kGemmBK, m * kGemmBM,
                           pol_a);
          tma_load_2d_hint(sB + stage * kStageB, &tmB, &full[stage], kb * kGemmBK, n * kGemmBN,
                           num_m == 1 ? pol_b : pol_a);
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16(kGemmBM, kGemmBN, false, false);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
      if (!mbar_wait(&acce[acc], acc_phase ^ 1, a.err, abort_flag, WHERE_GEMM_MMA)) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * kGemmBN;
      for (int kb = 0; kb < kb_n; ++kb) {
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
        if (++stage == kGemmStages) {
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
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
      const int m = tile % num_m, n = tile / num_m;
      if (!mbar_wait(&accf[acc], acc_phase, a.err, abort_flag, WHERE_GEMM_EPI)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + acc * kGemmBN + ((uint32_t)(q * 32) << 16);
      const int row = m * kGemmBM + q * 32 + lane;
      const int ncols = min(kGemmBN, a.N - n * kGemmBN);
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
        if (row < M) {
          const size_t o = (size_t)n * a.part_ld + row;
          a.part_v[o] = best;
          a.part_z[o] = z;
          a.part_a[o] = n * kGemmBN + bidx;
        }
      } else {
        for (int ch = 0; ch < nchunks; ++ch) {
          uint32_t r[32];
          tmem_ld32(tbase + ch * 32, r);
          tmem_wait_ld();
          if (row < M) {
            const int col0 = n * kGemmBN + ch * 32;
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

template <int EPI>
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                        int grid, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<EPI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGemmSmemBytes);
  if (e != cudaSuccess) return e;
  gemm_kernel<EPI><<<grid, kGemmThreads, kGemmSmemBytes, st>>>(tmA, tmB, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_vocab(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                              int grid, cudaStream_t st) {
  return launch_gemm<0>(tmA, tmB, a, grid, st);
}
cudaError_t launch_gemm_bf16(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                             int grid, cudaStream_t st) {
  return launch_gemm<1>(tmA, tmB, a, grid, st);
}

}  // namespace tt
