// Internal definitions shared by the translation units of libtwotower.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/twotower.h"

namespace tt {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per bounded wait

// Streaming multiprocessors of the current device (cudaDevAttrMultiProcessorCount,
// queried once per device); kDefaultSMs (a B200's count) when no device answers,
// e.g. when workspace sizes are computed on a host without a GPU.
constexpr int kDefaultSMs = 148;
int num_sms();
// Identity of the calling thread's current CUDA context (cuCtxGetId); false
// when no context is current or the driver lacks the call.
bool current_context_id(unsigned long long* id);

// Control block: the first 256 bytes of every workspace.
enum CtrlWord {
  CTRL_ERR = 0,        // first device error code (0 = none)
  CTRL_ERR_WHERE = 1,  // where it was raised (kernel-specific tag)
  CTRL_REMAINING = 2,  // masked positions left (the loop's active flag)
  CTRL_M = 3,          // masked rows of the current step (vocab GEMM rows)
  CTRL_ACTIVE = 4,     // 1 while the loop still has masked positions
  CTRL_STEPS_RUN = 5,  // loop steps that did work
  CTRL_WORDS = 64
};
constexpr size_t kCtrlBytes = CTRL_WORDS * sizeof(int);

// Device-side error tags (CTRL_ERR_WHERE).
enum WhereTag {
  WHERE_GEMM_PRODUCER = 0x100,
  WHERE_GEMM_MMA = 0x101,
  WHERE_GEMM_EPI = 0x102,
  WHERE_ATTN_PRODUCER = 0x200,
  WHERE_ATTN_MMA = 0x201,
  WHERE_ATTN_SOFTMAX = 0x202,
  WHERE_COMMIT_NAN = 0x300,
  WHERE_GATHER_TOKEN = 0x301,
  WHERE_SELFTEST = 0x400,
};

// ------------------------------------------------------------------ GEMM
// C = A[M, K] . B[N, K]^T with both operands K-major bf16, BM=128, BK=64.
// Two epilogues: vocabulary statistics (per row and column tile: max logit,
// sum of exp relative to it, argmax) or a plain bf16 store.  Tile widths: the
// vocabulary GEMM uses N tiles of 224 columns (131072 columns -> 586 tiles,
// 3.96 per SM, so the last round is nearly full) with a 5-deep ring; the
// linear update uses 256-column tiles (4608 columns x 1024 rows -> 144
// tiles, one wave) with a 4-deep ring when the block has several row tiles,
// and 128-column tiles with a 6-deep ring when it has one (the K split that
// fills the SMs is then half as deep, and so are its fp32 partials).
constexpr int kGemmBM = 128, kGemmBK = 64;
constexpr int kVocabBN = 224, kVocabStages = 5;
constexpr int kQkvBN = 256, kQkvStages = 4;
constexpr int kQkvBNSmall = 128, kQkvStagesSmall = 6;
inline int qkv_bn(int rows) { return rows <= kGemmBM ? kQkvBNSmall : kQkvBN; }
constexpr int kGemmThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr size_t gemm_smem_bytes(int bn, int stages) {
  return (size_t)stages * (kGemmBM + bn) * kGemmBK * 2 + 1024 + 256;
}

struct GemmArgs {
  int M_alloc;          // rows present in A's tensor map
  const int* M_dev;     // device row count (nullptr: M_alloc); rows >= M are ignored
  const int* active;    // optional device flag: kernel returns at once if *active == 0
  int N, K;             // N: columns of C (any multiple of 8); K multiple of 64
  // vocabulary-statistics epilogue: stats[row * n_tiles_n + tile] =
  //   {max raw logit, sum exp2(l*c - max*c), argmax column (int bits), 0}
  float4* stats;        // [row][ceil(N / kVocabBN)]
  float scale_log2;     // c = logit_scale * log2(e)
  // bf16 epilogue
  uint16_t* C;
  int ldc;
  // split-K (bf16 epilogue only): K is cut into ksplit ranges handled by
  // different CTAs, each storing its fp32 partial tile to
  // partial[ks][M_alloc][N]; splitk_reduce sums them into C.
  int ksplit;
  float* partial;
  int b_keep;           // 1: load B with evict-last (re-read every loop step and small
                        // enough to stay in L2); 0: streamed, evict-first
  int b_keep_tiles;     // streamed B: the first b_keep_tiles N tiles still use evict-last
  int* err;             // control block
};

cudaError_t launch_gemm_vocab(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                              int grid, cudaStream_t st);
// bn: kQkvBN or kQkvBNSmall (the B tensor map's box height)
cudaError_t launch_gemm_bf16(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a,
                             int grid, int bn, cudaStream_t st);
// C[r, :] = bf16(sum_k partial[k][r][:]) for r < rows (N multiple of 8), the
// partials tile-major in tiles of bn columns.
cudaError_t launch_splitk_reduce(const float* partial, int ksplit, int rows, int N, uint16_t* C,
                                 int ldc, const int* active, int bn, cudaStream_t st);

// ------------------------------------------------------------- attention
constexpr int kAttnBN = 128;       // keys per tile
// warp 0 TMA Q/K, warp 1 TMEM owner and TMA V + V padding, warps 2-3 MMA
// (one per 128-row half), warps 4-11 / 12-19 softmax of half 0 / half 1
constexpr int kAttnThreads = 640;

// A unit is (sequence b, KV head g, query tile qt), u = (b*Hkv + g)*n_qtiles
// + qt.  Its keys form 1 + ceil(L_b / 128) tiles (tile 0: the block's own S
// keys).  All units' tiles laid end to end form T tiles, cut into n_ctas
// contiguous ranges [c*T/n_ctas, (c+1)*T/n_ctas), one per CTA of a
// persistent grid.  The piece of unit u that CTA c runs (a segment) stores
// its partial at slot u + c: along the tile sequence both u and c only grow
// and one of them grows at each new segment, so slots are distinct and
// fewer than units + n_ctas.
struct AttnArgs {
  int B, S, Hq, Hkv, dh, G, L_cap;
  const int* ctx_len;
  const int* active;    // optional device flag
  int s_per_half;       // block positions per 128-row half
  int rows_per_half;    // s_per_half * G
  int halves;           // 128-row halves per query tile (1 or 2)
  int n_qtiles;         // query tiles per (b, g)
  int units;            // B * Hkv * n_qtiles
  int n_ctas;           // CTAs of the persistent grid
  int* tile_start;      // [units + 1] exclusive prefix sums of tiles per unit (device)
  int* first_unit;      // [n_ctas] the unit holding each CTA's first tile (device)
  int4* unit_ctas;      // [units] first and last CTA of the unit's range, how many CTAs
                        // hold a tile of it, and 1 if every CTA in the range does (device)
  int* unit_done;       // [units] segments of the unit finished so far (device; the plan
                        // kernel zeroes it, the CTA that completes a unit resets it)
  int fixup;            // 1: the CTA that completes a unit merges it into `out` (units
                        // span few CTAs); 0: partials only, merged by a separate kernel
  int* merge_list;      // [n_ctas][merge_cap] units each CTA completed (device)
  int merge_cap;        // >= the units any CTA can complete: min(units, ceil(T_max / n_ctas) + 1)
  float scale_log2;     // log2(e) / sqrt(dh)
  uint16_t* out;        // bf16 [B*S, ldo]
  int ldo;
  int kv_keep;          // 1: load K/V with evict-last (small cache re-read every step)
  float* part_o;        // [units + n_ctas - 1][dh/4][256 rows][4] unnormalised partial outputs
  float* part_ml;       // [units + n_ctas - 1][256][4]: running max (log2 units), the row
                        // sums of key columns 0..63 and 64..127 of every tile, unused
  int* err;
  // Optional L2 prefetch of the next vocabulary GEMM's first W tiles (pf_bytes
  // = 0: none): CTA c prefetches the first pf_bytes of each of rows
  // [c * pf_tile, (c + 1) * pf_tile) of W (pf_rows rows, pf_ld bytes apart).
  const uint8_t* pf_base;
  long long pf_ld;
  int pf_rows, pf_tile, pf_bytes;
};
size_t attn_smem_bytes(int dh, int halves);
cudaError_t launch_attn_plan(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKc, const CUtensorMap& tmVc,
                        const CUtensorMap& tmKb, const CUtensorMap& tmVb, const AttnArgs& a,
                        cudaStream_t st);
// Without the fix-up: every unit's segment partials merged into `out`.
cudaError_t launch_attn_merge(const AttnArgs& a, cudaStream_t st);


// ------------------------------------------------------ small kernels
struct PlanArgs {
  int B, S;
  const uint8_t* masked;
  int* rowlist;     // [2*B*S]: compact list of masked rows (b*S+s), then at
                    // B*S + row the compact index of each masked row
  float* t;         // [B]   masked fraction at the start of the step
  int* ctrl;        // writes CTRL_M, CTRL_REMAINING, CTRL_ACTIVE, CTRL_STEPS_RUN
  int count_step;   // unused (kept for layout); steps are counted by the commit kernel
};
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t st);

// masked == nullptr: every row, t[b] per sequence from `t`.  Otherwise (block
// loop) t_b = masked count / S computed in the kernel, and with a row list
// only the masked rows, written compacted (writes rowlist[j] and
// ctrl[CTRL_M]); with rowlist == nullptr every row at its own index (a
// denoiser layer before the last).
cudaError_t launch_adaln(const uint16_t* x, const uint16_t* shift_scale, const float* t,
                         uint16_t* y, int rows, int S, int H, const uint8_t* masked,
                         int* rowlist, int* ctrl, const int* active, cudaStream_t st);

// Block loop without the attention fix-up: the segment merge fused with
// adaLN, with the same row selection as launch_adaln's loop mode.
cudaError_t launch_merge_adaln(const AttnArgs& a, const uint16_t* shift_scale, uint16_t* y,
                               const uint8_t* masked, int* rowlist, int* ctrl, cudaStream_t st);

cudaError_t launch_gather_rows(const uint16_t* src, int ld_src, uint16_t* dst, int H,
                               const int* rowlist, const int* M_dev, int max_rows,
                               const int* active, cudaStream_t st);

cudaError_t launch_embed(const int* tokens, const uint8_t* masked, const uint16_t* emb,
                         const uint16_t* e_mask, uint16_t* dst, int rows, int H, int V,
                         const int* active, int* err, cudaStream_t st);

// The commit runs as B*S CTAs of kCommitThreads (one per block row); the
// last CTA of a sequence to finish (a per-sequence counter) applies the
// commit rule to the whole sequence.
constexpr int kCommitThreads = 256;
struct CommitArgs {
  int B, S, n_vt;
  float2* rowres;       // [B*S] (confidence, token bits) of each row
  int* seqcnt;          // [B] finished CTAs per sequence; zero before the call, left zero
  const float4* stats;  // [compact row][n_vt] tile statistics of the vocab GEMM
  float scale_log2;
  float gamma;
  const int* rowlist;   // compact row -> b*S+s, then b*S+s -> compact row (at B*S + row)
  const int* M_dev;
  int* tokens;
  uint8_t* masked;
  float* conf_out;      // optional [B*S]
  int* argmax_out;      // optional [B*S]
  int* n_committed;     // optional [B]
  int* commit_step;     // optional [B*S]
  int* steps_taken;     // optional [B]
  int step;
  const int* active;
  int* ctrl;
  // loop only: re-embedding of newly committed positions and next-step plan
  const uint16_t* emb;  // [V, H]
  uint16_t* egath;      // [B*S, H] or nullptr
  int H;
  int plan_next;        // 1: decrement ctrl[CTRL_REMAINING] by the commits, count the step
};
cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st);

cudaError_t launch_selftest_wait(int* ctrl, unsigned long long limit_ns, cudaStream_t st);

cudaError_t launch_append_kv(const uint16_t* kv, int ld, uint16_t* k_ctx, uint16_t* v_ctx,
                             int* ctx_len, int B, int S, int Hkv, int dh, int L_cap, int* err,
                             cudaStream_t st);
cudaError_t launch_loop_init(int B, int S, int* steps_taken, int* commit_step, int* ctrl,
                             cudaStream_t st);

// ---------------------------------------------------------------- host
// Tensor-map construction (driver entry point fetched at run time, so the
// library loads without a GPU driver present).
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                  uint32_t b2);

void count_launch(int n = 1);

// Record `msg` as the calling thread's last error and return `s`.
tt_status set_error(tt_status s, const char* msg);
// The shape checks of the public entry points.
tt_status check_dims_public(const tt_dims* d);

// The vocabulary confidence / commit step, shared by the workspace entry
// point and the allocation-free one: argument checks, scratch bytes, and the
// kernel sequence on a caller-chosen 256-byte-aligned scratch area.
tt_status check_vocab_args(const tt_dims* d, const tt_bf16* y, const tt_bf16* w, float gamma,
                           float logit_scale, const int32_t* tokens, const uint8_t* masked);
size_t vocab_scratch_bytes(const tt_dims& d);
tt_status run_vocab_commit(const tt_dims& d, void* scratch, const tt_bf16* y, const tt_bf16* W,
                           float gamma, float logit_scale, int32_t* tokens, uint8_t* masked,
                           float* conf_out, int32_t* argmax_out, int32_t* n_committed,
                           cudaStream_t st);

// Launch with programmatic dependent launch allowed: the kernel may be
// scheduled while its predecessor in the stream is still finishing; every
// kernel of this library executes griddepcontrol.wait before it reads
// anything a predecessor wrote, so only launch latency is overlapped.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  count_launch();
  return e;
}

// Profiler hooks (no-ops unless tt_profile_enable(1)): bracket one launch.
void prof_begin(int kind, cudaStream_t st);
void prof_end(int kind, cudaStream_t st);

}  // namespace tt
