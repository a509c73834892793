// Allocation-free variant of the vocabulary confidence / commit step.
//
// Some callers cannot hand the library a workspace: code that runs inside
// another runtime's execution hook where device allocation is forbidden
// (an inference engine's plugin callback, for instance), a process whose
// device memory is entirely reserved by its own pool, or a C caller with no
// allocator at all.  For them, tt_vocab_confidence_commit_noalloc keeps its
// scratch (masked-row list, gathered rows, per-tile vocabulary statistics)
// in one file-scope device array of kNoAllocScratchBytes, created when the
// library is loaded and held by every GPU that loads it until the process
// exits.  The work itself is the same sequence of kernels as
// tt_vocab_confidence_commit.
#include <cmath>
#include <cstdio>
#include <mutex>

#include "tt_internal.h"

namespace tt {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device

// The scratch.  In host code this name is only a stand-in for the device
// array: its device address must come from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (the first call on each device does this).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_addr_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace tt

using namespace tt;

extern "C" tt_status tt_vocab_confidence_commit_noalloc(
    const tt_dims* d, const tt_bf16* y, const tt_bf16* w, float gamma, float logit_scale,
    int32_t* tokens, uint8_t* masked, float* conf_out, int32_t* argmax_out,
    int32_t* n_committed, void* stream) {
  tt_status s = check_dims_public(d);
  if (s != TT_OK) return s;
  if (y == nullptr || w == nullptr || tokens == nullptr || masked == nullptr)
    return set_error(TT_ERR_INVALID_ARG, "y, w, tokens and masked must not be NULL");
  if ((reinterpret_cast<uintptr_t>(y) & 15u) || (reinterpret_cast<uintptr_t>(w) & 15u))
    return set_error(TT_ERR_INVALID_ARG, "y and w must be 16-byte aligned");
  if (!(gamma > 0.f && gamma <= 1.f)) return set_error(TT_ERR_INVALID_ARG, "gamma not in (0, 1]");
  if (!(logit_scale > 0.f) || !std::isfinite(logit_scale))
    return set_error(TT_ERR_INVALID_ARG, "logit_scale must be finite and > 0");

  // Scratch layout, checked against the built-in maximum before any launch.
  const size_t rows = (size_t)d->B * d->S;
  const size_t n_vt = (size_t)(d->V + kVocabBN - 1) / kVocabBN;
  size_t off = 0;
  const size_t o_ctrl = off;    off = up256(off + kCtrlBytes);
  const size_t o_seq = off;     off = up256(off + (size_t)d->B * sizeof(int));
  const size_t clear_bytes = off;  // control block and sequence counters start at zero
  const size_t o_rows = off;    off = up256(off + 2 * rows * sizeof(int));
  const size_t o_t = off;       off = up256(off + (size_t)d->B * sizeof(float));
  const size_t o_yc = off;      off = up256(off + rows * (size_t)d->H * 2);
  const size_t o_st = off;      off = up256(off + n_vt * rows * sizeof(float4));
  const size_t o_rr = off;      off = up256(off + rows * sizeof(float2));
  if (off > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof msg,
             "needs %zu bytes of scratch; the built-in maximum is %zu bytes "
             "(use tt_vocab_confidence_commit with a workspace)",
             off, kNoAllocScratchBytes);
    return set_error(TT_ERR_WORKSPACE, msg);
  }

  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return set_error(TT_ERR_CUDA, cudaGetErrorString(e));
  uint8_t* sb = static_cast<uint8_t*>(base);
  int* ctrl = reinterpret_cast<int*>(sb + o_ctrl);
  int* rowlist = reinterpret_cast<int*>(sb + o_rows);
  float* tvec = reinterpret_cast<float*>(sb + o_t);
  uint16_t* y_c = reinterpret_cast<uint16_t*>(sb + o_yc);
  float4* stats = reinterpret_cast<float4*>(sb + o_st);
  int* seqcnt = reinterpret_cast<int*>(sb + o_seq);
  float2* rowres = reinterpret_cast<float2*>(sb + o_rr);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // The array keeps the previous call's contents: the control block (row
  // count, error word) and the per-sequence counters must start from zero;
  // everything else is written before it is read.
  e = cudaMemsetAsync(ctrl, 0, clear_bytes, st);
  if (e != cudaSuccess) return set_error(TT_ERR_CUDA, cudaGetErrorString(e));

  PlanArgs p{d->B, d->S, masked, rowlist, tvec, ctrl, 0};
  if ((e = launch_plan(p, st)) != cudaSuccess) return set_error(TT_ERR_CUDA, cudaGetErrorString(e));
  if ((e = launch_gather_rows(y, d->H, y_c, d->H, rowlist, ctrl + CTRL_M, (int)rows, nullptr,
                              st)) != cudaSuccess)
    return set_error(TT_ERR_CUDA, cudaGetErrorString(e));

  CUtensorMap tmA, tmB;
  if (!make_tmap_2d(&tmA, y_c, d->H, rows, (uint64_t)d->H * 2, kGemmBK, kGemmBM) ||
      !make_tmap_2d(&tmB, w, d->H, d->V, (uint64_t)d->H * 2, kGemmBK, kVocabBN))
    return set_error(TT_ERR_CUDA, "cuTensorMapEncodeTiled failed for the vocab GEMM");
  GemmArgs g{};
  g.M_alloc = (int)rows;
  g.M_dev = ctrl + CTRL_M;
  g.N = d->V;
  g.K = d->H;
  g.stats = stats;
  g.scale_log2 = (float)(logit_scale * 1.4426950408889634);
  g.err = ctrl;
  const int tiles = (int)(((rows + kGemmBM - 1) / kGemmBM) * n_vt);
  if ((e = launch_gemm_vocab(tmA, tmB, g, tiles < kNumSMs ? tiles : kNumSMs, st)) != cudaSuccess)
    return set_error(TT_ERR_CUDA, cudaGetErrorString(e));

  CommitArgs c{};
  c.B = d->B;
  c.S = d->S;
  c.n_vt = (int)n_vt;
  c.stats = stats;
  c.scale_log2 = g.scale_log2;
  c.gamma = gamma;
  c.rowlist = rowlist;
  c.rowres = rowres;
  c.seqcnt = seqcnt;
  c.M_dev = ctrl + CTRL_M;
  c.tokens = tokens;
  c.masked = masked;
  c.conf_out = conf_out;
  c.argmax_out = argmax_out;
  c.n_committed = n_committed;
  c.ctrl = ctrl;
  if ((e = launch_commit(c, st)) != cudaSuccess) return set_error(TT_ERR_CUDA, cudaGetErrorString(e));
  return TT_OK;
}
