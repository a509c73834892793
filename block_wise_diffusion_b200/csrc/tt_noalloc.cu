// Allocation-free variant of the vocabulary confidence / commit step.
//
// Some callers cannot hand the library a workspace: code that runs inside
// another runtime's execution hook where device allocation is forbidden
// (an inference engine's plugin callback, for instance), a process whose
// device memory is entirely reserved by its own pool, or a C caller with no
// allocator at all.  For them, tt_vocab_confidence_commit_noalloc keeps its
// scratch (control words, masked-row list, gathered rows, per-tile
// vocabulary statistics, per-row results) in one file-scope device array of
// kNoAllocScratchBytes, created when the library is loaded and held by every
// GPU that loads it until the process exits.  The work itself is the kernel
// sequence of tt_vocab_confidence_commit (run_vocab_commit), carved from the
// array instead of a caller's workspace.
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
struct AddrSlot {
  unsigned long long ctx_id;  // context the address belongs to (0: none)
  void* addr;
};
std::mutex g_addr_mu;
AddrSlot g_addr[kMaxDevices] = {};

// Device address of the scratch on the current device.  It is looked up
// (cudaGetSymbolAddress, with the device current) on the first call on each
// device, and again whenever the current context is not the one the cached
// address belongs to (after a device reset the module, and with it the
// array, is loaded anew).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lk(g_addr_mu);
  if (have_id && g_addr[dev].addr != nullptr && g_addr[dev].ctx_id == id) {
    *out = g_addr[dev].addr;
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the primary context current
  if (e != cudaSuccess) return e;
  if (!have_id) have_id = current_context_id(&id);
  // without a context identity nothing is cached: the next call looks up again
  g_addr[dev] = have_id ? AddrSlot{id, p} : AddrSlot{0, nullptr};
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace tt

using namespace tt;

extern "C" tt_status tt_vocab_confidence_commit_noalloc(
    const tt_dims* d, const tt_bf16* y, const tt_bf16* w, float gamma, float logit_scale,
    int32_t* tokens, uint8_t* masked, float* conf_out, int32_t* argmax_out,
    int32_t* n_committed, void* stream) {
  tt_status s = check_vocab_args(d, y, w, gamma, logit_scale, tokens, masked);
  if (s != TT_OK) return s;
  // The scratch this problem needs (the workspace tt_vocab_confidence_commit
  // would take), checked against the built-in maximum before any CUDA call.
  const size_t need = vocab_scratch_bytes(*d);
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof msg,
             "needs %zu bytes of scratch; the built-in maximum is %zu bytes "
             "(use tt_vocab_confidence_commit with a workspace)",
             need, kNoAllocScratchBytes);
    return set_error(TT_ERR_WORKSPACE, msg);
  }
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return set_error(TT_ERR_CUDA, cudaGetErrorString(e));
  // The array keeps the previous call's contents; run_vocab_commit clears
  // the control block and the per-sequence counters, and writes everything
  // else before reading it.
  return run_vocab_commit(*d, base, y, w, gamma, logit_scale, tokens, masked, conf_out,
                          argmax_out, n_committed, reinterpret_cast<cudaStream_t>(stream));
}
