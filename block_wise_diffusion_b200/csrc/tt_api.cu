// C ABI of libtwotower: argument validation, workspace carving, tensor-map
// construction and kernel sequencing.  All compute happens in the kernels of
// tt_attn.cu, tt_gemm.cu and tt_small.cu.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "tt_internal.h"

namespace tt {

static thread_local char g_err[512];
static std::atomic<uint64_t> g_launches{0};
static thread_local uint64_t t_launches = 0;  // this thread's launches (graph capture bookkeeping)
static std::atomic<int> g_forced_splits{0};

void count_launch(int n) {
  g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed);
  t_launches += (uint64_t)n;
}

int num_sms() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();  // no device here: clear the error and use the default
    return kDefaultSMs;
  }
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return kDefaultSMs;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Identity of the calling thread's current CUDA context (cuCtxGetId: unique
// for the life of the process, so a context destroyed by a device reset and
// created again gets a new one).  False when no context is current yet or
// the driver lacks the call.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_cur == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- profiler
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
static std::mutex g_prof_mu;
static std::atomic<bool> g_prof_on{false};
static std::vector<ProfRec> g_prof_pending;
static std::vector<cudaEvent_t> g_prof_free;
static double g_prof_ms[TT_K_COUNT];
static int64_t g_prof_n[TT_K_COUNT];
static thread_local cudaEvent_t g_prof_open = nullptr;

static cudaEvent_t prof_event() {
  if (!g_prof_free.empty()) {
    cudaEvent_t e = g_prof_free.back();
    g_prof_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void prof_begin(int kind, cudaStream_t st) {
  (void)kind;
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_open = prof_event();
  if (g_prof_open) cudaEventRecord(g_prof_open, st);
}

void prof_end(int kind, cudaStream_t st) {
  if (!g_prof_on.load(std::memory_order_relaxed) || g_prof_open == nullptr) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t e = prof_event();
  if (e == nullptr) return;
  cudaEventRecord(e, st);
  g_prof_pending.push_back({kind, g_prof_open, e});
  g_prof_open = nullptr;
}

static void prof_harvest() {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (const ProfRec& r : g_prof_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      g_prof_ms[r.kind] += ms;
      g_prof_n[r.kind] += 1;
    }
    g_prof_free.push_back(r.a);
    g_prof_free.push_back(r.b);
  }
  g_prof_pending.clear();
}

static tt_status fail(tt_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

#define TT_LAUNCH(kind, st, call) \
  do {                             \
    prof_begin((kind), (st));      \
    TT_CUDA(call);                 \
    prof_end((kind), (st));        \
  } while (0)

#define TT_CUDA(call)                                                                      \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess)                                                                 \
      return fail(TT_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),     \
                  __FILE__, __LINE__);                                                     \
  } while (0)

// --------------------------------------------------------------- tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                  uint32_t b2) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- checks
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static tt_status check_dims(const tt_dims* d) {
  if (d == nullptr) return fail(TT_ERR_INVALID_ARG, "dims is NULL");
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->V < 2 || d->L_cap < 0)
    return fail(TT_ERR_INVALID_ARG, "bad sizes: B=%d Hq=%d Hkv=%d V=%d L_cap=%d", d->B, d->Hq,
                d->Hkv, d->V, d->L_cap);
  // S = 1 is the autoregressive baseline step (one position per block)
  if (d->S != 1 && d->S != 16 && d->S != 32 && d->S != 64 && d->S != 128)
    return fail(TT_ERR_UNSUPPORTED, "S=%d not in {1,16,32,64,128}", d->S);
  if (d->dh != 64 && d->dh != 128)
    return fail(TT_ERR_UNSUPPORTED, "dh=%d not in {64,128}", d->dh);
  if (d->Hq % d->Hkv != 0)
    return fail(TT_ERR_INVALID_ARG, "Hq=%d not a multiple of Hkv=%d", d->Hq, d->Hkv);
  const int G = d->Hq / d->Hkv;
  if (G > 128 || (G & (G - 1)) != 0)
    return fail(TT_ERR_UNSUPPORTED, "G=Hq/Hkv=%d must be a power of two <= 128", G);
  if (d->H != d->Hq * d->dh)
    return fail(TT_ERR_INVALID_ARG, "H=%d != Hq*dh=%d", d->H, d->Hq * d->dh);
  if (d->H % 64 != 0 || d->H > 8192)
    return fail(TT_ERR_UNSUPPORTED, "H=%d must be a multiple of 64 and <= 8192", d->H);
  if ((long long)d->B * d->Hkv * d->L_cap >= (1ll << 31) || (long long)d->B * d->S >= (1 << 24) ||
      (long long)d->V * d->H >= (1ll << 40))
    return fail(TT_ERR_UNSUPPORTED, "problem too large");
  return TT_OK;
}

static tt_status check_ptr(const void* p, const char* name, bool need16) {
  if (p == nullptr) return fail(TT_ERR_INVALID_ARG, "%s is NULL", name);
  if (need16 && !aligned16(p)) return fail(TT_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return TT_OK;
}
#define TT_CHECK(x)               \
  do {                            \
    tt_status s_ = (x);           \
    if (s_ != TT_OK) return s_;   \
  } while (0)

// ------------------------------------------------------------ geometry
struct AttnGeom {
  int G, s_per_half, rows_per_half, halves, n_qtiles, units, n_ctas, slots, merge_cap, fixup;
  size_t part_o_bytes, part_ml_bytes;
};

// Query packing (S positions x G heads in 128-row halves) and the persistent
// grid: one CTA per SM unless tt_set_attn_splits fixed the count.
static AttnGeom attn_geom(const tt_dims& d) {
  AttnGeom g;
  g.G = d.Hq / d.Hkv;
  g.s_per_half = std::min(d.S, 128 / g.G);
  g.rows_per_half = g.s_per_half * g.G;
  g.halves = std::min(2, d.S / g.s_per_half);
  g.n_qtiles = d.S / (g.halves * g.s_per_half);
  g.units = d.B * d.Hkv * g.n_qtiles;
  const int forced = g_forced_splits.load();
  g.n_ctas = forced > 0 ? forced : num_sms();
  g.slots = g.units + g.n_ctas - 1;
  // With at least half as many units as CTAs a unit spans about three CTAs
  // at most and the CTA that completes it merges it cheaply (the fix-up);
  // with fewer, units span many CTAs and one SM merging megabytes of
  // partials would trail the kernel, so a merge over the whole GPU follows.
  g.fixup = 2 * g.units >= g.n_ctas ? 1 : 0;
  // A CTA completes a unit only when the unit's last tile is in its range, and
  // every unit has a tile: at most its range's tiles, at most ceil(T / CTAs)
  // with T <= units * (1 + ceil(L_cap / 128)).
  const long long t_max = (long long)g.units * (1 + (d.L_cap + kAttnBN - 1) / kAttnBN);
  g.merge_cap = (int)std::min<long long>(g.units, (t_max + g.n_ctas - 1) / g.n_ctas + 1);
  g.part_o_bytes = (size_t)g.slots * 256 * d.dh * sizeof(float);
  g.part_ml_bytes = (size_t)g.slots * 256 * 4 * sizeof(float);
  return g;
}

// K splits of the linear-update GEMM: enough (tile, K range) units to fill
// the SMs when the block has few rows; a power of two dividing H/64.
static int ksplit_for(const tt_dims& d, int n_out) {
  const int rows = d.B * d.S;
  const int bn = qkv_bn(rows);
  const int tiles = ((rows + kGemmBM - 1) / kGemmBM) * ((n_out + bn - 1) / bn);
  const int kb = d.H / kGemmBK;
  const int sms = num_sms();
  int k = 1;
  while (2 * k <= kb && kb % (2 * k) == 0 && tiles * 2 * k <= sms) k *= 2;
  return k;
}
static int qkv_ksplit(const tt_dims& d) { return ksplit_for(d, d.H + 2 * d.Hkv * d.dh); }
// the projection of a committed block into the context: [k | v] per position
static int ctx_ksplit(const tt_dims& d) { return ksplit_for(d, 2 * d.Hkv * d.dh); }
static size_t splitk_bytes(const tt_dims& d, int n_out, int ks) {
  const size_t rows = (size_t)d.B * d.S;
  const size_t bn = (size_t)qkv_bn((int)rows);
  const size_t tiles = ((rows + kGemmBM - 1) / kGemmBM) * ((n_out + bn - 1) / bn);
  return ks > 1 ? (size_t)ks * tiles * kGemmBM * bn * sizeof(float) : 0;
}

struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <class T>
  T* take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += bytes;
    return p;
  }
};

struct Ws {
  int* ctrl = nullptr;
  int* rowlist = nullptr;
  float* tvec = nullptr;
  uint16_t* egath = nullptr;
  uint16_t* qkv = nullptr;
  uint16_t* y_c = nullptr;
  float* part_o = nullptr;
  float* part_ml = nullptr;
  int* tile_start = nullptr;   // attention plan: tiles per unit, prefix sums
  int* first_unit = nullptr;   // attention plan: first unit of each CTA
  int4* unit_ctas = nullptr;   // attention plan: first and last CTA of each unit, CTA count
  int* unit_done = nullptr;    // attention fix-up: finished segments per unit
  int* merge_list = nullptr;   // attention fix-up: units each CTA completed
  uint16_t* attn_out = nullptr;  // loop: the attention output rows
  float4* stats = nullptr;
  float* qkv_partial = nullptr;
  uint16_t* xrows = nullptr;  // loop: one layer's modulated rows for the next layer
  uint8_t* blk_masked = nullptr;  // block after block: the current block's mask
  int* seqcnt = nullptr;     // follows ctrl directly: cleared together
  float2* rowres = nullptr;
  size_t ctrl_clear = kCtrlBytes;  // bytes from ctrl to clear at the start of a call
  size_t total = 0;
};

static Ws carve(const tt_dims& d, int which, void* ws) {
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  Ws w;
  const size_t rows = (size_t)d.B * d.S;
  const size_t n_vt = (size_t)(d.V + kVocabBN - 1) / kVocabBN;
  w.ctrl = c.take<int>(kCtrlBytes);
  if (which == TT_WS_VOCAB || which == TT_WS_LOOP) {
    w.seqcnt = c.take<int>((size_t)d.B * sizeof(int));
    w.ctrl_clear = c.off;
  }
  if (which == TT_WS_ATTN || which == TT_WS_LOOP) {
    const AttnGeom g = attn_geom(d);
    w.tile_start = c.take<int>((size_t)(g.units + 1) * sizeof(int));
    w.first_unit = c.take<int>((size_t)g.n_ctas * sizeof(int));
    w.unit_ctas = c.take<int4>((size_t)g.units * sizeof(int4));
    w.unit_done = c.take<int>((size_t)g.units * sizeof(int));
    w.merge_list = c.take<int>((size_t)g.n_ctas * g.merge_cap * sizeof(int));
    w.part_o = c.take<float>(g.part_o_bytes);
    w.part_ml = c.take<float>(g.part_ml_bytes);
  }
  if (which == TT_WS_VOCAB || which == TT_WS_LOOP) {
    w.rowlist = c.take<int>(2 * rows * sizeof(int));
    w.tvec = c.take<float>((size_t)d.B * sizeof(float));
    w.y_c = c.take<uint16_t>(rows * d.H * 2);
    w.stats = c.take<float4>(n_vt * rows * sizeof(float4));
    w.rowres = c.take<float2>(rows * sizeof(float2));
  }
  if (which == TT_WS_LOOP) {
    const size_t n_qkv = (size_t)d.H + 2 * (size_t)d.Hkv * d.dh;
    w.egath = c.take<uint16_t>(rows * d.H * 2);
    w.xrows = c.take<uint16_t>(rows * d.H * 2);
    w.qkv = c.take<uint16_t>(rows * n_qkv * 2);
    w.attn_out = c.take<uint16_t>(rows * d.H * 2);
    // tile-major partials: ks planes of whole 128 x qkv_bn(rows) tiles, for the
    // linear update or the context projection, whichever needs more
    const size_t pb = std::max(splitk_bytes(d, (int)n_qkv, qkv_ksplit(d)),
                               splitk_bytes(d, 2 * d.Hkv * d.dh, ctx_ksplit(d)));
    if (pb) w.qkv_partial = c.take<float>(pb);
    w.blk_masked = c.take<uint8_t>(rows);
  }
  w.total = (c.off + 255) & ~size_t(255);
  return w;
}

static tt_status check_ws(const tt_dims& d, int which, void* ws, size_t ws_bytes, Ws* out) {
  TT_CHECK(check_ptr(ws, "ws", true));
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(TT_ERR_INVALID_ARG, "ws is not 256-byte aligned");
  *out = carve(d, which, ws);
  if (ws_bytes < out->total)
    return fail(TT_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, out->total);
  return TT_OK;
}

tt_status set_error(tt_status s, const char* msg) { return fail(s, "%s", msg); }
tt_status check_dims_public(const tt_dims* d) { return check_dims(d); }

// ---------------------------------------------------------- stage helpers
struct AttnMaps {
  CUtensorMap q, kc, vc, kb, vb;
};

static tt_status build_attn_maps(const tt_dims& d, const AttnGeom& g, const tt_bf16* q, int ldq,
                                 const tt_bf16* kb, const tt_bf16* vb, int ldkv,
                                 const tt_bf16* kc, const tt_bf16* vc, AttnMaps* m) {
  const uint64_t rows_ctx = (uint64_t)d.B * d.Hkv * std::max(d.L_cap, 1);
  bool ok = make_tmap_3d(&m->q, q, d.dh, d.Hq, (uint64_t)d.B * d.S, (uint64_t)d.dh * 2,
                         (uint64_t)ldq * 2, 64, g.G, g.s_per_half) &&
            make_tmap_3d(&m->kb, kb, d.dh, d.Hkv, (uint64_t)d.B * d.S, (uint64_t)d.dh * 2,
                         (uint64_t)ldkv * 2, 64, 1, d.S) &&
            make_tmap_3d(&m->vb, vb, d.dh, d.Hkv, (uint64_t)d.B * d.S, (uint64_t)d.dh * 2,
                         (uint64_t)ldkv * 2, 64, 1, d.S) &&
            make_tmap_2d(&m->kc, kc, d.dh, rows_ctx, (uint64_t)d.dh * 2, 64, kAttnBN) &&
            make_tmap_2d(&m->vc, vc, d.dh, rows_ctx, (uint64_t)d.dh * 2, 64, kAttnBN);
  if (!ok) return fail(TT_ERR_CUDA, "cuTensorMapEncodeTiled failed for the attention operands");
  return TT_OK;
}

static AttnArgs attn_args(const tt_dims& d, const AttnGeom& g, const int32_t* ctx_len,
                          tt_bf16* out, const Ws& w, const int* active) {
  AttnArgs a{};  // every field not set below (the optional prefetch) is zero
  a.B = d.B;
  a.S = d.S;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.dh = d.dh;
  a.G = g.G;
  a.L_cap = d.L_cap;
  a.ctx_len = ctx_len;
  a.active = active;
  a.s_per_half = g.s_per_half;
  a.rows_per_half = g.rows_per_half;
  a.halves = g.halves;
  a.n_qtiles = g.n_qtiles;
  a.units = g.units;
  a.n_ctas = g.n_ctas;
  a.tile_start = w.tile_start;
  a.first_unit = w.first_unit;
  a.unit_ctas = w.unit_ctas;
  a.unit_done = w.unit_done;
  a.fixup = g.fixup;
  a.merge_list = w.merge_list;
  a.merge_cap = g.merge_cap;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d.dh));
  a.out = out;
  a.ldo = d.H;
  a.part_o = w.part_o;
  a.part_ml = w.part_ml;
  a.err = w.ctrl;
  // keep a small context cache in L2 across loop steps (the vocab stream
  // uses evict-first, so up to ~64 MB of re-read operands can stay resident)
  a.kv_keep = (active != nullptr &&
               2.0 * d.B * d.Hkv * (double)d.L_cap * d.dh * 2 <= 48.0 * (1 << 20)) ? 1 : 0;
  return a;
}

// In a loop whose vocabulary GEMM has one row tile (B*S <= 128 rows) the
// GEMM streams W from HBM while the kernels before it leave HBM mostly idle
// when the context sits in L2.  The attention then prefetches into L2 the
// first kVocabPrefetchBytes of every W row of the GEMM's first wave (CTA c
// of the GEMM starts on the W tile c), a balanced head start of 34 MB at
// V = 131072, H = 4096.
#ifndef TT_VOCAB_PF_BYTES
#define TT_VOCAB_PF_BYTES 1024
#endif
constexpr int kVocabPrefetchBytes = TT_VOCAB_PF_BYTES;
static bool vocab_prefetch(const tt_dims& d, const AttnArgs& a) {
  return a.kv_keep && d.B * d.S <= kGemmBM && (double)d.V * d.H * 2 >= 64.0 * (1 << 20);
}

// The attention's tile plan (prefix sums of tiles per unit from the device
// context lengths, first unit of each CTA): once per call, since ctx_len does
// not change within one.
static tt_status run_attn_plan(const tt_dims& d, const AttnGeom& g, const int32_t* ctx_len,
                               const Ws& w, cudaStream_t st) {
  const AttnArgs a = attn_args(d, g, ctx_len, nullptr, w, nullptr);
  TT_LAUNCH(TT_K_ATTN_PLAN, st, launch_attn_plan(a, st));
  return TT_OK;
}

// The attention launch.  With the fix-up the kernel writes the bf16 output
// to `out`; otherwise, with `merge`, a merge kernel does (the loop fuses that
// merge into adaLN instead).
// `pf_w` (optional): the W the next vocabulary GEMM streams; see vocab_prefetch.
static tt_status run_attn(const tt_dims& d, const AttnGeom& g, const AttnMaps& m,
                          const int32_t* ctx_len, tt_bf16* out, const Ws& w, const int* active,
                          bool merge, cudaStream_t st, const tt_bf16* pf_w = nullptr) {
  AttnArgs a = attn_args(d, g, ctx_len, out, w, active);
  if (pf_w != nullptr && kVocabPrefetchBytes > 0) {
    a.pf_base = reinterpret_cast<const uint8_t*>(pf_w);
    a.pf_ld = (long long)d.H * 2;
    a.pf_rows = d.V;
    a.pf_tile = kVocabBN;
    a.pf_bytes = std::min(kVocabPrefetchBytes, d.H * 2);
  }
  TT_LAUNCH(TT_K_ATTN, st, launch_attn(m.q, m.kc, m.vc, m.kb, m.vb, a, st));
  if (merge && !g.fixup) TT_LAUNCH(TT_K_MERGE, st, launch_attn_merge(a, st));
  return TT_OK;
}

static tt_status run_vocab_gemm(const tt_dims& d, const Ws& w, const tt_bf16* W,
                                float logit_scale, const int* M_dev, const int* active,
                                int keep_tiles, cudaStream_t st) {
  const int rows = d.B * d.S;
  CUtensorMap tmA, tmB;
  if (!make_tmap_2d(&tmA, w.y_c, d.H, rows, (uint64_t)d.H * 2, kGemmBK, kGemmBM) ||
      !make_tmap_2d(&tmB, W, d.H, d.V, (uint64_t)d.H * 2, kGemmBK, kVocabBN))
    return fail(TT_ERR_CUDA, "cuTensorMapEncodeTiled failed for the vocab GEMM");
  GemmArgs a{};
  a.M_alloc = rows;
  a.M_dev = M_dev;
  a.active = active;
  a.N = d.V;
  a.K = d.H;
  a.stats = w.stats;
  a.scale_log2 = (float)(logit_scale * 1.4426950408889634);
  a.err = w.ctrl;
  a.b_keep_tiles = keep_tiles;
  const int tiles = ((rows + kGemmBM - 1) / kGemmBM) * ((d.V + kVocabBN - 1) / kVocabBN);
  TT_LAUNCH(TT_K_GEMM_VOCAB, st, launch_gemm_vocab(tmA, tmB, a, std::min(tiles, num_sms()), st));
  return TT_OK;
}

static CommitArgs commit_args(const tt_dims& d, const Ws& w, float gamma, float logit_scale,
                              int32_t* tokens, uint8_t* masked) {
  CommitArgs c{};
  c.B = d.B;
  c.S = d.S;
  c.n_vt = (d.V + kVocabBN - 1) / kVocabBN;
  c.stats = w.stats;
  c.scale_log2 = (float)(logit_scale * 1.4426950408889634);
  c.gamma = gamma;
  c.rowlist = w.rowlist;
  c.rowres = w.rowres;
  c.seqcnt = w.seqcnt;
  c.M_dev = w.ctrl + CTRL_M;
  c.tokens = tokens;
  c.masked = masked;
  c.ctrl = w.ctrl;
  return c;
}

static tt_status read_ctrl(const Ws& w, cudaStream_t st, int* host) {
  TT_CUDA(cudaMemcpyAsync(host, w.ctrl, 8 * sizeof(int), cudaMemcpyDeviceToHost, st));
  TT_CUDA(cudaStreamSynchronize(st));
  return TT_OK;
}

tt_status check_vocab_args(const tt_dims* d, const tt_bf16* y, const tt_bf16* w, float gamma,
                           float logit_scale, const int32_t* tokens, const uint8_t* masked) {
  TT_CHECK(check_dims(d));
  TT_CHECK(check_ptr(y, "y", true));
  TT_CHECK(check_ptr(w, "w", true));
  TT_CHECK(check_ptr(tokens, "tokens", false));
  TT_CHECK(check_ptr(masked, "masked", false));
  if (!(gamma > 0.f && gamma <= 1.f))
    return fail(TT_ERR_INVALID_ARG, "gamma=%g not in (0, 1]", (double)gamma);
  if (!(logit_scale > 0.f) || !std::isfinite(logit_scale))
    return fail(TT_ERR_INVALID_ARG, "logit_scale=%g must be finite and > 0", (double)logit_scale);
  return TT_OK;
}

size_t vocab_scratch_bytes(const tt_dims& d) { return carve(d, TT_WS_VOCAB, nullptr).total; }

// Plan -> row gather -> vocabulary GEMM with the confidence epilogue ->
// commit, with the scratch carved from `scratch` (256-byte aligned, at least
// vocab_scratch_bytes(d) bytes; the arguments already checked).
tt_status run_vocab_commit(const tt_dims& d, void* scratch, const tt_bf16* y, const tt_bf16* W,
                           float gamma, float logit_scale, int32_t* tokens, uint8_t* masked,
                           float* conf_out, int32_t* argmax_out, int32_t* n_committed,
                           cudaStream_t st) {
  const Ws w = carve(d, TT_WS_VOCAB, scratch);
  TT_CUDA(cudaMemsetAsync(w.ctrl, 0, w.ctrl_clear, st));
  PlanArgs p{d.B, d.S, masked, w.rowlist, w.tvec, w.ctrl, 0};
  TT_LAUNCH(TT_K_PLAN, st, launch_plan(p, st));
  TT_LAUNCH(TT_K_GATHER, st, launch_gather_rows(y, d.H, w.y_c, d.H, w.rowlist, w.ctrl + CTRL_M,
                                                d.B * d.S, nullptr, st));
  TT_CHECK(run_vocab_gemm(d, w, W, logit_scale, w.ctrl + CTRL_M, nullptr, 0, st));
  CommitArgs c = commit_args(d, w, gamma, logit_scale, tokens, masked);
  c.conf_out = conf_out;
  c.argmax_out = argmax_out;
  c.n_committed = n_committed;
  TT_LAUNCH(TT_K_COMMIT, st, launch_commit(c, st));
  return TT_OK;
}

// ------------------------------------------------------------ loop graphs
// The block loop enqueues five or six kernels per step.  A host thread that
// is slow to issue them (a busy host) leaves the GPU idle between them, so
// each distinct argument set is captured once into a CUDA graph and replayed:
// one launch per call, the same kernels with the same arguments (programmatic
// launch edges included), so results are bitwise those of direct launches.
// Captured on a library stream of the calling device, replayed on the
// caller's; keyed by every argument, the attention's CTA count, the device
// and its context identity; at most kMaxLoopGraphs kept, least recently used
// dropped first.  Off while the profiler is on (it brackets each launch).
struct LoopKey {
  tt_dims d;
  int n_layers, max_steps, n_ctas, dev;
  unsigned long long ctx;
  const void* p[14];
  size_t ws_bytes;
  uint32_t gamma_bits, scale_bits;
};
struct LoopGraph {
  LoopKey key;
  cudaGraphExec_t exec;
  uint64_t launches, last_use;
  int users;
};
constexpr size_t kMaxLoopGraphs = 32;
constexpr int kMaxGraphDevices = 64;
static std::mutex g_graph_mu;
static std::vector<LoopGraph> g_graphs;
static uint64_t g_graph_clock = 0;
static std::atomic<bool> g_graphs_on{true};
struct CapStream {
  unsigned long long ctx;
  cudaStream_t s;
};
static CapStream g_cap[kMaxGraphDevices];

static bool key_eq(const LoopKey& a, const LoopKey& b) { return std::memcmp(&a, &b, sizeof a) == 0; }

// The cached graph for `k`, marked in use (release with graph_release), or
// nullptr.
static LoopGraph* graph_acquire(const LoopKey& k) {
  std::lock_guard<std::mutex> lk(g_graph_mu);
  for (LoopGraph& e : g_graphs)
    if (key_eq(e.key, k)) {
      e.last_use = ++g_graph_clock;
      ++e.users;
      return &e;
    }
  return nullptr;
}
static void graph_release(LoopGraph* e) {
  std::lock_guard<std::mutex> lk(g_graph_mu);
  --e->users;
}
// Adds a graph (in use by the caller), replacing the least recently used
// idle entry when full.  Every replay of a replaced graph has completed: each
// loop call waits for its stream before it returns.
static LoopGraph* graph_insert(const LoopKey& k, cudaGraphExec_t exec, uint64_t launches) {
  std::lock_guard<std::mutex> lk(g_graph_mu);
  // capacity fixed before the first entry: entries never move while in use
  if (g_graphs.capacity() < kMaxLoopGraphs) g_graphs.reserve(kMaxLoopGraphs);
  if (g_graphs.size() < kMaxLoopGraphs) {
    g_graphs.push_back(LoopGraph{k, exec, launches, ++g_graph_clock, 1});
    return &g_graphs.back();
  }
  LoopGraph* victim = nullptr;
  for (LoopGraph& e : g_graphs)
    if (e.users == 0 && (victim == nullptr || e.last_use < victim->last_use)) victim = &e;
  if (victim == nullptr) return nullptr;  // all in use: the caller runs it uncached
  cudaGraphExecDestroy(victim->exec);
  *victim = LoopGraph{k, exec, launches, ++g_graph_clock, 1};
  return victim;
}
static cudaStream_t capture_stream(int dev, unsigned long long ctx) {
  std::lock_guard<std::mutex> lk(g_graph_mu);
  CapStream& c = g_cap[dev];
  if (c.s == nullptr || c.ctx != ctx) {
    cudaStream_t s = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    c = CapStream{ctx, s};
  }
  return c.s;
}

// Captures enqueue(cs) into an executable graph; false (and nothing cached)
// when capture or instantiation fails.
template <class F>
static bool capture_loop(F&& enqueue, cudaStream_t cs, cudaGraphExec_t* exec, uint64_t* launches) {
  const uint64_t t0 = t_launches;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const tt_status s = enqueue(cs);
  cudaGraph_t graph = nullptr;
  const cudaError_t e = cudaStreamEndCapture(cs, &graph);
  // the captured launches did not run: take them off the counters
  const uint64_t n = t_launches - t0;
  g_launches.fetch_sub(n, std::memory_order_relaxed);
  t_launches = t0;
  bool ok = s == TT_OK && e == cudaSuccess && graph != nullptr &&
            cudaGraphInstantiate(exec, graph, 0) == cudaSuccess;
  if (graph != nullptr) cudaGraphDestroy(graph);
  if (!ok) cudaGetLastError();
  *launches = n;
  return ok;
}

}  // namespace tt

using namespace tt;

extern "C" {

const char* tt_status_string(tt_status s) {
  switch (s) {
    case TT_OK: return "TT_OK";
    case TT_ERR_INVALID_ARG: return "TT_ERR_INVALID_ARG";
    case TT_ERR_UNSUPPORTED: return "TT_ERR_UNSUPPORTED";
    case TT_ERR_WORKSPACE: return "TT_ERR_WORKSPACE";
    case TT_ERR_CUDA: return "TT_ERR_CUDA";
    case TT_ERR_TIMEOUT: return "TT_ERR_TIMEOUT";
    case TT_ERR_INTERNAL: return "TT_ERR_INTERNAL";
  }
  return "TT_ERR_UNKNOWN";
}

const char* tt_last_error(void) { return g_err; }

uint64_t tt_launch_count(void) { return g_launches.load(); }

tt_status tt_profile_enable(int32_t on) {
  if (on) {
    prof_harvest();
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (int k = 0; k < TT_K_COUNT; ++k) {
      g_prof_ms[k] = 0.0;
      g_prof_n[k] = 0;
    }
  }
  g_prof_on.store(on != 0);
  return TT_OK;
}

tt_status tt_profile_read(int32_t kind, double* total_ms, int64_t* launches) {
  if (kind < 0 || kind >= TT_K_COUNT) return fail(TT_ERR_INVALID_ARG, "kind=%d", kind);
  if (total_ms == nullptr || launches == nullptr)
    return fail(TT_ERR_INVALID_ARG, "output pointer is NULL");
  prof_harvest();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  *total_ms = g_prof_ms[kind];
  *launches = g_prof_n[kind];
  return TT_OK;
}

tt_status tt_set_loop_graphs(int32_t on) {
  if (on != 0 && on != 1) return fail(TT_ERR_INVALID_ARG, "on=%d not 0 or 1", on);
  g_graphs_on.store(on != 0);
  return TT_OK;
}

tt_status tt_set_attn_splits(int32_t n_splits) {
  if (n_splits < 0 || n_splits > 1024)
    return fail(TT_ERR_INVALID_ARG, "n_splits=%d not in [0, 1024]", n_splits);
  g_forced_splits.store(n_splits);
  return TT_OK;
}

size_t tt_workspace_bytes(const tt_dims* d, int which) {
  if (check_dims(d) != TT_OK) return 0;
  if (which < TT_WS_ATTN || which > TT_WS_LOOP) {
    fail(TT_ERR_INVALID_ARG, "unknown workspace kind %d", which);
    return 0;
  }
  return carve(*d, which, nullptr).total;
}

tt_status tt_selftest_timeout(void* ws, int32_t limit_us, void* stream) {
  TT_CHECK(check_ptr(ws, "ws", true));
  if (limit_us < 1 || limit_us > 1000000)
    return fail(TT_ERR_INVALID_ARG, "limit_us=%d not in [1, 1000000]", limit_us);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TT_CUDA(cudaMemsetAsync(ws, 0, kCtrlBytes, st));
  TT_CUDA(launch_selftest_wait(reinterpret_cast<int*>(ws), 1000ull * (unsigned long long)limit_us,
                               st));
  return TT_OK;
}

tt_status tt_device_status(void* ws, void* stream) {
  TT_CHECK(check_ptr(ws, "ws", true));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int h[2] = {0, 0};
  TT_CUDA(cudaStreamSynchronize(st));
  TT_CUDA(cudaMemcpy(h, ws, sizeof h, cudaMemcpyDeviceToHost));
  if (h[0] != 0) {
    TT_CUDA(cudaMemset(ws, 0, sizeof h));
    return fail((tt_status)h[0], "device reported %s at tag 0x%x",
                tt_status_string((tt_status)h[0]), h[1]);
  }
  return TT_OK;
}

tt_status tt_block_denoise_attn(const tt_dims* d, const tt_bf16* q_blk, const tt_bf16* k_blk,
                                const tt_bf16* v_blk, const tt_bf16* k_ctx,
                                const tt_bf16* v_ctx, const int32_t* ctx_len, tt_bf16* out,
                                void* ws, size_t ws_bytes, void* stream) {
  TT_CHECK(check_dims(d));
  TT_CHECK(check_ptr(q_blk, "q_blk", true));
  TT_CHECK(check_ptr(k_blk, "k_blk", true));
  TT_CHECK(check_ptr(v_blk, "v_blk", true));
  TT_CHECK(check_ptr(k_ctx, "k_ctx", true));
  TT_CHECK(check_ptr(v_ctx, "v_ctx", true));
  TT_CHECK(check_ptr(ctx_len, "ctx_len", false));
  TT_CHECK(check_ptr(out, "out", true));
  Ws w;
  TT_CHECK(check_ws(*d, TT_WS_ATTN, ws, ws_bytes, &w));
  const AttnGeom g = attn_geom(*d);
  AttnMaps m;
  TT_CHECK(build_attn_maps(*d, g, q_blk, d->Hq * d->dh, k_blk, v_blk, d->Hkv * d->dh, k_ctx,
                           v_ctx, &m));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TT_CUDA(cudaMemsetAsync(w.ctrl, 0, kCtrlBytes, st));
  TT_CHECK(run_attn_plan(*d, g, ctx_len, w, st));
  return run_attn(*d, g, m, ctx_len, out, w, nullptr, true, st);
}

tt_status tt_adaln_modulate(const tt_dims* d, const tt_bf16* x, const tt_bf16* shift_scale,
                            const float* t, tt_bf16* y, void* ws, size_t ws_bytes,
                            void* stream) {
  TT_CHECK(check_dims(d));
  TT_CHECK(check_ptr(x, "x", true));
  TT_CHECK(check_ptr(shift_scale, "shift_scale", true));
  TT_CHECK(check_ptr(t, "t", false));
  TT_CHECK(check_ptr(y, "y", true));
  if (x == y) return fail(TT_ERR_INVALID_ARG, "y may not alias x");
  Ws w;
  TT_CHECK(check_ws(*d, TT_WS_ADALN, ws, ws_bytes, &w));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TT_CUDA(cudaMemsetAsync(w.ctrl, 0, kCtrlBytes, st));
  TT_LAUNCH(TT_K_ADALN, st, launch_adaln(x, shift_scale, t, y, d->B * d->S, d->S, d->H, nullptr,
                                         nullptr, nullptr, nullptr, st));
  return TT_OK;
}

tt_status tt_vocab_confidence_commit(const tt_dims* d, const tt_bf16* y, const tt_bf16* w,
                                     float gamma, float logit_scale, int32_t* tokens,
                                     uint8_t* masked, float* conf_out, int32_t* argmax_out,
                                     int32_t* n_committed, void* ws, size_t ws_bytes,
                                     void* stream) {
  TT_CHECK(check_vocab_args(d, y, w, gamma, logit_scale, tokens, masked));
  Ws ws_;
  TT_CHECK(check_ws(*d, TT_WS_VOCAB, ws, ws_bytes, &ws_));
  return run_vocab_commit(*d, ws, y, w, gamma, logit_scale, tokens, masked, conf_out, argmax_out,
                          n_committed, reinterpret_cast<cudaStream_t>(stream));
}

// The block loop over n_layers denoiser layers (n_layers = 1: the
// single-layer step).  Per-layer tensors are stacked with the layer index
// outermost: k_ctx/v_ctx [n_layers][B,Hkv,L_cap,dh], u_t [n_layers][n_qkv,H],
// shift_scale [n_layers][2,H].
static tt_status denoise_block_loop_impl(
    const tt_dims* d, int32_t n_layers, const tt_bf16* k_ctx, const tt_bf16* v_ctx,
    const int32_t* ctx_len, const tt_bf16* emb, const tt_bf16* e_mask, const tt_bf16* u_t,
    const tt_bf16* shift_scale, const tt_bf16* W, float gamma, float logit_scale,
    int32_t max_steps, int32_t* tokens, uint8_t* masked, int32_t* steps_taken,
    int32_t* commit_step, int32_t* steps_run, void* ws, size_t ws_bytes, void* stream,
    bool allow_graph = true) {
  TT_CHECK(check_dims(d));
  TT_CHECK(check_ptr(k_ctx, "k_ctx", true));
  TT_CHECK(check_ptr(v_ctx, "v_ctx", true));
  TT_CHECK(check_ptr(ctx_len, "ctx_len", false));
  TT_CHECK(check_ptr(emb, "emb", true));
  TT_CHECK(check_ptr(e_mask, "e_mask", true));
  TT_CHECK(check_ptr(u_t, "u_t", true));
  TT_CHECK(check_ptr(shift_scale, "shift_scale", true));
  TT_CHECK(check_ptr(W, "w", true));
  TT_CHECK(check_ptr(tokens, "tokens", false));
  TT_CHECK(check_ptr(masked, "masked", false));
  TT_CHECK(check_ptr(steps_taken, "steps_taken", false));
  TT_CHECK(check_ptr(commit_step, "commit_step", false));
  if (n_layers < 1 || n_layers > 64)
    return fail(TT_ERR_INVALID_ARG, "n_layers=%d not in [1, 64]", n_layers);
  if (!(gamma > 0.f && gamma <= 1.f))
    return fail(TT_ERR_INVALID_ARG, "gamma=%g not in (0, 1]", (double)gamma);
  if (!(logit_scale > 0.f) || !std::isfinite(logit_scale))
    return fail(TT_ERR_INVALID_ARG, "logit_scale=%g must be finite and > 0", (double)logit_scale);
  if (max_steps < 1 || max_steps > 1024)
    return fail(TT_ERR_INVALID_ARG, "max_steps=%d not in [1, 1024]", max_steps);
  Ws w;
  TT_CHECK(check_ws(*d, TT_WS_LOOP, ws, ws_bytes, &w));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int rows = d->B * d->S;
  const int n_qkv = d->H + 2 * d->Hkv * d->dh;
  const AttnGeom g = attn_geom(*d);
  const size_t ctx_elems = (size_t)d->B * d->Hkv * d->L_cap * d->dh;

  // Replay of a captured graph of this exact call (see LoopKey).
  LoopKey key;
  std::memset(&key, 0, sizeof key);
  int dev = 0;
  bool use_graph = allow_graph && g_graphs_on.load() && !g_prof_on.load();
  if (use_graph) {
    use_graph = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxGraphDevices &&
                current_context_id(&key.ctx);
    if (!use_graph) cudaGetLastError();
  }
  if (use_graph) {
    key.d = *d;
    key.n_layers = n_layers;
    key.max_steps = max_steps;
    key.n_ctas = g.n_ctas;
    key.dev = dev;
    const void* ptrs[14] = {k_ctx, v_ctx, ctx_len, emb,     e_mask,      u_t,         shift_scale,
                            W,     tokens, masked, steps_taken, commit_step, ws,          nullptr};
    std::memcpy(key.p, ptrs, sizeof ptrs);
    key.ws_bytes = ws_bytes;
    std::memcpy(&key.gamma_bits, &gamma, sizeof gamma);
    std::memcpy(&key.scale_bits, &logit_scale, sizeof logit_scale);
  }
  LoopGraph* cached = use_graph ? graph_acquire(key) : nullptr;
  cudaGraphExec_t uncached = nullptr;  // captured, but the cache is full of graphs in use
  uint64_t uncached_n = 0;
  if (cached == nullptr) {
    // Layer 0 reads the gathered embeddings, later layers the previous
    // layer's modulated rows (every position of the block).
    CUtensorMap tmE, tmX;
    if (!make_tmap_2d(&tmE, w.egath, d->H, rows, (uint64_t)d->H * 2, kGemmBK, kGemmBM) ||
        !make_tmap_2d(&tmX, w.xrows, d->H, rows, (uint64_t)d->H * 2, kGemmBK, kGemmBM))
      return fail(TT_ERR_CUDA, "cuTensorMapEncodeTiled failed for the linear update");
    std::vector<CUtensorMap> tmU(n_layers);
    std::vector<AttnMaps> maps(n_layers);
    for (int l = 0; l < n_layers; ++l) {
      if (!make_tmap_2d(&tmU[l], u_t + (size_t)l * n_qkv * d->H, d->H, n_qkv, (uint64_t)d->H * 2,
                        kGemmBK, qkv_bn(rows)))
        return fail(TT_ERR_CUDA, "cuTensorMapEncodeTiled failed for the linear update");
      TT_CHECK(build_attn_maps(*d, g, w.qkv, n_qkv, w.qkv + d->H, w.qkv + d->H + d->Hkv * d->dh,
                               n_qkv, k_ctx + (size_t)l * ctx_elems, v_ctx + (size_t)l * ctx_elems,
                               &maps[l]));
    }

    auto enqueue = [&](cudaStream_t st) -> tt_status {
      TT_CUDA(cudaMemsetAsync(w.ctrl, 0, w.ctrl_clear, st));
      TT_LAUNCH(TT_K_INIT, st, launch_loop_init(d->B, d->S, steps_taken, commit_step, w.ctrl, st));
      TT_CHECK(run_attn_plan(*d, g, ctx_len, w, st));
      // a step runs while masked positions remain (commit decrements the count)
      const int* active = w.ctrl + CTRL_REMAINING;
      GemmArgs ga{};
      ga.M_alloc = rows;
      ga.active = active;
      ga.N = n_qkv;
      ga.K = d->H;
      ga.C = w.qkv;
      ga.ldc = n_qkv;
      ga.err = w.ctrl;
      ga.ksplit = qkv_ksplit(*d);
      ga.partial = w.qkv_partial;
      ga.b_keep = 1;  // U is re-read by every step
      const int qkv_tiles =
          ((rows + kGemmBM - 1) / kGemmBM) * ((n_qkv + qkv_bn(rows) - 1) / qkv_bn(rows)) *
          ga.ksplit;
      // W streams with evict-first; pinning part of it in L2 across steps was
      // measured slower (the vocab GEMM lost ~10 us per step), so none is kept.
      const int w_keep_tiles = 0;
      const bool pf_w = vocab_prefetch(*d, attn_args(*d, g, ctx_len, w.attn_out, w, active));
      // Step 0's plan and the embedding of every position; afterwards the commit
      // kernel re-embeds what it commits and its last CTA plans the next step.
      PlanArgs p{d->B, d->S, masked, w.rowlist, w.tvec, w.ctrl, 0};
      TT_LAUNCH(TT_K_PLAN, st, launch_plan(p, st));
      TT_LAUNCH(TT_K_EMBED, st, launch_embed(tokens, masked, emb, e_mask, w.egath, rows, d->H, d->V,
                                             active, w.ctrl, st));
      for (int step = 0; step < max_steps; ++step) {
        for (int l = 0; l < n_layers; ++l) {
          const bool last = l == n_layers - 1;
          const tt_bf16* ss = shift_scale + (size_t)l * 2 * d->H;
          TT_LAUNCH(TT_K_GEMM_QKV, st, launch_gemm_bf16(l == 0 ? tmE : tmX, tmU[l], ga,
                                                        std::min(qkv_tiles, num_sms()),
                                                        qkv_bn(rows), st));
          if (ga.ksplit > 1)
            TT_LAUNCH(TT_K_REDUCE, st, launch_splitk_reduce(w.qkv_partial, ga.ksplit, rows, n_qkv,
                                                              w.qkv, n_qkv, active, qkv_bn(rows),
                                                              st));
          TT_CHECK(run_attn(*d, g, maps[l], ctx_len, w.attn_out, w, active, false, st,
                            last && pf_w ? W : nullptr));
          // The last layer keeps the masked rows, compacted, for the vocabulary;
          // earlier layers modulate every row (all positions are keys of the
          // next layer).  A null row list selects the latter.
          uint16_t* y = last ? w.y_c : w.xrows;
          int* rl = last ? w.rowlist : nullptr;
          if (g.fixup) {
            TT_LAUNCH(TT_K_ADALN, st, launch_adaln(w.attn_out, ss, nullptr, y, rows, d->S, d->H,
                                                   masked, rl, w.ctrl, active, st));
          } else {
            const AttnArgs aa = attn_args(*d, g, ctx_len, w.attn_out, w, active);
            TT_LAUNCH(TT_K_ADALN, st, launch_merge_adaln(aa, ss, y, masked, rl, w.ctrl, st));
          }
        }
        TT_CHECK(run_vocab_gemm(*d, w, W, logit_scale, w.ctrl + CTRL_M, active, w_keep_tiles, st));
        CommitArgs c = commit_args(*d, w, gamma, logit_scale, tokens, masked);
        c.commit_step = commit_step;
        c.steps_taken = steps_taken;
        c.step = step;
        c.active = active;
        c.emb = emb;
        c.egath = w.egath;
        c.H = d->H;
        c.plan_next = 1;
        TT_LAUNCH(TT_K_COMMIT, st, launch_commit(c, st));
      }
      return TT_OK;
    };
    cudaGraphExec_t exec = nullptr;
    uint64_t n = 0;
    cudaStream_t cs = use_graph ? capture_stream(dev, key.ctx) : nullptr;
    if (cs != nullptr && capture_loop(enqueue, cs, &exec, &n)) {
      cached = graph_insert(key, exec, n);
      if (cached == nullptr) {
        uncached = exec;
        uncached_n = n;
      }
    } else {
      TT_CHECK(enqueue(st));
    }
  }
  cudaGraphExec_t run = cached != nullptr ? cached->exec : uncached;
  if (run != nullptr) {
    const cudaError_t e = cudaGraphLaunch(run, st);
    count_launch((int)(cached != nullptr ? cached->launches : uncached_n));
    if (e != cudaSuccess) {
      if (cached != nullptr) graph_release(cached);
      if (uncached != nullptr) cudaGraphExecDestroy(uncached);
      return fail(TT_ERR_CUDA, "cudaGraphLaunch failed: %s", cudaGetErrorString(e));
    }
  }
  int h[8];
  const tt_status rs = read_ctrl(w, st, h);
  if (cached != nullptr) graph_release(cached);
  if (uncached != nullptr) cudaGraphExecDestroy(uncached);
  TT_CHECK(rs);
  if (g_prof_on.load()) prof_harvest();
  if (steps_run != nullptr) *steps_run = h[CTRL_STEPS_RUN];
  if (h[CTRL_ERR] != 0)
    return fail((tt_status)h[CTRL_ERR], "device reported %s at tag 0x%x",
                tt_status_string((tt_status)h[CTRL_ERR]), h[CTRL_ERR_WHERE]);
  return TT_OK;
}

tt_status tt_denoise_block_loop(const tt_dims* d, const tt_bf16* k_ctx, const tt_bf16* v_ctx,
                                const int32_t* ctx_len, const tt_bf16* emb,
                                const tt_bf16* e_mask, const tt_bf16* u_t,
                                const tt_bf16* shift_scale, const tt_bf16* W, float gamma,
                                float logit_scale, int32_t max_steps, int32_t* tokens,
                                uint8_t* masked, int32_t* steps_taken, int32_t* commit_step,
                                int32_t* steps_run, void* ws, size_t ws_bytes, void* stream) {
  return denoise_block_loop_impl(d, 1, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale, W,
                                 gamma, logit_scale, max_steps, tokens, masked, steps_taken,
                                 commit_step, steps_run, ws, ws_bytes, stream);
}

tt_status tt_denoise_block_loop_layers(const tt_dims* d, int32_t n_layers, const tt_bf16* k_ctx,
                                       const tt_bf16* v_ctx, const int32_t* ctx_len,
                                       const tt_bf16* emb, const tt_bf16* e_mask,
                                       const tt_bf16* u_t, const tt_bf16* shift_scale,
                                       const tt_bf16* W, float gamma, float logit_scale,
                                       int32_t max_steps, int32_t* tokens, uint8_t* masked,
                                       int32_t* steps_taken, int32_t* commit_step,
                                       int32_t* steps_run, void* ws, size_t ws_bytes,
                                       void* stream) {
  return denoise_block_loop_impl(d, n_layers, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t,
                                 shift_scale, W, gamma, logit_scale, max_steps, tokens, masked,
                                 steps_taken, commit_step, steps_run, ws, ws_bytes, stream);
}

tt_status tt_loop_last_step(const tt_dims* d, void* ws, size_t ws_bytes, tt_bf16* y_rows,
                            int32_t* row_ids, float* conf, int32_t* argmax, int32_t* n_rows,
                            void* stream) {
  TT_CHECK(check_dims(d));
  TT_CHECK(check_ptr(y_rows, "y_rows", true));
  TT_CHECK(check_ptr(row_ids, "row_ids", false));
  TT_CHECK(check_ptr(conf, "conf", false));
  TT_CHECK(check_ptr(argmax, "argmax", false));
  TT_CHECK(check_ptr(n_rows, "n_rows", false));
  Ws w;
  TT_CHECK(check_ws(*d, TT_WS_LOOP, ws, ws_bytes, &w));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int rows = d->B * d->S;
  int h[8];
  TT_CHECK(read_ctrl(w, st, h));
  const int M = h[CTRL_M];
  if (M < 0 || M > rows)
    return fail(TT_ERR_INTERNAL, "workspace holds a row count of %d (B*S = %d): not a loop "
                "workspace after a step", M, rows);
  if (M > 0) {
    TT_CUDA(cudaMemcpyAsync(y_rows, w.y_c, (size_t)M * d->H * 2, cudaMemcpyDeviceToDevice, st));
    TT_CUDA(cudaMemcpyAsync(row_ids, w.rowlist, (size_t)M * sizeof(int), cudaMemcpyDeviceToDevice,
                            st));
  }
  // per-row (confidence, token bits) pairs -> the two output arrays
  TT_CUDA(cudaMemcpy2DAsync(conf, sizeof(float), w.rowres, sizeof(float2), sizeof(float), rows,
                            cudaMemcpyDeviceToDevice, st));
  TT_CUDA(cudaMemcpy2DAsync(argmax, sizeof(int32_t), reinterpret_cast<const char*>(w.rowres) + 4,
                            sizeof(float2), sizeof(int32_t), rows, cudaMemcpyDeviceToDevice, st));
  TT_CUDA(cudaStreamSynchronize(st));
  *n_rows = M;
  return TT_OK;
}

tt_status tt_decode_blocks(const tt_dims* d, int32_t n_blocks, tt_bf16* k_ctx, tt_bf16* v_ctx,
                           int32_t* ctx_len, const tt_bf16* emb, const tt_bf16* e_mask,
                           const tt_bf16* u_t, const tt_bf16* shift_scale, const tt_bf16* W,
                           const tt_bf16* u_ctx, float gamma, float logit_scale,
                           int32_t* tokens, int32_t* steps_taken, int32_t* commit_step,
                           int32_t* steps_run, void* ws, size_t ws_bytes, void* stream) {
  TT_CHECK(check_dims(d));
  TT_CHECK(check_ptr(u_ctx, "u_ctx", true));
  TT_CHECK(check_ptr(tokens, "tokens", false));
  TT_CHECK(check_ptr(steps_taken, "steps_taken", false));
  TT_CHECK(check_ptr(commit_step, "commit_step", false));
  if (n_blocks < 1 || n_blocks > 4096)
    return fail(TT_ERR_INVALID_ARG, "n_blocks=%d not in [1, 4096]", n_blocks);
  Ws w;
  TT_CHECK(check_ws(*d, TT_WS_LOOP, ws, ws_bytes, &w));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int rows = d->B * d->S;
  const int n_kv = 2 * d->Hkv * d->dh;
  CUtensorMap tmE, tmC;
  if (!make_tmap_2d(&tmE, w.egath, d->H, rows, (uint64_t)d->H * 2, kGemmBK, kGemmBM) ||
      !make_tmap_2d(&tmC, u_ctx, d->H, n_kv, (uint64_t)d->H * 2, kGemmBK, qkv_bn(rows)))
    return fail(TT_ERR_CUDA, "cuTensorMapEncodeTiled failed for the context projection");
  GemmArgs ga{};
  ga.M_alloc = rows;
  ga.N = n_kv;
  ga.K = d->H;
  ga.C = w.qkv;  // free between blocks
  ga.ldc = n_kv;
  ga.err = w.ctrl;
  ga.ksplit = ctx_ksplit(*d);
  ga.partial = w.qkv_partial;
  const int bn = qkv_bn(rows);
  const int tiles = ((rows + kGemmBM - 1) / kGemmBM) * ((n_kv + bn - 1) / bn) * ga.ksplit;
  int total_steps = 0;
  for (int j = 0; j < n_blocks; ++j) {
    int32_t* tok = tokens + (size_t)j * rows;
    // a new block: every position masked, no token yet
    TT_CUDA(cudaMemsetAsync(tok, 0xff, (size_t)rows * sizeof(int32_t), st));
    TT_CUDA(cudaMemsetAsync(w.blk_masked, 1, (size_t)rows, st));
    int32_t n = 0;
    TT_CHECK(denoise_block_loop_impl(d, 1, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale,
                                     W, gamma, logit_scale, d->S, tok, w.blk_masked,
                                     steps_taken + (size_t)j * d->B,
                                     commit_step + (size_t)j * rows, &n, ws, ws_bytes, stream,
                                     /*allow_graph=*/false));
    total_steps += n;
    // The committed block joins the context: its rows of the workspace's
    // embeddings are Emb[token] (the commit re-embeds what it commits), so
    // [k | v] = Emb[token] . U_ctx^T, appended at each sequence's end.
    TT_LAUNCH(TT_K_GEMM_QKV, st,
              launch_gemm_bf16(tmE, tmC, ga, std::min(tiles, num_sms()), bn, st));
    if (ga.ksplit > 1)
      TT_LAUNCH(TT_K_REDUCE, st, launch_splitk_reduce(w.qkv_partial, ga.ksplit, rows, n_kv,
                                                        w.qkv, n_kv, nullptr, bn, st));
    TT_LAUNCH(TT_K_APPEND, st, launch_append_kv(w.qkv, n_kv, k_ctx, v_ctx, ctx_len, d->B, d->S,
                                                d->Hkv, d->dh, d->L_cap, w.ctrl, st));
    // the next block's loop clears the control block: check this append now
    int h[8];
    TT_CHECK(read_ctrl(w, st, h));
    if (h[CTRL_ERR] != 0) {
      if (steps_run != nullptr) *steps_run = total_steps;
      return fail((tt_status)h[CTRL_ERR], "block %d: device reported %s at tag 0x%x", j,
                  tt_status_string((tt_status)h[CTRL_ERR]), h[CTRL_ERR_WHERE]);
    }
  }
  if (g_prof_on.load()) prof_harvest();
  if (steps_run != nullptr) *steps_run = total_steps;
  return TT_OK;
}

}  // extern "C"
