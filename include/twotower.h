/*
 * libtwotower - block-wise diffusion denoise step on one B200 (sm_100a).
 *
 * The operations follow "Nemotron-TwoTower: Diffusion Language Modeling with
 * Pretrained Autoregressive Context" (gist.science technical summary, sections
 * Architecture, Generation Process, Training and Conditioning) and the
 * snilld.dk TwoTower article (sections "Hvad TwoTower aendrer teknisk",
 * "Blockwise generering i praksis").  The pages fix the method qualitatively;
 * the numeric readings this library takes are stated beside each call.
 *
 * Conventions for every call
 *  - All tensor pointers are DEVICE pointers, allocated and owned by the
 *    caller.  The library never allocates device or pinned memory; scratch
 *    space comes from a caller-provided workspace sized by tt_workspace_bytes.
 *  - bf16 tensors are passed as tt_bf16 (the 16-bit pattern) and are dense,
 *    row-major, with the layouts given below.  Base pointers of bf16 tensors
 *    and workspaces must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream unless stated otherwise.
 *  - Argument errors are detected on the host before any launch; the call
 *    then returns an error code, launches nothing and modifies nothing.
 *    tt_last_error() gives a thread-local description of the last failure.
 *  - Errors a kernel detects (a bounded wait that timed out, an out-of-range
 *    token id, a non-finite confidence) are recorded in the first 4 bytes of
 *    the workspace and reported by tt_device_status() or, for the loop, by
 *    the loop's own return code.
 *  - Inputs are never modified, except `tokens` and `masked`, which are
 *    in/out state of the commit step and of the loop.
 *
 * Supported shapes: dh in {64, 128}; S in {1, 16, 32, 64, 128} (S = 1 is
 * the autoregressive baseline: one position per block); H == Hq*dh with H a
 * multiple of 64, at most 8192; G = Hq/Hkv a power of two, at most 128; V >= 2;
 * B >= 1; 0 <= ctx_len[b] <= L_cap.  Other shapes return TT_ERR_UNSUPPORTED.
 */
#ifndef TWOTOWER_H
#define TWOTOWER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TT_API __attribute__((visibility("default")))
#else
#define TT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tt_bf16; /* bit pattern of one bfloat16 value */

typedef enum {
  TT_OK = 0,
  TT_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, gamma out of (0,1] */
  TT_ERR_UNSUPPORTED = 2, /* shape outside the supported set above */
  TT_ERR_WORKSPACE = 3,   /* workspace smaller than tt_workspace_bytes() */
  TT_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (text in tt_last_error) */
  TT_ERR_TIMEOUT = 5,     /* a kernel's bounded wait gave up (recorded on the device) */
  TT_ERR_INTERNAL = 6     /* device-detected inconsistency (bad token id, NaN confidence) */
} tt_status;

/* Problem sizes.  B sequences, block size S, Hq query heads, Hkv KV heads,
 * head size dh, hidden size H (= Hq*dh), vocabulary V, context capacity
 * L_cap (rows allocated per sequence and KV head in the context cache). */
typedef struct {
  int32_t B, S, Hq, Hkv, dh, H, V, L_cap;
} tt_dims;

/* Which call a workspace is sized for. */
enum { TT_WS_ATTN = 0, TT_WS_ADALN = 1, TT_WS_VOCAB = 2, TT_WS_LOOP = 3 };

/* Human-readable name of a status code (static string). */
TT_API const char* tt_status_string(tt_status s);

/* Description of the last error raised on the calling thread ("" if none). */
TT_API const char* tt_last_error(void);

/* Bytes of workspace the call `which` needs for dims `d` on the current
 * device (the attention's split plan follows the device's SM count; a host
 * without a GPU sizes for a B200's 148 SMs); 0 if `d` is invalid
 * (tt_last_error says why). */
TT_API size_t tt_workspace_bytes(const tt_dims* d, int which);

/* Synchronises `stream`, then reads and clears the device error word at the
 * start of workspace `ws`.  Returns TT_OK, TT_ERR_TIMEOUT, TT_ERR_INTERNAL or
 * TT_ERR_CUDA. */
TT_API tt_status tt_device_status(void* ws, void* stream);

/* Failure-detection self test: launches one kernel that waits on a barrier
 * nothing completes, bounded by limit_us (1 .. 1e6 microseconds), exactly
 * like the kernels' own pipeline waits.  The wait gives up, records
 * TT_ERR_TIMEOUT in the control block of `ws` (>= 256 bytes) and the kernel
 * returns; tt_device_status(ws, stream) then reports TT_ERR_TIMEOUT and the
 * context stays usable.  Nothing faults and nothing hangs. */
TT_API tt_status tt_selftest_timeout(void* ws, int32_t limit_us, void* stream);

/* Number of kernels this library has launched in this process so far. */
TT_API uint64_t tt_launch_count(void);

/* Number of CTAs the attention's key tiles are divided over (0 = the
 * library's choice, the default; otherwise at most 1024, CTAs beyond the
 * SM count running in later waves): all units' tiles, laid end to end, are
 * cut into that many equal contiguous ranges.  Process-wide, read when a
 * workspace is sized and when a call runs, so set it before sizing the
 * workspace; results are independent of it up to float rounding. */
TT_API tt_status tt_set_attn_splits(int32_t n_splits);

/* 1 (the default): tt_denoise_block_loop and tt_denoise_block_loop_layers
 * replay a captured CUDA graph per argument set; 0: they launch every kernel
 * directly (as they also do while the profiler is on).  Process-wide.  Any
 * other value is TT_ERR_INVALID_ARG. */
TT_API tt_status tt_set_loop_graphs(int32_t on);

/* Kernel kinds of the per-kernel profiler. */
enum {
  TT_K_PLAN = 0, TT_K_EMBED = 1, TT_K_GEMM_QKV = 2, TT_K_ATTN = 3, TT_K_MERGE = 4,
  TT_K_ADALN = 5, TT_K_GEMM_VOCAB = 6, TT_K_COMMIT = 7, TT_K_GATHER = 8, TT_K_INIT = 9,
  TT_K_REDUCE = 10, TT_K_APPEND = 11, TT_K_ATTN_PLAN = 12, TT_K_COUNT = 13
};

/* Per-kernel profiler: while enabled, every kernel this library launches is
 * bracketed by two CUDA events recorded on the caller's stream.  on = 1
 * clears the table and starts recording, on = 0 stops.  Off by default; it
 * adds two event records per launch and nothing else. */
TT_API tt_status tt_profile_enable(int32_t on);

/* Total device time (ms) and launch count of kernel kind `kind` since the
 * last tt_profile_enable(1).  Waits for the recorded events to complete. */
TT_API tt_status tt_profile_read(int32_t kind, double* total_ms, int64_t* launches);

/*
 * a1 - block-denoise attention of one denoiser layer.
 * Source: gist.science summary, "Architecture" (bidirectional block attention
 * plus attention to the corresponding layer of the frozen context tower) and
 * "Generation Process" (each layer attends to the context KV cache of past
 * blocks and to the block's own bidirectional KV).
 *
 * For every sequence b, query head h (KV head g = h / (Hq/Hkv)) and block
 * position s:
 *   out[b,s,h,:] = softmax_j( q_blk[b,s,h,:] . key_j / sqrt(dh) ) value_j
 * over the keys [k_ctx[b,g,0:ctx_len[b],:] ; k_blk[b,0:S,g,:]] and the
 * matching values: one joint softmax, no mask inside the block, no
 * positional encoding.  Rows of the context cache at or past ctx_len[b] are
 * never used.  fp32 accumulation, bf16 result.
 *
 *   q_blk   bf16 [B, S, Hq, dh]
 *   k_blk   bf16 [B, S, Hkv, dh]       v_blk bf16 [B, S, Hkv, dh]
 *   k_ctx   bf16 [B, Hkv, L_cap, dh]   v_ctx bf16 [B, Hkv, L_cap, dh]
 *   ctx_len int32 [B] (device)
 *   out     bf16 [B, S, Hq, dh]  (= [B*S, H])
 *   ws      workspace of at least tt_workspace_bytes(d, TT_WS_ATTN) bytes
 */
TT_API tt_status tt_block_denoise_attn(const tt_dims* d, const tt_bf16* q_blk, const tt_bf16* k_blk,
                                const tt_bf16* v_blk, const tt_bf16* k_ctx,
                                const tt_bf16* v_ctx, const int32_t* ctx_len, tt_bf16* out,
                                void* ws, size_t ws_bytes, void* stream);

/*
 * a2 - adaLN-single time modulation.
 * Source: gist.science summary, "Training and Conditioning" (time conditioning
 * through adaptive layer normalisation); snilld.dk, every layer modulated by a
 * small adaLN-single block.  Reading of this library (the pages give no
 * formula): for row r of sequence b = r / S,
 *   [shift ; scale] = shift_scale + phi(t[b]),
 *   phi(t) = [sin(t*w_i) for i < H] ++ [cos(t*w_i) for i < H], w_i = 10000^(-i/H),
 *   y[r] = LN(x[r]) * (1 + scale) + shift,
 * LN without affine parameters, biased variance, eps 1e-6.
 *
 *   x           bf16 [B*S, H]
 *   shift_scale bf16 [2, H]   (row 0 shift, row 1 scale)
 *   t           float [B] (device)
 *   y           bf16 [B*S, H]   (may not alias x)
 *   ws          workspace of at least tt_workspace_bytes(d, TT_WS_ADALN) bytes
 */
TT_API tt_status tt_adaln_modulate(const tt_dims* d, const tt_bf16* x, const tt_bf16* shift_scale,
                            const float* t, tt_bf16* y, void* ws, size_t ws_bytes, void* stream);

/*
 * a3 + a4 - vocabulary projection, confidence and commit.
 * Source: gist.science summary, "Training and Conditioning", Sampling:
 * all masked positions are predicted in parallel; confident ones commit,
 * uncertain ones stay masked, so the number committed per step adapts.
 * Commit rule of this library: among positions with masked[b,s] != 0,
 *   logits = logit_scale * y[b*S+s,:] . w[v,:]   (fp32 accumulation),
 *   conf   = max_v softmax(logits),  tok = argmax_v (lowest id on ties);
 * every one with conf >= gamma commits tok; if none in sequence b does, the
 * single masked position with the largest conf commits (lowest s on ties).
 * Committed positions get tokens[b,s] = tok and masked[b,s] = 0; positions
 * already committed never change.  Logits are never written to memory.
 *
 *   y           bf16 [B*S, H]   (rows of unmasked positions are not read)
 *   w           bf16 [V, H]     (one row per token: the "out x in" layout)
 *   gamma       threshold in (0, 1];  logit_scale > 0 (1 = plain softmax)
 *   tokens      int32 [B, S] in/out;  masked uint8 [B, S] in/out (1 = masked)
 *   conf_out    float [B, S]  confidence of positions masked on entry, -1 elsewhere
 *   argmax_out  int32 [B, S]  argmax of positions masked on entry, -1 elsewhere
 *   n_committed int32 [B]     positions committed in this call
 *   ws          workspace of at least tt_workspace_bytes(d, TT_WS_VOCAB) bytes
 */
TT_API tt_status tt_vocab_confidence_commit(const tt_dims* d, const tt_bf16* y, const tt_bf16* w,
                                     float gamma, float logit_scale, int32_t* tokens,
                                     uint8_t* masked, float* conf_out, int32_t* argmax_out,
                                     int32_t* n_committed, void* ws, size_t ws_bytes,
                                     void* stream);

/*
 * a5 + a6 - the denoise loop of one block: repeat
 *   embed (Emb[token] for committed positions, e_mask for masked ones)
 *   -> [q | k | v] = e . u_t^T  (one linear update, bf16 result)
 *   -> tt_block_denoise_attn -> tt_adaln_modulate (t_b = masked count / S)
 *   -> tt_vocab_confidence_commit
 * until no position is masked or max_steps steps have run.
 * Source: gist.science summary, "Generation Process" (the denoiser refines a
 * block of S masked tokens over T steps; the context tower only updates after
 * the block commits, so k_ctx / v_ctx are fixed here).
 *
 *   k_ctx, v_ctx, ctx_len  as in tt_block_denoise_attn
 *   emb          bf16 [V, H]   token embedding table
 *   e_mask       bf16 [H]      embedding of a masked position
 *   u_t          bf16 [H + 2*Hkv*dh, H]   linear update, output-major:
 *                rows [0,H) give q, [H, H+Hkv*dh) give k, the rest give v
 *   shift_scale  bf16 [2, H];  w bf16 [V, H];  gamma, logit_scale as above
 *   max_steps    1..1024 (S is always enough: every step commits at least
 *                one position of every sequence that still has one masked)
 *   tokens, masked  in/out state [B, S] (device); a partly committed block
 *                resumes from where it is
 *   steps_taken  int32 [B] (device): steps sequence b took in this call
 *   commit_step  int32 [B, S] (device): step index at which (b,s) committed
 *                in this call, -1 if it was committed on entry
 *   steps_run    optional host int32*: number of steps that did work
 *   ws           workspace of at least tt_workspace_bytes(d, TT_WS_LOOP) bytes
 * Blocking: returns after the stream has finished the loop (one host
 * synchronisation at the end, none per step).
 * Launch: the first call with a given set of arguments (every pointer and
 * size, gamma, logit_scale, max_steps, the attention's CTA count) captures
 * its kernel sequence into a CUDA graph on a library stream; later calls with
 * the same set replay it on `stream` as one launch (results bitwise those of
 * direct launches).  Up to 32 sets are kept per process; see
 * tt_set_loop_graphs.
 */
TT_API tt_status tt_denoise_block_loop(const tt_dims* d, const tt_bf16* k_ctx, const tt_bf16* v_ctx,
                                const int32_t* ctx_len, const tt_bf16* emb,
                                const tt_bf16* e_mask, const tt_bf16* u_t,
                                const tt_bf16* shift_scale, const tt_bf16* w, float gamma,
                                float logit_scale, int32_t max_steps, int32_t* tokens,
                                uint8_t* masked, int32_t* steps_taken, int32_t* commit_step,
                                int32_t* steps_run, void* ws, size_t ws_bytes, void* stream);

/*
 * Blocks one after the other ("Generation Process" of the gist.science
 * summary: a block of S masked tokens is refined until committed, then the
 * context tower updates and the next block starts).  For j = 0 .. n_blocks-1:
 * tokens_j = -1 and every position masked; the block loop of
 * tt_denoise_block_loop (up to S steps) commits it; then the block joins the
 * context: for each position, [k | v] = Emb[token] . U_ctx^T (bf16) is written
 * at context position ctx_len[b] + s of every KV head and ctx_len[b] += S.
 * The frozen context tower itself is not modelled: U_ctx is a seeded
 * projection standing in for it (this library's reading).
 *
 *   k_ctx, v_ctx   bf16 [B, Hkv, L_cap, dh]   IN/OUT: the rows
 *                  ctx_len[b] .. ctx_len[b] + n_blocks*S - 1 are written
 *   ctx_len        int32 [B] device            IN/OUT: grows by S per block
 *   u_ctx          bf16 [2*Hkv*dh, H]          rows 0..Hkv*dh-1 give k (head g
 *                  at rows g*dh..), the rest give v
 *   tokens         int32 [n_blocks, B, S]      OUT
 *   steps_taken    int32 [n_blocks, B]         OUT (as tt_denoise_block_loop)
 *   commit_step    int32 [n_blocks, B, S]      OUT
 *   steps_run      host int32, may be NULL     total steps that did work
 *   other arguments, workspace (TT_WS_LOOP) and errors as
 *   tt_denoise_block_loop; one host synchronisation per block.
 * n_blocks outside 1..4096 is TT_ERR_INVALID_ARG.  A sequence whose cache has
 * no room for a block (ctx_len[b] + S > L_cap) is found only when that block
 * is appended, after its loop has run: the call then returns
 * TT_ERR_INVALID_ARG (recorded on the device) with block j's tokens,
 * steps_taken and commit_step written but nothing of block j appended for
 * that sequence (its cache rows and ctx_len unchanged); blocks before j are
 * complete and no later block runs.  Callers that know ctx_len on the host
 * avoid this by checking ctx_len[b] + n_blocks*S <= L_cap first.
 */
TT_API tt_status tt_decode_blocks(const tt_dims* d, int32_t n_blocks, tt_bf16* k_ctx,
                                  tt_bf16* v_ctx, int32_t* ctx_len, const tt_bf16* emb,
                                  const tt_bf16* e_mask, const tt_bf16* u_t,
                                  const tt_bf16* shift_scale, const tt_bf16* w,
                                  const tt_bf16* u_ctx, float gamma, float logit_scale,
                                  int32_t* tokens, int32_t* steps_taken, int32_t* commit_step,
                                  int32_t* steps_run, void* ws, size_t ws_bytes, void* stream);

/*
 * The block loop over n_layers denoiser layers ("Architecture" of the
 * gist.science summary: each denoiser layer attends to the frozen context
 * tower's KV of the same layer; each has its own adaLN-single table).  One
 * step: x_0 = the block's embeddings (every position); for each layer l,
 * [q|k|v] = x_l.U_l, o = attention over [Kctx_l ; k] (as
 * tt_block_denoise_attn), x_{l+1} = adaLN_l(o, t_b) for every position
 * (bf16); the last layer's masked rows feed the vocabulary and the commit
 * (as tt_denoise_block_loop).  n_layers = 1 is tt_denoise_block_loop.
 *
 *   n_layers    1 .. 64
 *   k_ctx/v_ctx bf16 [n_layers][B, Hkv, L_cap, dh]   layer outermost
 *   u_t         bf16 [n_layers][H + 2*Hkv*dh, H]
 *   shift_scale bf16 [n_layers][2, H]
 *   other arguments, ownership, workspace (TT_WS_LOOP) and errors as
 *   tt_denoise_block_loop; n_layers outside 1..64 is TT_ERR_INVALID_ARG.
 * The pages fix only the layer alignment; the composition
 * x_{l+1} = adaLN_l(attention_l(x_l)) without a residual is this library's
 * reading (one layer reduces to the single-layer step).
 */
TT_API tt_status tt_denoise_block_loop_layers(const tt_dims* d, int32_t n_layers,
                                              const tt_bf16* k_ctx, const tt_bf16* v_ctx,
                                              const int32_t* ctx_len, const tt_bf16* emb,
                                              const tt_bf16* e_mask, const tt_bf16* u_t,
                                              const tt_bf16* shift_scale, const tt_bf16* w,
                                              float gamma, float logit_scale, int32_t max_steps,
                                              int32_t* tokens, uint8_t* masked,
                                              int32_t* steps_taken, int32_t* commit_step,
                                              int32_t* steps_run, void* ws, size_t ws_bytes,
                                              void* stream);

/*
 * Inspection of the block loop's last step: data copies only, no arithmetic.
 * After tt_denoise_block_loop or tt_denoise_block_loop_layers has returned,
 * its workspace still holds what the last step that did work fed the
 * vocabulary projection - the adaLN rows of the positions masked at the
 * start of that step, compacted in row order - and the confidence and
 * argmax token the commit rule used for each of them.  This call copies them
 * out, so a caller can check the projection and the commit rule on the
 * kernels' own rows (run the loop with max_steps = 1 to see every step; a
 * resumed loop continues exactly where the previous call stopped).  Source
 * of the quantities: gist.science summary, "Training and Conditioning",
 * Sampling (all masked positions are predicted in parallel; confident ones
 * commit).
 *
 *   ws, ws_bytes  the TT_WS_LOOP workspace the loop ran with (read only)
 *   y_rows   bf16 [B*S, H]  rows 0 .. n_rows-1 receive the compacted rows,
 *            the rest are left untouched
 *   row_ids  int32 [B*S]    row_ids[j] = b*S + s of compacted row j (j < n_rows)
 *   conf     float [B*S]    confidence of each position masked at the start
 *            of the step, -1 elsewhere
 *   argmax   int32 [B*S]    its argmax token, -1 elsewhere
 *   n_rows   host int32     number of compacted rows
 * Blocking: synchronises `stream` (the loop's stream) before reading.  A
 * workspace whose row count is out of range (never used by a loop) gives
 * TT_ERR_INTERNAL.
 */
TT_API tt_status tt_loop_last_step(const tt_dims* d, void* ws, size_t ws_bytes, tt_bf16* y_rows,
                                   int32_t* row_ids, float* conf, int32_t* argmax,
                                   int32_t* n_rows, void* stream);

/*
 * Allocation-free variant of tt_vocab_confidence_commit.
 * The paper has no counterpart: this entry point exists for callers that
 * cannot provide a workspace - code running inside another runtime's
 * execution hook where device allocation is not allowed (an inference
 * engine's plugin callback, say), a process whose device memory is fully
 * reserved by its own pool, or a C caller with no allocator at all.
 *
 * Same arguments, results and commit rule as tt_vocab_confidence_commit,
 * minus the workspace.  Its scratch is one built-in device array of 16 MiB
 * (16777216 bytes) that every GPU which loads this library holds until the
 * process exits.  A problem whose scratch exceeds it - 256 bytes of control
 * words, B*4 bytes of per-sequence counters, the masked-row list and its
 * inverse (B*S*8 bytes), B*4 bytes of timesteps, B*S*H*2 bytes of gathered
 * rows, B*S*ceil(V/224)*16 bytes of tile statistics and B*S*8 bytes of row
 * results, each rounded up to 256 bytes - is rejected with
 * TT_ERR_WORKSPACE before any launch.  It allocates nothing:
 * no cudaMalloc/cudaFree and no allocating library routine.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The address is cached per device together
 *    with the identity of the context it belongs to, and looked up again
 *    when the current context differs (after a device reset, whose new
 *    context loads the array anew); a call that does this look-up must not
 *    be captured either.
 *  - All calls share the one array and it keeps the last call's contents;
 *    the call clears what must start at zero.  Calls whose work overlaps on
 *    the GPU (different streams, or several host threads) race on it:
 *    serialise them.
 *  - Device-detected errors (a timed-out wait, a non-finite confidence) are
 *    recorded in the array only; this variant does not report them.
 */
TT_API tt_status tt_vocab_confidence_commit_noalloc(const tt_dims* d, const tt_bf16* y,
                                                    const tt_bf16* w, float gamma,
                                                    float logit_scale, int32_t* tokens,
                                                    uint8_t* masked, float* conf_out,
                                                    int32_t* argmax_out, int32_t* n_committed,
                                                    void* stream);

#ifdef __cplusplus
}
#endif
#endif /* TWOTOWER_H */
