/*
 * libtwotower used from plain C (and, compiled as C++, from C++): the status
 * names, workspace sizes and the argument checks that return before any
 * launch.  Nothing here needs a GPU: every pointer is an aligned address that
 * the library rejects or never dereferences.  Exit status 0 when every check
 * holds.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "twotower.h"

static int failures = 0;

#define CHECK(cond)                                                     \
  do {                                                                  \
    if (!(cond)) {                                                      \
      fprintf(stderr, "abi_check.c:%d: %s\n", __LINE__, #cond);         \
      ++failures;                                                       \
    }                                                                   \
  } while (0)

int main(void) {
  /* the mid workload: 8 sequences, 32/2 heads of 128, V = 131072, L = 4096 */
  const tt_dims d = {8, 16, 32, 2, 128, 4096, 131072, 4096};
  tt_dims bad = d;
  const uintptr_t addr = (uintptr_t)1 << 20; /* 16-byte aligned, never dereferenced */
  tt_bf16* bf = (tt_bf16*)addr;
  int32_t* i32 = (int32_t*)addr;
  uint8_t* u8 = (uint8_t*)addr;
  float* f32 = (float*)addr;
  void* ws = (void*)addr;
  int32_t steps_run = -1;
  size_t ws_attn, ws_vocab, ws_loop;

  CHECK(strcmp(tt_status_string(TT_OK), "TT_OK") == 0);
  CHECK(strcmp(tt_status_string(TT_ERR_TIMEOUT), "TT_ERR_TIMEOUT") == 0);
  CHECK(strcmp(tt_status_string((tt_status)99), "TT_ERR_UNKNOWN") == 0);
  CHECK(tt_launch_count() == 0);

  ws_attn = tt_workspace_bytes(&d, TT_WS_ATTN);
  ws_vocab = tt_workspace_bytes(&d, TT_WS_VOCAB);
  ws_loop = tt_workspace_bytes(&d, TT_WS_LOOP);
  CHECK(ws_attn > 0 && ws_vocab > 0);
  CHECK(ws_loop >= ws_attn && ws_loop >= ws_vocab);

  /* an unsupported head size: no workspace size, and the call refuses */
  bad.dh = 96;
  bad.H = bad.Hq * bad.dh;
  CHECK(tt_workspace_bytes(&bad, TT_WS_ATTN) == 0);
  CHECK(strlen(tt_last_error()) > 0);
  CHECK(tt_block_denoise_attn(&bad, bf, bf, bf, bf, bf, i32, bf, ws, ws_attn, NULL) ==
        TT_ERR_UNSUPPORTED);

  /* a missing input, then a workspace one byte short */
  CHECK(tt_block_denoise_attn(&d, NULL, bf, bf, bf, bf, i32, bf, ws, ws_attn, NULL) ==
        TT_ERR_INVALID_ARG);
  CHECK(strstr(tt_last_error(), "q_blk") != NULL);
  CHECK(tt_block_denoise_attn(&d, bf, bf, bf, bf, bf, i32, bf, ws, ws_attn - 1, NULL) ==
        TT_ERR_WORKSPACE);

  /* gamma outside (0, 1] */
  CHECK(tt_vocab_confidence_commit(&d, bf, bf, 1.5f, 1.0f, i32, u8, f32, i32, i32, ws, ws_vocab,
                                   NULL) == TT_ERR_INVALID_ARG);

  /* max_steps outside 1..1024, and n_layers outside 1..64 */
  CHECK(tt_denoise_block_loop(&d, bf, bf, i32, bf, bf, bf, bf, bf, 0.8f, 1.0f, 0, i32, u8, i32, i32,
                              &steps_run, ws, ws_loop, NULL) == TT_ERR_INVALID_ARG);
  CHECK(tt_denoise_block_loop_layers(&d, 0, bf, bf, i32, bf, bf, bf, bf, bf, 0.8f, 1.0f, 4, i32, u8,
                                     i32, i32, &steps_run, ws, ws_loop, NULL) ==
        TT_ERR_INVALID_ARG);

  /* n_blocks outside 1..4096 */
  CHECK(tt_decode_blocks(&d, 0, bf, bf, i32, bf, bf, bf, bf, bf, bf, 0.8f, 1.0f, i32, i32, i32,
                         &steps_run, ws, ws_loop, NULL) == TT_ERR_INVALID_ARG);
  CHECK(tt_decode_blocks(&d, 4097, bf, bf, i32, bf, bf, bf, bf, bf, bf, 0.8f, 1.0f, i32, i32, i32,
                         &steps_run, ws, ws_loop, NULL) == TT_ERR_INVALID_ARG);

  /* the last-step inspection needs a whole loop workspace and an n_rows slot */
  {
    int32_t n_rows = -3;
    CHECK(tt_loop_last_step(&d, ws, ws_loop, bf, i32, f32, i32, NULL, NULL) ==
          TT_ERR_INVALID_ARG);
    CHECK(tt_loop_last_step(&d, ws, ws_vocab, bf, i32, f32, i32, &n_rows, NULL) ==
          TT_ERR_WORKSPACE);
    CHECK(n_rows == -3);
  }

  /* the allocation-free commit refuses a problem beyond its built-in scratch */
  {
    const tt_dims big = {128, 32, 32, 2, 128, 4096, 131072, 32768};
    CHECK(tt_vocab_confidence_commit_noalloc(&big, bf, bf, 0.8f, 1.0f, i32, u8, f32, i32, i32,
                                             NULL) == TT_ERR_WORKSPACE);
  }

  /* the attention split knob is process-wide and bounded */
  CHECK(tt_set_attn_splits(1025) == TT_ERR_INVALID_ARG);
  CHECK(tt_set_attn_splits(0) == TT_OK);
  CHECK(tt_set_loop_graphs(2) == TT_ERR_INVALID_ARG);
  CHECK(tt_set_loop_graphs(1) == TT_OK);

  /* none of the refused calls launched anything */
  CHECK(tt_launch_count() == 0);

  printf(failures ? "abi_check: %d failed\n" : "abi_check: ok\n", failures);
  return failures != 0;
}
