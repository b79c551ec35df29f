/* The host-only behaviour of libmimoattn, called from C99 through include/mimoattn.h:
 * linkage, the window helper, the workspace queries and argument validation (every call
 * here returns before touching a device).  Built and run by tests/test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "mimoattn.h"

#define CHECK(c)                                                      \
  do {                                                                \
    if (!(c)) {                                                       \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                       \
    }                                                                 \
  } while (0)

static mimo_layer model_layer(int num_kv_heads) {
  mimo_layer L;
  memset(&L, 0, sizeof(L));
  L.num_q_heads = 64;
  L.num_kv_heads = num_kv_heads;
  L.head_dim_qk = 192;
  L.head_dim_v = 128;
  L.rope_dim = 64;
  L.rope_base = 1e4;
  L.softmax_scale = 0.07216878f;
  L.v_scale = 0.707f;
  L.window = 128;
  return L;
}

int main(void) {
  int w = -5;
  CHECK(strstr(mimo_version(), "sm_100a") != NULL);

  CHECK(mimo_window_from_left_right(128, 0, &w) == MIMO_OK && w == 129);
  CHECK(mimo_window_from_left_right(127, 0, &w) == MIMO_OK && w == 128);
  CHECK(mimo_window_from_left_right(-1, 0, &w) == MIMO_OK && w == 0);
  CHECK(mimo_window_from_left_right(128, 1, &w) == MIMO_ERR_UNSUPPORTED);
  CHECK(strstr(mimo_last_error(), "mimo_window_from_left_right") != NULL);
  CHECK(mimo_window_from_left_right(5, 0, NULL) == MIMO_ERR_INVALID_ARG);

  CHECK(mimo_attn_prefill_workspace_size(8, 40696, 40696, 8, MIMO_CACHE_NONE) > 0);
  CHECK(mimo_attn_decode_workspace_size(64, 65536, 4, 0) > 0);

  CHECK(mimo_attn_prefill(NULL, NULL) == MIMO_ERR_INVALID_ARG);
  CHECK(mimo_attn_decode(NULL, NULL) == MIMO_ERR_INVALID_ARG);
  CHECK(mimo_kv_append(NULL, NULL) == MIMO_ERR_INVALID_ARG);
  {
    mimo_prefill_args a;
    memset(&a, 0, sizeof(a));
    a.layer = model_layer(8);
    a.layer.head_dim_qk = 128; /* not the model's 192 */
    a.num_seqs = 1;
    CHECK(mimo_attn_prefill(&a, NULL) == MIMO_ERR_UNSUPPORTED);
    a.layer = model_layer(6); /* neither 8 nor 4 KV heads */
    CHECK(mimo_attn_prefill(&a, NULL) == MIMO_ERR_UNSUPPORTED);
    a.layer = model_layer(8);
    a.num_seqs = 0;
    CHECK(mimo_attn_prefill(&a, NULL) == MIMO_ERR_INVALID_ARG);
    a.num_seqs = 1;
    a.total_q = 0; /* nothing to do */
    CHECK(mimo_attn_prefill(&a, NULL) == MIMO_OK);
  }
  {
    mimo_decode_args d;
    memset(&d, 0, sizeof(d));
    d.layer = model_layer(4);
    d.layer.window = -1;
    d.batch = 1;
    CHECK(mimo_attn_decode(&d, NULL) == MIMO_ERR_INVALID_ARG);
    d.layer.window = 0;
    d.batch = 0; /* an empty batch is a no-op */
    CHECK(mimo_attn_decode(&d, NULL) == MIMO_OK);
    d.ring_slots = 136; /* not a multiple of the 16-key tile */
    d.batch = 1;
    d.max_seq_len = 16;
    d.cache_kind = MIMO_CACHE_RING;
    CHECK(mimo_attn_decode(&d, NULL) == MIMO_ERR_INVALID_ARG);
    CHECK(strstr(mimo_last_error(), "ring_slots") != NULL);
  }
  {
    mimo_prefill_args a;
    memset(&a, 0, sizeof(a));
    a.layer = model_layer(8);
    /* the stall test checks its wait limit before anything else */
    CHECK(mimo_attn_prefill_stall_test(&a, NULL, 10ull) == MIMO_ERR_INVALID_ARG);
  }
  CHECK(MIMO_STATUS_TIMEOUT == 1u && MIMO_STATUS_BAD_INDEX == 2u && MIMO_STATUS_RANGE == 4u &&
        MIMO_STATUS_BAD_SCALE == 8u);
  CHECK(MIMO_RING_SLOTS_DEFAULT == 128 && MIMO_RING_SLOTS_MAX == 512);
  printf("ok\n");
  return 0;
}
