/*
 * c_consumer.c -- a plain C11 user of libfmoe.so's headers (no CUDA headers, no C++).
 *
 * Built and run by tests/test_c_consumer.py on a machine without a GPU: it makes only
 * the calls that need none (layout and size queries, status strings, argument checks)
 * and prints what it sees as `key value` lines, which the test compares with the
 * Python binding's view of the same structs and calls.
 */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fmoe.h"
#include "fmoe_cache.h"
#include "fmoe_gdn.h"

static fmoe_bank fake_bank(int bits, int H, int I, int E) {
  fmoe_bank b;
  int64_t rec = 0;
  memset(&b, 0, sizeof(b));
  b.bits = bits;
  b.group_size = 64;
  b.hidden = H;
  b.inter = I;
  b.num_experts = E;
  b.base = (const void*)(uintptr_t)0x10000000u; /* never dereferenced: no call here launches */
  if (fmoe_bank_layout(bits, 64, H, I, &rec, b.off) != FMOE_OK) return b;
  b.stride = rec;
  return b;
}

int main(void) {
  int64_t rec = 0, off[9];
  int k;
  fmoe_layer L;

  printf("version %d\n", fmoe_version());
  printf("debug_bounds %d\n", fmoe_debug_bounds());
  printf("sizeof_bank %zu\n", sizeof(fmoe_bank));
  printf("sizeof_layer %zu\n", sizeof(fmoe_layer));
  printf("sizeof_cache %zu\n", sizeof(fmoe_expert_cache));
  printf("offsetof_bank_base %zu\n", offsetof(fmoe_bank, base));
  printf("offsetof_bank_off %zu\n", offsetof(fmoe_bank, off));
  printf("offsetof_layer_shared %zu\n", offsetof(fmoe_layer, shared));
  printf("offsetof_layer_eps %zu\n", offsetof(fmoe_layer, eps));
  printf("offsetof_layer_top_k %zu\n", offsetof(fmoe_layer, top_k));
  printf("offsetof_cache_num_experts %zu\n", offsetof(fmoe_expert_cache, num_experts));
  printf("offsetof_cache_state %zu\n", offsetof(fmoe_expert_cache, state));
  for (k = 0; k <= 7; ++k) printf("status_%d %s\n", k, fmoe_status_string((fmoe_status)k));
  printf("gdn_state_early %u\n", (unsigned)FMOE_GDN_STATE_EARLY);
  printf("static_scratch_bytes %d\n", (int)FMOE_STATIC_SCRATCH_BYTES);

  if (fmoe_bank_layout(4, 64, 4096, 1024, &rec, off) != FMOE_OK) return 1;
  printf("record_bytes_4bit %lld\n", (long long)rec);
  printf("record_off_4bit");
  for (k = 0; k < 9; ++k) printf(" %lld", (long long)off[k]);
  printf("\n");
  if (fmoe_bank_layout(2, 64, 4096, 1024, &rec, off) != FMOE_OK) return 1;
  printf("record_bytes_2bit %lld\n", (long long)rec);

  memset(&L, 0, sizeof(L));
  L.routed = fake_bank(4, 4096, 1024, 512);
  L.shared = fake_bank(4, 4096, 1024, 1);
  L.w_router = (const uint16_t*)(uintptr_t)0x20000000u;
  L.w_shared_gate = (const uint16_t*)(uintptr_t)0x30000000u;
  L.gamma = (const float*)(uintptr_t)0x40000000u;
  L.eps = 1e-6f;
  L.top_k = 4;
  printf("layer_ws_1 %zu\n", fmoe_moe_layer_workspace_size(&L, 1));
  printf("layer_ws_64 %zu\n", fmoe_moe_layer_workspace_size(&L, 64));
  printf("router_ws_1_512 %zu\n", fmoe_router_topk_workspace_size(1, 512));
  printf("ffn_ws %zu\n", fmoe_expert_ffn_workspace_size(&L.routed));
  printf("cache_state_512_64 %zu\n", fmoe_expert_cache_state_size(512, 64));

  /* argument errors come back as status codes, before anything touches a device */
  printf("null_layer %d\n", (int)fmoe_moe_layer(NULL, NULL, 1, NULL, NULL, NULL, NULL, 0, NULL));
  printf("null_layer_message %s\n", strlen(fmoe_last_error()) > 0 ? "set" : "empty");
  printf("empty_batch %d\n", (int)fmoe_moe_layer(&L, (const float*)(uintptr_t)0x60000000u, 0,
                                                 (float*)(uintptr_t)0x60000000u, NULL, NULL, NULL, 0, NULL));
  printf("short_workspace %d\n", (int)fmoe_moe_layer(&L, (const float*)(uintptr_t)0x60000000u, 1,
                                                     (float*)(uintptr_t)0x60000000u, NULL, NULL,
                                                     (void*)(uintptr_t)0x50000000u, 1024, NULL));
  L.top_k = 0;
  printf("bad_top_k %d\n", (int)fmoe_moe_layer(&L, (const float*)(uintptr_t)0x60000000u, 1,
                                               (float*)(uintptr_t)0x60000000u, NULL, NULL,
                                               (void*)(uintptr_t)0x50000000u, (size_t)1 << 30, NULL));
  printf("gdn_null_state %d\n", (int)fmoe_gdn_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 64, 128, 128, 0u, NULL));
  return 0;
}
