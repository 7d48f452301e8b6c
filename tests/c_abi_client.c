/* A plain C client of libkca.so, built and run by tests/test_c_abi_cpu.py:
 * it uses the library through include/kca.h alone (no Python, no torch) and
 * prints, one per line, what the host-only calls return -- status strings,
 * the integer plans of a prefill chunk and of a decode batch, and the codes
 * of calls rejected on the host -- for the test to compare with the Python
 * binding.  Nothing here touches a GPU. */
#include <stdint.h>
#include <stdio.h>

#include "kca.h"

static void print_items(const char *tag, const int64_t *items, int32_t n, int32_t extra) {
  int64_t sum = 0, mix = 0;
  for (int32_t i = 0; i < 4 * n; ++i) {
    sum += items[i];
    mix = (mix * 1000003 + items[i]) % 2147483647;
  }
  printf("%s n=%d extra=%d sum=%lld mix=%lld\n", tag, n, extra, (long long)sum, (long long)mix);
}

int main(void) {
  static int64_t items[4 * 4096];
  const int32_t cap[3] = {74, 33, 15};
  int32_t n = 0, path = -1, cluster = -1;

  for (int s = 0; s >= -8; --s) printf("status %d %s\n", s, attn_status_string(s));

  /* a tensor-core prefill chunk, a window chunk, a few-row chunk (rows path) */
  const int64_t starts[3] = {7680, 3840, 1000};
  const int32_t rows[3] = {768, 256, 9}, windows[3] = {0, 512, 0}, dts[3] = {KCA_BF16, KCA_BF16, KCA_F32};
  for (int c = 0; c < 3; ++c) {
    const int st = attn_prefill_plan(dts[c], dts[c], starts[c], rows[c], windows[c], 148, cap, items, 4096, &n,
                                     &path);
    char tag[64];
    snprintf(tag, sizeof tag, "prefill_plan %lld %d %d st=%d", (long long)starts[c], rows[c], windows[c], st);
    print_items(tag, items, n, path);
  }

  /* a ragged decode batch on the tensor-core kernel, given capacities */
  const int64_t ctx[4] = {16384, 1000, 0, 131072};
  int st = attn_decode_plan(4, ctx, 0, KCA_F16, 148, cap, items, 4096, &n, &cluster);
  char tag[64];
  snprintf(tag, sizeof tag, "decode_plan st=%d", st);
  print_items(tag, items, n, cluster);

  /* rejected on the host, before any device call */
  float out_dummy[4];
  printf("reject prefill_null_q %d\n",
         attn_prefill(NULL, KCA_BF16, items, items, KCA_BF16, 8, 1, 256, 1024, 0, 16, 16, 0, 0.0625f, out_dummy,
                      items, 1 << 20, NULL));
  printf("reject prefill_heads %d\n",
         attn_prefill(items, KCA_BF16, items, items, KCA_BF16, 4, 1, 256, 1024, 0, 16, 16, 0, 0.0625f, out_dummy,
                      items, 1 << 20, NULL));
  printf("reject prefill_rows %d\n",
         attn_prefill(items, KCA_BF16, items, items, KCA_BF16, 8, 1, 256, 1024, 0, 769, 769, 0, 0.0625f, out_dummy,
                      items, 1 << 20, NULL));
  printf("reject decode_dtype %d\n",
         attn_decode(items, 7, items, items, KCA_F16, 8, 1, 256, 1024, 1, ctx + 1, 0, 0.0625f, out_dummy, items,
                     1 << 20, NULL));
  printf("reject decode_batch %d\n",
         attn_decode(items, KCA_F32, items, items, KCA_F16, 8, 1, 256, 1024, 0, ctx + 1, 0, 0.0625f, out_dummy,
                     items, 1 << 20, NULL));
  printf("reject plan_capacity %d\n", attn_decode_plan(1, ctx, 0, KCA_F16, 148, (const int32_t[3]){74, -1, 15},
                                                       items, 4096, &n, &cluster));
  return 0;
}
