/* A plain C client of libbbattn.so: uses only include/bb_attn.h.  Runs the
 * host-only calls (no GPU needed): the ABI version, the random table (with
 * and without the layer options), workspace sizing and host-side argument
 * validation of the compute calls.  Prints the tables, one row of ids per
 * line, for the caller to compare with an independent generator; exits
 * nonzero on the first failed check. */
#include <stdio.h>
#include <stdlib.h>

#include "bb_attn.h"

#define CHECK(c)                                                  \
  do {                                                            \
    if (!(c)) {                                                   \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                   \
    }                                                             \
  } while (0)

static int print_table(const char* name, const int32_t* t, int H, int nb, int r) {
  int h, i, a;
  printf("table %s %d %d %d\n", name, H, nb, r);
  for (h = 0; h < H; ++h)
    for (i = 0; i < nb; ++i) {
      for (a = 0; a < r; ++a) printf(a ? " %d" : "%d", t[((size_t)h * nb + i) * r + a]);
      printf("\n");
    }
  return 0;
}

int main(void) {
  enum { H = 3, NB = 16, R = 3 };
  int32_t table[H * NB * R], table_ex[H * NB * R];
  int h, i, a;
  size_t ws = 0;
  bb_attn_desc d = {2, H, NB * 64, 64, 64, R, BB_BF16, 0.f, 0.f, 0.f, 0, 0, 0, NULL};
  bb_attn_desc bad = d;
  const uintptr_t fake = (uintptr_t)1 << 20; /* never dereferenced */
  void* p = (void*)fake;

  CHECK(bb_abi_version() == BB_ABI_VERSION);

  CHECK(bb_rand_attn_build(7, H, NB, R, table) == BB_OK);
  for (h = 0; h < H; ++h)
    for (i = 0; i < NB; ++i) {
      const int32_t* row = table + ((size_t)h * NB + i) * R;
      for (a = 0; a < R; ++a) {
        if (i == 0 || i == NB - 1) {
          CHECK(row[a] == -1);
          continue;
        }
        CHECK(row[a] >= 1 && row[a] <= NB - 2);                 /* middle block */
        CHECK(row[a] < i - 1 || row[a] > i + 1);                /* off-window */
        if (a) CHECK(row[a] > row[a - 1]);                      /* sorted, distinct */
      }
    }
  print_table("plain", table, H, NB, R);
  CHECK(bb_rand_attn_build_ex(7, H, NB, R, 64, 16, table_ex) == BB_OK);
  print_table("layer", table_ex, H, NB, R);
  CHECK(bb_rand_attn_build_ex(7, H, NB, R, NB - 1, 0, table_ex) == BB_ERR_INVALID);
  CHECK(bb_rand_attn_build(7, H, NB, R, NULL) == BB_ERR_INVALID);

  CHECK(bb_attn_workspace_size(&d, 0, &ws) == BB_OK && ws > 0);
  CHECK(bb_attn_workspace_size(&d, 1, &ws) == BB_OK && ws > 0);
  bad.L = 1000; /* not a multiple of the block size */
  CHECK(bb_attn_workspace_size(&bad, 0, &ws) == BB_ERR_INVALID);
  bad = d;
  bad.d = 128;
  CHECK(bb_attn_workspace_size(&bad, 0, &ws) == BB_ERR_UNSUPPORTED);
  bad = d;
  bad.dropout = 1.0f;
  CHECK(bb_attn_workspace_size(&bad, 0, &ws) == BB_ERR_INVALID);
  /* dropout keep-bit buffer: 1 bit per attended probability slot */
  CHECK(bb_attn_dropout_bits_size(&d, &ws) == BB_OK && ws == 0);
  bad = d;
  bad.dropout = 0.1f;
  CHECK(bb_attn_dropout_bits_size(&bad, &ws) == BB_OK &&
        ws == (size_t)2 * H * (2 * NB + (NB - 2) * (5 + R)) * 64 * 64 / 8);
  bad.dropout_bits = (void*)(fake + 4); /* misaligned */
  CHECK(bb_attn_dropout_bits_size(&bad, &ws) == BB_ERR_INVALID);

  /* Compute calls: refused on the host before any CUDA call. */
  CHECK(bb_attn_workspace_size(&d, 0, &ws) == BB_OK);
  CHECK(bb_attn_fwd(&d, NULL, p, p, NULL, p, p, (float*)p, p, ws, NULL) == BB_ERR_INVALID);
  CHECK(bb_attn_fwd(NULL, p, p, p, NULL, p, p, (float*)p, p, ws, NULL) == BB_ERR_INVALID);
  CHECK(bb_attn_fwd(&d, p, p, p, NULL, p, p, (float*)p, p, ws - 1, NULL) == BB_ERR_WORKSPACE);
  CHECK(bb_attn_workspace_size(&d, 1, &ws) == BB_OK);
  CHECK(bb_attn_bwd(&d, p, p, p, p, (const float*)p, p, NULL, p, p, p, NULL, p, ws, NULL) ==
        BB_ERR_INVALID); /* dv NULL */
  CHECK(bb_status_str(BB_ERR_TIMEOUT) != NULL);
  printf("ok\n");
  return 0;
}
