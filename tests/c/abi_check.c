/* The C ABI used from plain C99 (no C++, no Python): the header compiles as
 * C, and the host-side entry points behave as declared.  CPU only: the
 * decode and cache entry points are called only with arguments they must
 * refuse before touching a device.  Exit status 0 = every check held. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pagedattn.h"

static int failures = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  /* status names and version */
  CHECK(strcmp(pa_status_string(PA_OK), "PA_OK") == 0);
  CHECK(strcmp(pa_status_string(PA_ERR_OUT_OF_BLOCKS), "PA_ERR_OUT_OF_BLOCKS") == 0);
  CHECK(pa_version() >= 200);

  /* arguments refused before any launch */
  CHECK(pa_decode_attention(NULL, PA_BF16, NULL, NULL, NULL, NULL, 1, NULL, 4, 16, 4, 2, 64, 8,
                            4, 0.125f, PA_BF16, 0, NULL, 0, NULL, NULL) == PA_ERR_INVALID_ARG);
  CHECK(pa_reshape_and_cache(NULL, NULL, 128, 128, NULL, NULL, NULL, 4, 8, 4, 2, 64, PA_F16,
                             PA_KV_AUTO, NULL, NULL, NULL, NULL) == PA_ERR_INVALID_ARG);
  CHECK(pa_stream_read((const void*)(uintptr_t)4096, 100, (uint32_t*)(uintptr_t)4096, 4, NULL) ==
        PA_ERR_INVALID_ARG);

  /* the decode step from host buffers: refusals made before any device work */
  {
    pa_step_shape sh;
    memset(&sh, 0, sizeof(sh));
    sh.num_seqs = 2; sh.num_q_heads = 4; sh.num_kv_heads = 2; sh.head_dim = 64;
    sh.num_blocks = 8; sh.block_size = 16; sh.table_width = 4; sh.max_seq_len = 64;
    sh.dtype = PA_F16; sh.out_dtype = PA_F16; sh.kv_cache_dtype = PA_KV_AUTO;
    char host[64];
    pa_step_layout lay;
    CHECK(pa_decode_step_layout(NULL, &lay) == PA_ERR_INVALID_ARG);
    CHECK(pa_decode_step_layout(&sh, NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_decode_step(NULL, host, 0, host, host, NULL, NULL, 0.125f, host, 64, host, NULL,
                         NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_decode_step(&sh, NULL, 0, host, host, NULL, NULL, 0.125f, host, 64, host, NULL,
                         NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_decode_step(&sh, host, 0, host, host, NULL, NULL, 0.125f, host, 64, NULL, NULL,
                         NULL) == PA_ERR_INVALID_ARG);
    sh.table_width = 3; /* below ceil(64 / 16) */
    CHECK(pa_decode_step_layout(&sh, &lay) == PA_ERR_INVALID_ARG);
    sh.table_width = 4;
    sh.head_dim = 96; /* not a built head size */
    CHECK(pa_decode_step_layout(&sh, &lay) == PA_ERR_UNSUPPORTED);
    sh.head_dim = 64;
    sh.dtype = PA_F32; /* the query and new rows are 16-bit */
    CHECK(pa_decode_step_layout(&sh, &lay) == PA_ERR_UNSUPPORTED);
  }

  /* the split plan on the host: 4 sequences (1, 3, 0 and 7 tiles) over 7
   * CTAs.  Weighted line: the three sequences with tiles start at virtual
   * tiles 0, 4 and 10 (3 more each), 20 in all; cut at 0, 2, 5, 8, 11, 14, 17,
   * 20 -> first tiles 0, 0, 1, 2, 4, 5, 8, 11 */
  {
    const int32_t lens4[4] = {5, 40, 0, 100};
    int32_t tiles[5], segs[5], start[7], firstk[7], ctalo[8], nseg = -1, comb = -1;
    CHECK(pa_split_plan(lens4, 4, 128, 0, 7, tiles, segs, start, firstk, ctalo, &nseg, &comb) ==
          PA_OK);
    CHECK(tiles[0] == 0 && tiles[1] == 1 && tiles[2] == 4 && tiles[3] == 4 && tiles[4] == 11);
    CHECK(ctalo[0] == 0 && ctalo[1] == 0 && ctalo[2] == 1 && ctalo[3] == 2 && ctalo[4] == 4 &&
          ctalo[5] == 5 && ctalo[6] == 8 && ctalo[7] == 11);
    CHECK(segs[1] == 1 && segs[2] == 3 && segs[3] == 3 && segs[4] == 6 && nseg == 6 && comb == 1);
    CHECK(start[3] == 1 && firstk[3] == 1 && start[6] == 3 && firstk[6] == 2);
    CHECK(pa_split_plan(lens4, 4, 64, 0, 7, tiles, segs, start, firstk, ctalo, &nseg, &comb) ==
          PA_ERR_INVALID_ARG); /* a length above max_seq_len */
    char plan[64];
    CHECK(pa_decode_plan(NULL, 4, 4, 2, 64, 16, 128, 0, PA_KV_AUTO, plan, 64, NULL) ==
          PA_ERR_INVALID_ARG);
  }

  /* block manager: parallel sampling with copy-on-write */
  pa_block_manager* bm = NULL;
  CHECK(pa_bm_create(16, 4, NULL, &bm) == PA_OK && bm != NULL);
  CHECK(pa_bm_add_sequence(bm, 0, 6) == PA_OK);   /* blocks 0, 1 (2 tokens in 1) */
  CHECK(pa_bm_fork(bm, 0, 1) == PA_OK);
  int64_t seqs[2] = {0, 1};
  int64_t need = -1;
  CHECK(pa_bm_blocks_needed(bm, seqs, 2, NULL, &need) == PA_OK && need == 1);
  int32_t slots[2], pairs[4], ncow = -1;
  CHECK(pa_bm_append_slots(bm, seqs, 2, slots, pairs, &ncow) == PA_OK);
  CHECK(ncow == 1 && pairs[0] == 1 && pairs[1] == 2);      /* seq 0 copies block 1 */
  CHECK(slots[0] == 2 * 4 + 2 && slots[1] == 1 * 4 + 2);   /* seq 1 writes in place */
  int32_t tables[2 * 3], lens[2];
  CHECK(pa_bm_fill_tables(bm, seqs, 2, tables, 3, lens) == PA_OK);
  CHECK(tables[0] == 0 && tables[1] == 2 && tables[2] == -1);
  CHECK(tables[3] == 0 && tables[4] == 1 && tables[5] == -1);
  CHECK(lens[0] == 7 && lens[1] == 7);
  pa_bm_stats_t st;
  CHECK(pa_bm_stats(bm, &st) == PA_OK);
  CHECK(st.held_blocks == 3 && st.logical_blocks == 4 && st.tokens == 14);
  CHECK(st.stored_slots == 10 && st.waste_slots == 2 && st.free_blocks == 13);

  /* prefix caching: a second request with the same 9-token prompt shares
   * the two full blocks */
  int32_t prompt[9] = {11, 12, 13, 14, 21, 22, 23, 24, 31};
  int64_t cached = -1;
  CHECK(pa_bm_add_sequence_with_prefix(bm, 5, prompt, 9, &cached) == PA_OK && cached == 0);
  CHECK(pa_bm_add_sequence_with_prefix(bm, 6, prompt, 9, &cached) == PA_OK && cached == 8);
  CHECK(pa_bm_add_sequence_with_prefix(bm, 6, prompt, 9, &cached) == PA_ERR_INVALID_ARG);
  CHECK(pa_bm_free_sequence(bm, 42) == PA_ERR_NOT_FOUND);
  pa_bm_destroy(bm);

  if (failures == 0) printf("abi_check: all checks held\n");
  return failures == 0 ? 0 : 1;
}
