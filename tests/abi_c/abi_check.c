/*
 * A plain C99 client of libqlora: include/qlora.h must compile as C, every
 * entry point must link, and the host-only calls must behave as the header
 * documents. Nothing here launches a kernel, so it runs without a GPU.
 * It also prints the size and field offsets of each struct of the header, one
 * "layout" line per struct, for a binding to compare its own mirrors with.
 * Exit status 0 and "ok" as the last line when every check holds; otherwise
 * each failing check is printed and the status is 1.
 */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "qlora.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      printf("FAILED line %d: %s\n", __LINE__, #cond);                \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

typedef void (*any_fn)(void);

int main(void) {
  /* every entry point of the header, taken by address (the link must resolve all) */
  const any_fn entry[] = {
      (any_fn)qlora_nf4_sizes,           (any_fn)qlora_nf4_codebook,
      (any_fn)qlora_nf4_quantize,        (any_fn)qlora_nf4_dequantize,
      (any_fn)qlora_codec_levels,        (any_fn)qlora_codec_quantize,
      (any_fn)qlora_codec_dequantize,    (any_fn)qlora_dqfp8_sizes,
      (any_fn)qlora_dqfp8_quantize,      (any_fn)qlora_dqfp8_dequantize,
      (any_fn)qlora_linear_workspace,    (any_fn)qlora_linear_fwd,
      (any_fn)qlora_linear_bwd,          (any_fn)qlora_linear_fwd_group_workspace,
      (any_fn)qlora_linear_fwd_group,    (any_fn)qlora_lora_xa,
      (any_fn)qlora_fused_workspace,     (any_fn)qlora_fused_fwd,
      (any_fn)qlora_lora_dyb,            (any_fn)qlora_fused_dx,
      (any_fn)qlora_lora_grads,          (any_fn)qlora_swiglu_fwd,
      (any_fn)qlora_swiglu_bwd,          (any_fn)qlora_swiglu_pack_b,
      (any_fn)qlora_swiglu_unpack_db,    (any_fn)qlora_nf4_merge,
      (any_fn)qlora_adamw8_step,         (any_fn)qlora_lora_grads_adamw8,
      (any_fn)qlora_linear_fwd_noalloc,  (any_fn)qlora_set_gemm_schedule,
      (any_fn)qlora_selftest_bounded_wait, (any_fn)qlora_status_string,
  };
  size_t i;
  for (i = 0; i < sizeof(entry) / sizeof(entry[0]); ++i) CHECK(entry[i] != NULL);

  /* storage of an NF4 matrix: 4 bits per weight, one byte per 64-weight
     block, one float per 256 blocks, i.e. 4.126953125 bits per weight when
     the block count is a multiple of 256 */
  {
    size_t codes = 0, s8 = 0, s2 = 0;
    CHECK(qlora_nf4_sizes(4096, 4096, &codes, &s8, &s2) == QLORA_OK);
    CHECK(codes == (size_t)4096 * 4096 / 2);
    CHECK(s8 == (size_t)4096 * 4096 / 64);
    CHECK(s2 == (size_t)4096 * 4096 / 64 / 256 * 4);
    CHECK((double)(codes + s8 + s2) * 8.0 / (4096.0 * 4096.0) == 4.126953125);
    /* a short last group still gets its own second-level scale */
    CHECK(qlora_nf4_sizes(1, 64 * 257, &codes, &s8, &s2) == QLORA_OK);
    CHECK(s8 == 257 && s2 == 2 * 4);
    CHECK(qlora_nf4_sizes(16, 100, &codes, &s8, &s2) == QLORA_ERR_UNSUPPORTED_SHAPE);
    CHECK(qlora_nf4_sizes(0, 64, &codes, &s8, &s2) == QLORA_ERR_INVALID_ARG);
    CHECK(qlora_nf4_sizes(16, 64, NULL, &s8, &s2) == QLORA_ERR_INVALID_ARG);
  }

  /* the codebook: 16 ascending levels, -1, 0 and 1 exactly, 7 below zero */
  {
    float lv[16];
    int neg = 0;
    memset(lv, 0, sizeof(lv));
    CHECK(qlora_nf4_codebook(lv) == QLORA_OK);
    CHECK(lv[0] == -1.0f && lv[7] == 0.0f && lv[15] == 1.0f);
    for (i = 1; i < 16; ++i) CHECK(lv[i] > lv[i - 1]);
    for (i = 0; i < 16; ++i) neg += lv[i] < 0.0f;
    CHECK(neg == 7);
    CHECK(qlora_nf4_codebook(NULL) == QLORA_ERR_INVALID_ARG);
    CHECK(qlora_codec_levels(QLORA_CODEBOOK_NF4, lv) == QLORA_OK && lv[7] == 0.0f);
    CHECK(qlora_codec_levels(QLORA_CODEBOOK_INT4, lv) == QLORA_OK && lv[8] == 0.0f && lv[0] == -8.0f / 7.0f);
    CHECK(qlora_codec_levels(7, lv) == QLORA_ERR_INVALID_ARG);
  }

  /* argument errors come back before anything is launched */
  {
    qlora_nf4_t q;
    q.rows = 64;
    q.cols = 64;
    q.codes = NULL;
    q.scale8 = NULL;
    q.scale2 = NULL;
    CHECK(qlora_nf4_quantize(NULL, &q, NULL, NULL) == QLORA_ERR_INVALID_ARG);
    CHECK(qlora_nf4_dequantize(&q, NULL, NULL) == QLORA_ERR_INVALID_ARG);
    CHECK(qlora_nf4_dequantize(NULL, NULL, NULL) == QLORA_ERR_INVALID_ARG);
    CHECK(qlora_set_gemm_schedule(99) == QLORA_ERR_INVALID_ARG);
    CHECK(qlora_set_gemm_schedule(QLORA_SCHEDULE_AUTO) == QLORA_OK);
  }

  /* status names */
  {
    const qlora_status_t all[] = {QLORA_OK, QLORA_ERR_INVALID_ARG, QLORA_ERR_UNSUPPORTED_SHAPE,
                                  QLORA_ERR_MISALIGNED, QLORA_ERR_WORKSPACE, QLORA_ERR_NONFINITE,
                                  QLORA_ERR_TIMEOUT, QLORA_ERR_CUDA};
    size_t j;
    for (i = 0; i < sizeof(all) / sizeof(all[0]); ++i) {
      CHECK(qlora_status_string(all[i]) != NULL);
      for (j = 0; j < i; ++j) CHECK(strcmp(qlora_status_string(all[i]), qlora_status_string(all[j])) != 0);
    }
    CHECK(strcmp(qlora_status_string((qlora_status_t)12345), "QLORA_ERR_UNKNOWN") == 0);
  }

  /* the layouts a binding must mirror: "layout <struct> <size> <field>=<offset> ..." */
  printf("layout qlora_nf4_t %u rows=%u cols=%u codes=%u scale8=%u scale2=%u\n", (unsigned)sizeof(qlora_nf4_t),
         (unsigned)offsetof(qlora_nf4_t, rows), (unsigned)offsetof(qlora_nf4_t, cols),
         (unsigned)offsetof(qlora_nf4_t, codes), (unsigned)offsetof(qlora_nf4_t, scale8),
         (unsigned)offsetof(qlora_nf4_t, scale2));
  printf("layout qlora_linear_problem_t %u W=%u X=%u A=%u B=%u r=%u s=%u Y=%u sU_out=%u\n",
         (unsigned)sizeof(qlora_linear_problem_t), (unsigned)offsetof(qlora_linear_problem_t, W),
         (unsigned)offsetof(qlora_linear_problem_t, X), (unsigned)offsetof(qlora_linear_problem_t, A),
         (unsigned)offsetof(qlora_linear_problem_t, B), (unsigned)offsetof(qlora_linear_problem_t, r),
         (unsigned)offsetof(qlora_linear_problem_t, s), (unsigned)offsetof(qlora_linear_problem_t, Y),
         (unsigned)offsetof(qlora_linear_problem_t, sU_out));
  printf("layout qlora_adamw8_tensor_t %u p=%u p_bf16=%u m_q=%u v_q=%u m_scale=%u v_scale=%u\n",
         (unsigned)sizeof(qlora_adamw8_tensor_t), (unsigned)offsetof(qlora_adamw8_tensor_t, p),
         (unsigned)offsetof(qlora_adamw8_tensor_t, p_bf16), (unsigned)offsetof(qlora_adamw8_tensor_t, m_q),
         (unsigned)offsetof(qlora_adamw8_tensor_t, v_q), (unsigned)offsetof(qlora_adamw8_tensor_t, m_scale),
         (unsigned)offsetof(qlora_adamw8_tensor_t, v_scale));

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
