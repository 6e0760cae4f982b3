/* Plain C client of the library's C ABI (host-side calls only): the header
 * compiles as C, the library links, and the host entry points behave as the
 * header states.  Built and run by tests/test_c_abi.py; prints "ok" on success. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "w4a16.h"

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                       \
    }                                                                 \
  } while (0)

int main(void) {
  enum { N = 40, K = 256 };
  CHECK(w4a16_version() > 0);
  CHECK(w4a16_packed_weight_bytes(W4A16_FMT_INT4_G128, N, K) == 48 * K / 2);
  CHECK(w4a16_packed_scale_bytes(W4A16_FMT_INT4_G128, N, K) == 48 * (K / 128) * 2);
  CHECK(w4a16_packed_weight_bytes(W4A16_FMT_FP8_E4M3, N, K) == 48 * K);
  CHECK(w4a16_packed_scale_bytes(W4A16_FMT_FP8_E4M3, N, K) == 0);
  CHECK(strncmp(w4a16_status_string(W4A16_ERR_SHAPE), "W4A16_ERR_SHAPE", 15) == 0);

  /* int4 round trip through the host packer */
  int8_t* q = (int8_t*)malloc(N * K);
  uint16_t* s = (uint16_t*)malloc(N * (K / 128) * 2);
  uint8_t* pw = (uint8_t*)malloc(w4a16_packed_weight_bytes(W4A16_FMT_INT4_G128, N, K));
  uint8_t* ps = (uint8_t*)malloc(w4a16_packed_scale_bytes(W4A16_FMT_INT4_G128, N, K));
  int8_t* q2 = (int8_t*)malloc(N * K);
  uint16_t* s2 = (uint16_t*)malloc(N * (K / 128) * 2);
  for (int i = 0; i < N * K; ++i) q[i] = (int8_t)((i * 7 + 3) % 16 - 8);
  for (int i = 0; i < N * (K / 128); ++i) s[i] = (uint16_t)(0x3C00 + i);
  CHECK(w4a16_pack_host(W4A16_FMT_INT4_G128, N, K, q, s, pw, ps) == W4A16_OK);
  CHECK(w4a16_unpack_host(W4A16_FMT_INT4_G128, N, K, pw, ps, q2, s2) == W4A16_OK);
  CHECK(memcmp(q, q2, N * K) == 0 && memcmp(s, s2, N * (K / 128) * 2) == 0);
  q[5] = 9; /* out of range */
  CHECK(w4a16_pack_host(W4A16_FMT_INT4_G128, N, K, q, s, pw, ps) == W4A16_ERR_ARG);

  /* validation before any device call */
  CHECK(w4a16_gemm(W4A16_FMT_INT4_G128, 0, N, K, pw, pw, ps, NULL, pw, NULL) == W4A16_ERR_SHAPE);
  CHECK(w4a16_gemm(7, 1, N, K, pw, pw, ps, NULL, pw, NULL) == W4A16_ERR_ARG);
  CHECK(w4a16_gemm_gate_up_silu(W4A16_FMT_INT4_G128, 1, 24, K, pw, pw, ps, NULL, pw, NULL) ==
        W4A16_ERR_SHAPE);
  CHECK(w4a16_gemm_path(W4A16_FMT_INT4_G128, 1, 17408, 5120) == W4A16_PATH_GEMV);
  CHECK(w4a16_gemm_path(W4A16_FMT_INT4_G128, 64, 34816, 5120) == W4A16_PATH_TC);

  /* the planner, on the host */
  int plan[9];
  CHECK(w4a16_plan(W4A16_PATH_AUTO, W4A16_FMT_INT4_G128, 64, 34816, 5120, 0, 148, plan, 9) ==
        W4A16_PATH_TC);
  CHECK(plan[0] == 1 && plan[2] == 64 && plan[7] <= 227 * 1024);

  free(q); free(s); free(pw); free(ps); free(q2); free(s2);
  printf("ok\n");
  return 0;
}
