/* A plain C99 caller of libtp: include/tp.h must compile as C and the library must link and answer
 * without a GPU on every path that returns before a launch (validation, empty inputs, sizes). Each
 * line printed is "name value"; tests/test_c_abi.py compiles this file, runs it and checks the lines. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "tp.h"

int main(void) {
  const void* in2[2] = {0, 0};
  void* out2[2] = {0, 0};
  const uint16_t* w4[4] = {0, 0, 0, 0};
  void* c4[4] = {0, 0, 0, 0};
  float* f4[4] = {0, 0, 0, 0};
  const uintptr_t fake = (uintptr_t)1 << 20;   /* 16-byte aligned, never dereferenced */
  const void* fin3[3] = {(const void*)fake, (const void*)fake, (const void*)fake};
  void* fout3[3] = {(void*)fake, (void*)fake, (void*)fake};

  printf("status_ok %s\n", tp_status_str(TP_OK));
  printf("status_unknown %s\n", tp_status_str((tp_status)99));
  /* empty inputs: OK with null data pointers, nothing launched */
  printf("empty_rs %d\n", (int)tp_reduce_scatter(in2, out2, 0, 16, 0, TP_F32, 2, NULL));
  printf("empty_mlp %d\n", (int)tp_mlp_fwd(NULL, 0, 256, 1024, 4, TP_ACT_GELU, NULL, NULL, NULL, NULL,
                                           TP_OUT_RS, f4, NULL));
  /* validation before launch */
  printf("bad_t %d\n", (int)tp_reduce_scatter(in2, out2, 16, 16, 0, TP_F32, 0, NULL));
  printf("indivisible %d\n", (int)tp_reduce_scatter(fin3, fout3, 16, 16, 0, TP_F32, 3, NULL));
  printf("last_error_nonempty %d\n", (int)(strlen(tp_last_error()) > 0));
  printf("negative %d\n", (int)tp_all_gather(in2, out2, -2, 16, 0, TP_BF16, 2, NULL));
  printf("empty_contraction %d\n", (int)tp_sharded_matmul(3, TP_CASE3_RS_B, w4, w4, 64, 0, 64, 4,
                                                          c4, TP_F32, NULL, 0, NULL));
  /* workspace sizes (host arithmetic) */
  printf("ws_case4_gather_w %zu\n", tp_sharded_matmul_ws_bytes(4, TP_CASE4_GATHER_W, 8192, 8192, 28672, 4));
  printf("ws_case4_gather_w_ragged %zu\n", tp_sharded_matmul_ws_bytes(4, TP_CASE4_GATHER_W, 8192, 8192, 384, 4));
  printf("ws_case3_fused %zu\n", tp_sharded_matmul_ws_bytes(3, TP_CASE3_RS_B, 8192, 8192, 28672, 4));
  /* strategy choice by the pages' byte rule (host arithmetic) */
  {
    int st2 = -1, st4 = -1;
    tp_status a = tp_sharded_matmul_choose(2, 8192, 8192, 28672, 4, &st2);
    tp_status b = tp_sharded_matmul_choose(4, 8192, 8192, 28672, 4, &st4);
    printf("choose_case2 %d %d\n", (int)a, st2);
    printf("choose_case4 %d %d\n", (int)b, st4);
    printf("choose_case3 %d\n", (int)tp_sharded_matmul_choose(3, 8192, 8192, 28672, 4, &st2));
  }
  return 0;
}
