/* Prints the size and every field offset of the argument structs in include/fp8q.h, as the
 * host C compiler lays them out, one "name value" pair per line. */
#include <stddef.h>
#include <stdio.h>

#include "fp8q.h"

#define F(T, f) printf("%s.%s %zu\n", #T, #f, offsetof(T, f))

int main(void) {
  printf("fp8q_gemm_args %zu\n", sizeof(fp8q_gemm_args));
  F(fp8q_gemm_args, recipe); F(fp8q_gemm_args, layout); F(fp8q_gemm_args, M); F(fp8q_gemm_args, N);
  F(fp8q_gemm_args, K); F(fp8q_gemm_args, a); F(fp8q_gemm_args, a_scale); F(fp8q_gemm_args, lda);
  F(fp8q_gemm_args, ld_sa); F(fp8q_gemm_args, b); F(fp8q_gemm_args, b_scale); F(fp8q_gemm_args, ldb);
  F(fp8q_gemm_args, ld_sb); F(fp8q_gemm_args, a_global); F(fp8q_gemm_args, b_global); F(fp8q_gemm_args, c);
  F(fp8q_gemm_args, ldc); F(fp8q_gemm_args, m_offsets); F(fp8q_gemm_args, num_groups);
  F(fp8q_gemm_args, c_fp32_accumulate); F(fp8q_gemm_args, a_format); F(fp8q_gemm_args, b_format);
  F(fp8q_gemm_args, q_out); F(fp8q_gemm_args, s_out); F(fp8q_gemm_args, ld_q_out); F(fp8q_gemm_args, ld_s_out);
  F(fp8q_gemm_args, workspace); F(fp8q_gemm_args, workspace_bytes);
  printf("fp8q_quant_item %zu\n", sizeof(fp8q_quant_item));
  F(fp8q_quant_item, kind); F(fp8q_quant_item, x); F(fp8q_quant_item, rows); F(fp8q_quant_item, cols);
  F(fp8q_quant_item, ld_x); F(fp8q_quant_item, q_row); F(fp8q_quant_item, s_row); F(fp8q_quant_item, ld_s_row);
  F(fp8q_quant_item, q_col); F(fp8q_quant_item, s_col); F(fp8q_quant_item, ld_s_col); F(fp8q_quant_item, q_t);
  F(fp8q_quant_item, q); F(fp8q_quant_item, s);
  return 0;
}
