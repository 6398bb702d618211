// Column-group kernels instantiated for __nv_bfloat16 (templates in bq_col_impl.cuh).
#include "bq_col_impl.cuh"

namespace bq {
BQ_COL_ENTRY(__nv_bfloat16, bf16)
}  // namespace bq
