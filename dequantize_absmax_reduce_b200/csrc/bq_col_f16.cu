// Column-group kernels instantiated for __half (templates in bq_col_impl.cuh).
#include "bq_col_impl.cuh"

namespace bq {
BQ_COL_ENTRY(__half, f16)
}  // namespace bq
