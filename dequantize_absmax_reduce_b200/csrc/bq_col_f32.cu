// Column-group kernels instantiated for float (templates in bq_col_impl.cuh).
#include "bq_col_impl.cuh"

namespace bq {
BQ_COL_ENTRY(float, f32)
}  // namespace bq
