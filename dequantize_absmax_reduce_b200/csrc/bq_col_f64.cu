// Column-group kernels instantiated for double (templates in bq_col_impl.cuh).
#include "bq_col_impl.cuh"

namespace bq {
BQ_COL_ENTRY(double, f64)
}  // namespace bq
