// Pipelined quantize kernels instantiated for __nv_bfloat16 (templates in bq_pipe_impl.cuh).
#include "bq_pipe_impl.cuh"

namespace bq {
BQ_PIPE_ENTRIES(__nv_bfloat16, bf16)
}  // namespace bq
