// Pipelined quantize kernels instantiated for float (templates in bq_pipe_impl.cuh).
#include "bq_pipe_impl.cuh"

namespace bq {
BQ_PIPE_ENTRIES(float, f32)
}  // namespace bq
