// Pipelined quantize kernels instantiated for __half (templates in bq_pipe_impl.cuh).
#include "bq_pipe_impl.cuh"

namespace bq {
BQ_PIPE_ENTRIES(__half, f16)
}  // namespace bq
