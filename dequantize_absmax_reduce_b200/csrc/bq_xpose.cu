// Packed weight / scale transpose (metrale QuantizedWeight
// transpose_for_gemm(_gs) and transpose_concat_for_gemm_padded with one
// part): bytes [rows, cols] -> [cols, stride], stride = align_up(rows, align),
// columns [rows, stride) of the output zeroed. Packed E2M1 bytes move whole,
// so their nibble order is unchanged.
//
// k_xpose: a CTA moves a 64 x 64 byte tile. Each thread reads a 4 x 4 byte
// block as four 32-bit words (coalesced along the input rows), transposes it
// in registers with byte permutes, and parks the four output words in shared
// memory; the CTA then writes 16-byte runs along the output rows.
#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {

__global__ void __launch_bounds__(256) k_xpose(const uint8_t* __restrict__ in, int64_t rows,
                                               int64_t cols, int64_t stride, int64_t ntr,
                                               uint8_t* __restrict__ out) {
    __shared__ uint32_t sm[64][17];
    const int64_t tr = blockIdx.x % ntr;          // tile along input rows / output columns
    const int64_t tc = blockIdx.x / ntr;          // tile along input columns / output rows
    const int64_t r0 = tr * 64, c0 = tc * 64;
    const int t = threadIdx.x;
    {
        const int rb = t >> 4, cb = t & 15;
        const int64_t c = c0 + 4 * cb;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t r = r0 + 4 * rb + i;
            w[i] = (r < rows && c < cols) ? __ldg(reinterpret_cast<const uint32_t*>(in + r * cols + c)) : 0u;
        }
        const uint32_t a_lo = __byte_perm(w[0], w[1], 0x5140), a_hi = __byte_perm(w[0], w[1], 0x7362);
        const uint32_t b_lo = __byte_perm(w[2], w[3], 0x5140), b_hi = __byte_perm(w[2], w[3], 0x7362);
        sm[4 * cb + 0][rb] = __byte_perm(a_lo, b_lo, 0x5410);
        sm[4 * cb + 1][rb] = __byte_perm(a_lo, b_lo, 0x7632);
        sm[4 * cb + 2][rb] = __byte_perm(a_hi, b_hi, 0x5410);
        sm[4 * cb + 3][rb] = __byte_perm(a_hi, b_hi, 0x7632);
    }
    __syncthreads();
    {
        const int orow = t >> 2, seg = t & 3;
        const int64_t oc = c0 + orow;                 // output row
        const int64_t ob = r0 + 16 * seg;             // output byte column
        if (oc < cols && ob < stride) {
            U4 v;
            v.x = sm[orow][4 * seg + 0];
            v.y = sm[orow][4 * seg + 1];
            v.z = sm[orow][4 * seg + 2];
            v.w = sm[orow][4 * seg + 3];
            st16(out + oc * stride + ob, v);
        }
    }
}

// Any shape / alignment: one output byte per thread step.
__global__ void __launch_bounds__(256) k_xpose_scalar(const uint8_t* __restrict__ in, int64_t rows,
                                                      int64_t cols, int64_t stride,
                                                      uint8_t* __restrict__ out) {
    const int64_t n = cols * stride;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t oc = i / stride, orr = i % stride;
        out[i] = (orr < rows) ? __ldg(in + orr * cols + oc) : (uint8_t)0;
    }
}

cudaError_t byte_transpose(const uint8_t* in, int64_t rows, int64_t cols, int64_t stride,
                           uint8_t* out, cudaStream_t st) {
    if (cols == 0 || stride == 0) return cudaSuccess;
    const bool vec = (cols % 4 == 0) && (stride % 16 == 0) && ((uintptr_t)in % 4 == 0) &&
                     ((uintptr_t)out % 16 == 0);
    if (vec) {
        const int64_t ntr = (stride + 63) / 64, ntc = (cols + 63) / 64;
        const int64_t nb = ntr * ntc;
        if (nb > 0x7FFFFFFFll) return cudaErrorInvalidValue;
        k_xpose<<<(unsigned)nb, 256, 0, st>>>(in, rows, cols, stride, ntr, out);
    } else {
        int64_t need = (cols * stride + 255) / 256;
        const int64_t cap = (int64_t)sm_count() * 8;
        k_xpose_scalar<<<(unsigned)(need < cap ? need : cap), 256, 0, st>>>(in, rows, cols, stride, out);
    }
    return cudaGetLastError();
}

}  // namespace bq
