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

// Wide tiles for the common case (cols % 16 == 0, stride % 16 == 0, 16-byte
// aligned buffers): a CTA moves a 64-row x 256-byte tile. Thread (rb, cb) =
// (t % 16, t / 16) loads rows 4rb..4rb+3 at bytes 16cb..16cb+15 (four 16-byte
// loads; a warp reads 32 full-sector bytes from each of 16 rows), transposes
// the four 4x4 byte blocks in registers and parks sixteen output words in
// shared memory (the 32 lanes of one store hit 32 distinct banks); the CTA
// then writes each of the tile's 256 output rows as four 16-byte runs. Two
// independent transposes (weights and scales) share one launch: blocks
// [0, jobs[0].n_tiles) serve the first.
struct XJob {
    const uint8_t* in;
    int64_t rows, cols, stride, ntr, n_tiles;
    uint8_t* out;
};
struct XJobs { XJob j[2]; };

__global__ void __launch_bounds__(256) k_xpose_wide(XJobs jobs) {
    __shared__ uint32_t sm[256][17];                  // [output row][input-row word], padded
    const bool second = (int64_t)blockIdx.x >= jobs.j[0].n_tiles;
    const XJob& J = second ? jobs.j[1] : jobs.j[0];
    const int64_t b = second ? (int64_t)blockIdx.x - jobs.j[0].n_tiles : (int64_t)blockIdx.x;
    const int64_t tr = b % J.ntr, tc = b / J.ntr;
    const int64_t r0 = tr * 64, c0 = tc * 256;
    const int t = threadIdx.x;
    {
        const int rb = t & 15, cb = t >> 4;
        const int64_t c = c0 + 16 * cb;
        U4 w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t r = r0 + 4 * rb + i;
            w[i] = (r < J.rows && c < J.cols) ? ld16_stream(J.in + r * J.cols + c) : U4{0u, 0u, 0u, 0u};
        }
        const uint32_t x0[4] = {w[0].x, w[0].y, w[0].z, w[0].w};
        const uint32_t x1[4] = {w[1].x, w[1].y, w[1].z, w[1].w};
        const uint32_t x2[4] = {w[2].x, w[2].y, w[2].z, w[2].w};
        const uint32_t x3[4] = {w[3].x, w[3].y, w[3].z, w[3].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            // 4x4 bytes: rows 4rb+i, columns 16cb+4q+j -> word j holds byte j of each row.
            const uint32_t a_lo = __byte_perm(x0[q], x1[q], 0x5140), a_hi = __byte_perm(x0[q], x1[q], 0x7362);
            const uint32_t b_lo = __byte_perm(x2[q], x3[q], 0x5140), b_hi = __byte_perm(x2[q], x3[q], 0x7362);
            const int orow = 16 * cb + 4 * q;
            sm[orow + 0][rb] = __byte_perm(a_lo, b_lo, 0x5410);
            sm[orow + 1][rb] = __byte_perm(a_lo, b_lo, 0x7632);
            sm[orow + 2][rb] = __byte_perm(a_hi, b_hi, 0x5410);
            sm[orow + 3][rb] = __byte_perm(a_hi, b_hi, 0x7632);
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int orow = 64 * k + (t >> 2), seg = t & 3;
        const int64_t oc = c0 + orow;                 // output row
        const int64_t ob = r0 + 16 * seg;             // output byte column
        if (oc < J.cols && ob < J.stride) {
            U4 v;
            v.x = sm[orow][4 * seg + 0];
            v.y = sm[orow][4 * seg + 1];
            v.z = sm[orow][4 * seg + 2];
            v.w = sm[orow][4 * seg + 3];
            st16(J.out + oc * J.stride + ob, v);
        }
    }
}

static bool xpose_wide_ok(const uint8_t* in, int64_t cols, int64_t stride, const uint8_t* out) {
    return cols % 16 == 0 && stride % 16 == 0 && ((uintptr_t)in % 16 == 0) && ((uintptr_t)out % 16 == 0);
}
static XJob make_xjob(const uint8_t* in, int64_t rows, int64_t cols, int64_t stride, uint8_t* out) {
    XJob j;
    j.in = in; j.rows = rows; j.cols = cols; j.stride = stride; j.out = out;
    j.ntr = (stride + 63) / 64;
    j.n_tiles = j.ntr * ((cols + 255) / 256);
    if (cols == 0 || stride == 0) j.n_tiles = 0;
    return j;
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

cudaError_t byte_transpose2(const uint8_t* in0, int64_t rows0, int64_t cols0, uint8_t* out0,
                            const uint8_t* in1, int64_t rows1, int64_t cols1, uint8_t* out1,
                            int64_t stride, cudaStream_t st) {
    const bool wide0 = xpose_wide_ok(in0, cols0, stride, out0);
    const bool wide1 = !in1 || xpose_wide_ok(in1, cols1, stride, out1);
    if (wide0 && wide1) {
        XJobs jobs;
        jobs.j[0] = make_xjob(in0, rows0, cols0, stride, out0);
        jobs.j[1] = in1 ? make_xjob(in1, rows1, cols1, stride, out1) : make_xjob(nullptr, 0, 0, 0, nullptr);
        const int64_t nb = jobs.j[0].n_tiles + jobs.j[1].n_tiles;
        if (nb == 0) return cudaSuccess;
        if (nb > 0x7FFFFFFFll) return cudaErrorInvalidValue;
        k_xpose_wide<<<(unsigned)nb, 256, 0, st>>>(jobs);
        return cudaGetLastError();
    }
    cudaError_t e = byte_transpose(in0, rows0, cols0, stride, out0, st);
    if (e == cudaSuccess && in1) e = byte_transpose(in1, rows1, cols1, stride, out1, st);
    return e;
}

}  // namespace bq
