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
// aligned buffers): a CTA of 128 threads moves a 64-row x 512-byte tile.
// Warp w holds input rows 16w..16w+15 and lane l the 16 bytes 16l..16l+15 of
// each (sixteen 16-byte loads; one load instruction reads 512 contiguous
// bytes of one row). The lane's 16 x 16 byte block is transposed in
// registers (sixteen 4 x 4 byte transposes by byte permutes) into sixteen
// 16-byte pieces of output rows 16l..16l+15, stored to shared memory whole;
// the CTA then writes each output row's 64 bytes as four 16-byte runs.
// Shared memory holds the 512 output rows x 64 bytes as pairs of rows per
// 128-byte line, the eight 16-byte slots of a line permuted by XOR with
// bits 4-6 of the row: the eight lanes of a store phase (rows 16 apart) and
// of a load phase (two rows of one line) then touch eight distinct slots.
// Up to XJOBS independent transposes share one launch (the weights and
// scales of every part of a concatenation); job j owns blocks [first_j,
// first_j + n_tiles_j). A job writes bytes [0, olim) of each output row from
// its base `out` (a part's column offset into the shared rows); input rows
// beyond `rows` read as zero, which fills the pad columns of the last part.
constexpr int XJOBS = 8;
constexpr int XT_ROWS = 64, XT_COLS = 512, XT_THREADS = 128;
struct XJob {
    const uint8_t* in;
    int64_t rows, cols, stride, olim, ntr, n_tiles, first;
    uint8_t* out;
};
struct XJobs {
    XJob j[XJOBS];
    int n;
};

// Byte offset in the staging tile of output row `orow`, 16-byte piece `c`
// (input rows 16c..16c+15 of the tile).
__device__ __forceinline__ uint32_t xt_slot(int orow, int c) {
    return (uint32_t)(orow >> 1) * 128u + 16u * (uint32_t)((c + 4 * (orow & 1)) ^ ((orow >> 4) & 7));
}

__global__ void __launch_bounds__(XT_THREADS) k_xpose_wide(XJobs jobs) {
    __shared__ __align__(128) uint8_t sm[XT_COLS * XT_ROWS];
    int ji = 0;
#pragma unroll 1
    for (int q = 1; q < jobs.n; ++q)
        if ((int64_t)blockIdx.x >= jobs.j[q].first) ji = q;
    const XJob& J = jobs.j[ji];
    const int64_t b = (int64_t)blockIdx.x - J.first;
    const int64_t tr = b % J.ntr, tc = b / J.ntr;
    const int64_t r0 = tr * XT_ROWS, c0 = tc * XT_COLS;
    const int t = threadIdx.x, lane = t & 31, rg = t >> 5;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
    {
        const int64_t c = c0 + 16 * lane;
        U4 w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int64_t r = r0 + 16 * rg + i;
            w[i] = (r < J.rows && c < J.cols) ? ld16_stream(J.in + r * J.cols + c) : U4{0u, 0u, 0u, 0u};
        }
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {               // input bytes 4bb..4bb+3 of the lane's 16
            uint32_t o[4][4];                          // [j][ib]: output row 4bb + j, input rows 4ib..4ib+3
#pragma unroll
            for (int ib = 0; ib < 4; ++ib) {
                const uint32_t x0 = (&w[4 * ib + 0].x)[bb], x1 = (&w[4 * ib + 1].x)[bb];
                const uint32_t x2 = (&w[4 * ib + 2].x)[bb], x3 = (&w[4 * ib + 3].x)[bb];
                const uint32_t a_lo = __byte_perm(x0, x1, 0x5140), a_hi = __byte_perm(x0, x1, 0x7362);
                const uint32_t b_lo = __byte_perm(x2, x3, 0x5140), b_hi = __byte_perm(x2, x3, 0x7362);
                o[0][ib] = __byte_perm(a_lo, b_lo, 0x5410);
                o[1][ib] = __byte_perm(a_lo, b_lo, 0x7632);
                o[2][ib] = __byte_perm(a_hi, b_hi, 0x5410);
                o[3][ib] = __byte_perm(a_hi, b_hi, 0x7632);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int orow = 16 * lane + 4 * bb + j;
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                             :: "r"(sbase + xt_slot(orow, rg)), "r"(o[j][0]), "r"(o[j][1]), "r"(o[j][2]),
                                "r"(o[j][3]) : "memory");
            }
        }
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < XT_COLS * XT_ROWS / 16 / XT_THREADS; ++k) {
        const int idx = k * XT_THREADS + t;
        const int orow = idx >> 2, seg = idx & 3;
        const int64_t oc = c0 + orow;                 // output row
        const int64_t ob = r0 + 16 * seg;             // output byte column
        if (oc < J.cols && ob < J.olim) {
            U4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(sbase + xt_slot(orow, seg)));
            st16(J.out + oc * J.stride + ob, v);
        }
    }
}

static bool xpose_wide_ok(const uint8_t* in, int64_t cols, int64_t stride, int64_t olim,
                          const uint8_t* out) {
    return cols % 16 == 0 && stride % 16 == 0 && olim % 16 == 0 && ((uintptr_t)in % 16 == 0) &&
           ((uintptr_t)out % 16 == 0);
}
static XJob make_xjob(const uint8_t* in, int64_t rows, int64_t cols, int64_t stride, int64_t olim,
                      uint8_t* out) {
    XJob j;
    j.in = in; j.rows = rows; j.cols = cols; j.stride = stride; j.olim = olim; j.out = out;
    j.ntr = (olim + XT_ROWS - 1) / XT_ROWS;
    j.n_tiles = j.ntr * ((cols + XT_COLS - 1) / XT_COLS);
    if (cols == 0 || olim == 0) j.n_tiles = 0;
    j.first = 0;
    return j;
}

// Byte-wise transpose of one job (any widths and alignments): output byte
// (oc, o) for o < olim is in[o][oc] for o < rows, else 0.
__global__ void __launch_bounds__(256) k_xpose_bytes(const uint8_t* __restrict__ in, int64_t rows,
                                                     int64_t cols, int64_t stride, int64_t olim,
                                                     uint8_t* __restrict__ out) {
    const int64_t n = cols * olim;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t oc = i / olim, o = i - oc * olim;
        out[oc * stride + o] = (o < rows) ? __ldg(in + o * cols + oc) : (uint8_t)0;
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

cudaError_t byte_transpose2(const uint8_t* in0, int64_t rows0, int64_t cols0, uint8_t* out0,
                            const uint8_t* in1, int64_t rows1, int64_t cols1, uint8_t* out1,
                            int64_t stride, cudaStream_t st) {
    XPart parts[2] = {{in0, rows0, cols0, out0, stride}, {in1, rows1, cols1, out1, stride}};
    return byte_transpose_parts(parts, in1 ? 2 : 1, stride, st);
}

cudaError_t byte_transpose_parts(const XPart* parts, int n_parts, int64_t stride, cudaStream_t st) {
    bool wide = stride % 16 == 0;
    for (int i = 0; i < n_parts && wide; ++i)
        wide = xpose_wide_ok(parts[i].in, parts[i].cols, stride, parts[i].olim, parts[i].out);
    if (wide) {
        for (int i0 = 0; i0 < n_parts; i0 += XJOBS) {
            XJobs jobs{};
            int64_t nb = 0;
            jobs.n = 0;
            for (int i = i0; i < n_parts && i < i0 + XJOBS; ++i) {
                XJob j = make_xjob(parts[i].in, parts[i].rows, parts[i].cols, stride, parts[i].olim,
                                   parts[i].out);
                j.first = nb;
                nb += j.n_tiles;
                jobs.j[jobs.n++] = j;
            }
            if (nb == 0) continue;
            if (nb > 0x7FFFFFFFll) return cudaErrorInvalidValue;
            k_xpose_wide<<<(unsigned)nb, XT_THREADS, 0, st>>>(jobs);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    for (int i = 0; i < n_parts; ++i) {
        const XPart& p = parts[i];
        if (p.cols == 0 || p.olim == 0) continue;
        if (p.olim == stride && p.rows <= stride) {
            const cudaError_t e = byte_transpose(p.in, p.rows, p.cols, stride, p.out, st);
            if (e != cudaSuccess) return e;
            continue;
        }
        const int64_t need = (p.cols * p.olim + 255) / 256;
        const int64_t cap = (int64_t)sm_count() * 8;
        k_xpose_bytes<<<(unsigned)(need < cap ? need : cap), 256, 0, st>>>(p.in, p.rows, p.cols, stride,
                                                                           p.olim, p.out);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace bq
