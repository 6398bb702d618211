// Microscaled formats: FP8 E4M3 with f32 scales per 1x128 group or 128x128
// tile (smile llm.quant Fp8BlockGemm / Fp8BlockDequant), MXFP8 with an E8M0
// scale per 32 (smile llm.quant MxFp8), and NVFP4 with E2M1 codes packed two
// per byte, an E4M3 scale per 16 and an f32 per-tensor scale (metrale
// QuantizedWeight).
//
// k_mx_quant: contiguous groups of 16 / 32 / 128 elements along a row, one
//   team of 2..32 lanes per group, 16-byte streaming loads, the group held in
//   registers between its amax and its codes (one HBM pass; NVFP4 also reads
//   the per-tensor range record written by a prior amax pass).
// k_fp8_tile: one CTA per 128x128 tile (or ragged / unaligned 1x128 group).
// k_mx_deq: element-wise decode with the group's scale.
#include <type_traits>

#include "bq_device.cuh"
#include "bq_internal.h"
#include "bq_quant_ops.cuh"

namespace bq {

struct MxArgs {
    const void* x;
    int64_t n_seg;
    uint8_t* codes;
    void* scales;
    const unsigned long long* amax_rec;
    float* global_scale;
    int static_global;
};

// Lanes per group and vectors per lane for each format / element size: each
// lane holds NV vectors of its group so that the per-group work (amax
// shuffles, scale, reciprocal) is shared by many elements.
template <class T, int FMT> struct MxShape {
    static constexpr int VEC = Traits<T>::VEC;
    static constexpr int U = MxG<FMT>::G / VEC;              // vectors per group
    static constexpr int NV = (U >= 4) ? 4 : U;
    static constexpr int TEAM = U / NV;
    static constexpr int SEGS = (NV == 2) ? 4 : 2;
};

template <class T, int FMT>
__global__ void __launch_bounds__(256) k_mx_quant(MxArgs a) {
    using S = MxShape<T, FMT>;
    constexpr int VEC = S::VEC, NV = S::NV, TEAM = S::TEAM, SEGS = S::SEGS;
    constexpr int G = MxG<FMT>::G;
    constexpr int TPW = 32 / TEAM;
    constexpr int CB = (FMT == MX_NVFP4 || FMT == MX_MXFP4) ? VEC / 2 : VEC;   // code bytes per vector
    const T* __restrict__ x = (const T*)a.x;
    const int lane = threadIdx.x & 31;
    const int tm = lane / TEAM, l = lane % TEAM;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t per_chunk = (int64_t)SEGS * TPW;
    const int64_t n_chunks = (a.n_seg + per_chunk - 1) / per_chunk;

    float s2 = 1.0f;
    Recip R6;
    if constexpr (FMT == MX_NVFP4) {
        if (a.static_global == 1) {
            s2 = *a.global_scale;
        } else {
            float h, n;
            range_from_bits(a.amax_rec[0], h);
            range_from_bits(a.amax_rec[1], n);
            s2 = __fdiv_rn(fmaxf(h, n), 2688.0f);    // 2688 = 448 * 6
            if (s2 == 0.0f) s2 = 1.0f;
            if (blockIdx.x == 0 && threadIdx.x == 0) *a.global_scale = s2;
        }
        R6 = make_recip(__fmul_rn(6.0f, s2));
    }

    for (int64_t c = gwarp; c < n_chunks; c += nwarps) {
        U4 raw[SEGS][NV];
#pragma unroll
        for (int r = 0; r < SEGS; ++r) {
            const int64_t seg = c * per_chunk + r * TPW + tm;
#pragma unroll
            for (int j = 0; j < NV; ++j)
                raw[r][j] = (seg < a.n_seg) ? ld16_nc(x + seg * G + (j * TEAM + l) * VEC)
                                            : U4{0u, 0u, 0u, 0u};
        }
#pragma unroll
        for (int r = 0; r < SEGS; ++r) {
            const int64_t seg = c * per_chunk + r * TPW + tm;
            float v[NV][VEC];
            float am = 0.0f;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                load_vec<T>(raw[r][j], v[j]);
#pragma unroll
                for (int i = 0; i < VEC; ++i) am = fmaxf(am, fabsf(v[j][i]));
            }
#pragma unroll
            for (int o = TEAM / 2; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
            const bool ok = seg < a.n_seg;
            uint8_t* base = a.codes + seg * (G / VEC) * CB;
            if constexpr (FMT == MX_FP8_1x128) {
                float s = __fdiv_rn(am, 448.0f);
                if (s == 0.0f) s = 1.0f;
                if (ok && l == 0) ((float*)a.scales)[seg] = s;
                const Recip R = make_recip(s);
                if (ok) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) {
                        if (R.fast) mx_emit<T, FMT, true>(v[j], R, 0.f, false, base + (j * TEAM + l) * CB);
                        else mx_emit<T, FMT, false>(v[j], R, 0.f, false, base + (j * TEAM + l) * CB);
                    }
                }
            } else if constexpr (FMT == MX_MXFP8 || FMT == MX_MXFP4) {
                const int E = mx_exponent(am, FMT == MX_MXFP4 ? 2 : 8);
                if (ok && l == 0) ((uint8_t*)a.scales)[seg] = (uint8_t)(E + 127);
                const Recip R{};
                const float mul = exp2i(-E);
                if (ok) {
#pragma unroll
                    for (int j = 0; j < NV; ++j)
                        mx_emit<T, FMT, true>(v[j], R, mul, false, base + (j * TEAM + l) * CB);
                }
            } else {
                const float q6 = div_any(am, R6);                 // a_b / (6 s2)
                const uint32_t sb = e4m3x2(q6, 0.0f) & 0xFFu;
                if (ok && l == 0) ((uint8_t*)a.scales)[seg] = (uint8_t)sb;
                const float eff = __fmul_rn(e4m3_to_f32(sb), s2);
                const Recip R = make_recip(eff);
                const bool fast = R.fast && a.static_global != 1;
                if (ok) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) {
                        if (fast) mx_emit<T, FMT, true>(v[j], R, 0.f, eff == 0.0f, base + (j * TEAM + l) * CB);
                        else mx_emit<T, FMT, false>(v[j], R, 0.f, eff == 0.0f, base + (j * TEAM + l) * CB);
                    }
                }
            }
        }
    }
}

// Scalar fallback for unaligned inputs: one thread per group.
template <class T, int FMT>
__global__ void __launch_bounds__(256) k_mx_quant_scalar(MxArgs a) {
    constexpr int G = MxG<FMT>::G;
    const T* __restrict__ x = (const T*)a.x;
    float s2 = 1.0f;
    Recip R6;
    if constexpr (FMT == MX_NVFP4) {
        if (a.static_global == 1) {
            s2 = *a.global_scale;
        } else {
            float h, n;
            range_from_bits(a.amax_rec[0], h);
            range_from_bits(a.amax_rec[1], n);
            s2 = __fdiv_rn(fmaxf(h, n), 2688.0f);
            if (s2 == 0.0f) s2 = 1.0f;
            if (blockIdx.x == 0 && threadIdx.x == 0) *a.global_scale = s2;
        }
        R6 = make_recip(__fmul_rn(6.0f, s2));
    }
    for (int64_t seg = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; seg < a.n_seg;
         seg += (int64_t)gridDim.x * blockDim.x) {
        const T* p = x + seg * G;
        float am = 0.0f;
        for (int i = 0; i < G; ++i) am = fmaxf(am, fabsf(ld1<T>(p + i)));
        if constexpr (FMT == MX_FP8_1x128) {
            float s = __fdiv_rn(am, 448.0f);
            if (s == 0.0f) s = 1.0f;
            ((float*)a.scales)[seg] = s;
            const Recip R = make_recip(s);
            for (int i = 0; i < G; i += 2) {
                const float v0 = ld1<T>(p + i), v1 = ld1<T>(p + i + 1);
                const uint32_t w = e4m3x2(with_quotient_sign(div_any(v0, R), v0, s),
                                          with_quotient_sign(div_any(v1, R), v1, s));
                a.codes[seg * G + i] = (uint8_t)w;
                a.codes[seg * G + i + 1] = (uint8_t)(w >> 8);
            }
        } else if constexpr (FMT == MX_MXFP4) {
            const int E = mx_exponent(am, 2);
            ((uint8_t*)a.scales)[seg] = (uint8_t)(E + 127);
            const float inv = exp2i(-E);
            for (int i = 0; i < G; i += 8) {
                float t[8];
                for (int j = 0; j < 8; ++j) t[j] = __fmul_rn(ld1<T>(p + i + j), inv);
                const uint32_t w = e2m1x8(t);
                uint8_t* d = a.codes + (seg * G + i) / 2;
                d[0] = (uint8_t)w; d[1] = (uint8_t)(w >> 8); d[2] = (uint8_t)(w >> 16); d[3] = (uint8_t)(w >> 24);
            }
        } else if constexpr (FMT == MX_MXFP8) {
            const int E = mx_exponent(am);
            ((uint8_t*)a.scales)[seg] = (uint8_t)(E + 127);
            const float inv = exp2i(-E);
            for (int i = 0; i < G; i += 2) {
                const uint32_t w = e4m3x2(__fmul_rn(ld1<T>(p + i), inv), __fmul_rn(ld1<T>(p + i + 1), inv));
                a.codes[seg * G + i] = (uint8_t)w;
                a.codes[seg * G + i + 1] = (uint8_t)(w >> 8);
            }
        } else {
            const uint32_t sb = e4m3x2(div_any(am, R6), 0.0f) & 0xFFu;
            ((uint8_t*)a.scales)[seg] = (uint8_t)sb;
            const float eff = __fmul_rn(e4m3_to_f32(sb), s2);
            const Recip R = make_recip(eff);
            for (int i = 0; i < G; i += 8) {
                float t[8];
                for (int j = 0; j < 8; ++j) {
                    const float v = ld1<T>(p + i + j);
                    t[j] = with_quotient_sign(div_any(v, R), v, eff);
                }
                const uint32_t w = (eff == 0.0f) ? 0u : e2m1x8(t);
                uint8_t* d = a.codes + (seg * G + i) / 2;
                d[0] = (uint8_t)w; d[1] = (uint8_t)(w >> 8); d[2] = (uint8_t)(w >> 16); d[3] = (uint8_t)(w >> 24);
            }
        }
    }
}

// ------------------------------------------------------------ FP8 tiles
// One CTA per br x 128 block; a block on the bottom / right edge may be
// partial. VECP: cols % VEC == 0 and x 16-byte aligned.
template <class T, int BR, int NTH, bool VECP>
__global__ void __launch_bounds__(NTH) k_fp8_tile(const T* __restrict__ x, int64_t rows,
                                                  int64_t cols, int64_t nbc, uint8_t* e4m3,
                                                  float* scale) {
    constexpr int BC = 128;
    constexpr int W = VECP ? Traits<T>::VEC : 1;
    constexpr int IPR = BC / W;                     // items per block row
    constexpr int NI = (BR * IPR + NTH - 1) / NTH;  // items per thread
    constexpr int NW = NTH / 32;
    __shared__ float sh[NW];
    const int64_t bi = blockIdx.x / nbc, bj = blockIdx.x % nbc;
    const int tid = threadIdx.x;
    float v[NI][W];
    bool ok[NI];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int item = tid + i * NTH;
        const int64_t r = bi * BR + item / IPR;
        const int64_t c = bj * BC + (int64_t)(item % IPR) * W;
        ok[i] = (item < BR * IPR) && (r < rows) && (c < cols);
        if (ok[i]) {
            if constexpr (VECP) load_vec<T>(ld16_stream(x + r * cols + c), v[i]);
            else v[i][0] = ld1<T>(x + r * cols + c);
        } else {
#pragma unroll
            for (int k = 0; k < W; ++k) v[i][k] = 0.0f;
        }
#pragma unroll
        for (int k = 0; k < W; ++k) am = fmaxf(am, fabsf(v[i][k]));
    }
    am = warp_max(am);
    if ((tid & 31) == 0) sh[tid >> 5] = am;
    __syncthreads();
    am = sh[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) am = fmaxf(am, sh[w]);
    float s = __fdiv_rn(am, 448.0f);
    if (s == 0.0f) s = 1.0f;
    if (tid == 0) scale[blockIdx.x] = s;
    const Recip R = make_recip(s);
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        if (!ok[i]) continue;
        const int item = tid + i * NTH;
        const int64_t r = bi * BR + item / IPR;
        const int64_t c = bj * BC + (int64_t)(item % IPR) * W;
        float t[W];
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const float d = R.fast ? div_chain(v[i][k], R) : __fdiv_rn(v[i][k], s);
            t[k] = with_quotient_sign(d, v[i][k], s);
        }
        uint8_t* dst = e4m3 + r * cols + c;
        if constexpr (W == 8) {
            st8(dst, e4m3x4(t[0], t[1], t[2], t[3]), e4m3x4(t[4], t[5], t[6], t[7]));
        } else if constexpr (W == 4) {
            st4(dst, e4m3x4(t[0], t[1], t[2], t[3]));
        } else {
            *dst = (uint8_t)e4m3x2(t[0], 0.0f);
        }
    }
}

// ------------------------------------------------------------ dequantize
struct DeqArgs {
    const uint8_t* codes;
    const void* scales;
    const float* global_scale;
    int64_t rows, k;           // row length k (cols for FP8 blocks)
    int br, bc;                // FP8 block shape
    int64_t nbc;               // FP8 blocks per row of blocks
    int64_t numel;
    FastDiv fk;
    int use_fd;
    void* y;
};

template <int FMT>
__device__ __forceinline__ float mx_group_mul(const DeqArgs& a, int64_t r, int64_t c, float s2) {
    if constexpr (FMT == MX_NVFP4) {
        const uint32_t sb = __ldg(((const uint8_t*)a.scales) + r * (a.k / 16) + c / 16);
        return __fmul_rn(e4m3_to_f32(sb), s2);
    } else if constexpr (FMT == MX_MXFP8 || FMT == MX_MXFP4) {
        const uint32_t b = __ldg(((const uint8_t*)a.scales) + r * (a.k / 32) + c / 32);
        return (b == 0xFFu) ? __uint_as_float(0x7FC00000u) : exp2i((int)b - 127);
    } else {
        return __ldg(((const float*)a.scales) + (r / a.br) * a.nbc + c / a.bc);
    }
}

// FMT as above; MX_FP8_1x128 here covers every FP8 block shape.
template <class T, int FMT, bool VECP>
__global__ void __launch_bounds__(256) k_mx_deq(DeqArgs a) {
    constexpr int W = VECP ? 16 : 1;
    const float s2 = (FMT == MX_NVFP4) ? __ldg(a.global_scale) : 1.0f;
    const int64_t n_items = a.numel / W;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < n_items;
         it += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e0 = it * W;
        const int64_t r = a.use_fd ? (int64_t)fdiv((uint32_t)e0, a.fk) : e0 / a.k;
        const int64_t c = e0 - r * a.k;
        const float mul = mx_group_mul<FMT>(a, r, c, s2);
        float o[W];
        if constexpr (FMT == MX_NVFP4 || FMT == MX_MXFP4) {
            if constexpr (VECP) {
                const uint2 w = __ldg(reinterpret_cast<const uint2*>(a.codes + e0 / 2));
                const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const float2 f = e2m1x2_to_f32((ws[h] >> (8 * b)) & 0xFFu);
                        o[h * 8 + 2 * b] = __fmul_rn(f.x, mul);
                        o[h * 8 + 2 * b + 1] = __fmul_rn(f.y, mul);
                    }
            } else {
                const uint32_t byte = __ldg(a.codes + e0 / 2);
                const float2 f = e2m1x2_to_f32(byte);
                o[0] = __fmul_rn((e0 & 1) ? f.y : f.x, mul);
            }
        } else {
            if constexpr (VECP) {
                const uint4 w = __ldg(reinterpret_cast<const uint4*>(a.codes + e0));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 f0 = e4m3x2_to_f32(ws[h] & 0xFFFFu);
                    const float2 f1 = e4m3x2_to_f32(ws[h] >> 16);
                    o[4 * h] = __fmul_rn(f0.x, mul);
                    o[4 * h + 1] = __fmul_rn(f0.y, mul);
                    o[4 * h + 2] = __fmul_rn(f1.x, mul);
                    o[4 * h + 3] = __fmul_rn(f1.y, mul);
                }
            } else {
                o[0] = __fmul_rn(e4m3_to_f32(__ldg(a.codes + e0)), mul);
            }
        }
        T* y = (T*)a.y + e0;
        if constexpr (VECP) {
            constexpr int VEC = Traits<T>::VEC;
#pragma unroll
            for (int h = 0; h < 16 / VEC; ++h) {
                float part[VEC];
#pragma unroll
                for (int k = 0; k < VEC; ++k) part[k] = o[h * VEC + k];
                st16(y + h * VEC, pack_vec<T>(part));
            }
        } else {
            *y = to_out<T>(o[0]);
        }
    }
}

// ------------------------------------------------------------ dequantize, coalesced
// Flat stream of items of 8 elements: 4 code bytes (NVFP4) or 8 (FP8), and
// one 16-byte vector of 16-bit outputs, so that consecutive lanes write
// consecutive 16 bytes and each warp store covers 512 contiguous bytes. Each
// thread issues DQ_U item loads, with their scales, before it decodes any.
// NVFP4 and MXFP8 scales are laid out like the elements ([rows, k/16],
// [rows, k/32]): the scale of element e is scale[e / 16] or scale[e / 32].
// FP8 block scales need the row and column of e.
constexpr int DQ_U = 8;

template <class T>
__device__ __forceinline__ void st_vals8(T* y, const float (&o)[8]) {
    if constexpr (sizeof(T) == 2) {
        st16(y, pack_vec<T>(o));
    } else {
        st16(y, U4{__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]), __float_as_uint(o[3])});
        st16(y + 4, U4{__float_as_uint(o[4]), __float_as_uint(o[5]), __float_as_uint(o[6]), __float_as_uint(o[7])});
    }
}
// Eight E2M1 codes (one word, low nibble first) times m, as f32 products.
__device__ __forceinline__ void e2m1x8_mul(uint32_t w, F2 m2, float (&o)[8]) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const float2 f = e2m1x2_to_f32((w >> (8 * b)) & 0xFFu);
        f2_split(f2_mul(f2_pack(f.x, f.y), m2), o[2 * b], o[2 * b + 1]);
    }
}
// Eight E4M3 codes (two words, low byte first) times m.
__device__ __forceinline__ void e4m3x8_mul(uint32_t w0, uint32_t w1, F2 m2, float (&o)[8]) {
    const uint32_t w[2] = {w0, w1};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float2 a = e4m3x2_to_f32(w[h] & 0xFFFFu), b = e4m3x2_to_f32(w[h] >> 16);
        f2_split(f2_mul(f2_pack(a.x, a.y), m2), o[4 * h], o[4 * h + 1]);
        f2_split(f2_mul(f2_pack(b.x, b.y), m2), o[4 * h + 2], o[4 * h + 3]);
    }
}
// Multiplier of an MXFP8 scale byte: 2^(b-127), NaN for 0xFF.
__device__ __forceinline__ float e8m0_mul(uint32_t b) {
    return (b == 0xFFu) ? __uint_as_float(0x7FC00000u) : exp2i((int)b - 127);
}

// FP8 block scale index of the item starting at element e0. BR: block rows
// (1 or 128); BR = 0: 1x128 blocks on rows of whole blocks, where the index
// is e0 / 128. FD: the element count is below 2^32 (32-bit row division).
template <int BR, bool FD>
__device__ __forceinline__ int64_t fp8_block_index(const DeqArgs& a, int64_t it) {
    if constexpr (BR < 0) {
        return 0;                 // one scale for the whole tensor
    } else if constexpr (BR == 0) {
        return it >> 4;
    } else if constexpr (FD) {
        const uint32_t e0 = (uint32_t)it * 8u;
        const uint32_t r = fdiv(e0, a.fk);
        const uint32_t c = e0 - r * (uint32_t)a.k;
        const uint32_t rb = (BR == 1) ? r : (r >> 7);
        return (int64_t)rb * a.nbc + (c >> 7);
    } else {
        const int64_t e0 = it * 8;
        const int64_t r = e0 / a.k;
        const int64_t c = e0 - r * a.k;
        const int64_t rb = (BR == 1) ? r : (r >> 7);
        return rb * a.nbc + (c >> 7);
    }
}

// BR, FD: the FP8 block index variant (fp8_block_index); unused by NVFP4 / MXFP8.
template <class T, int FMT, int BR, bool FD>
__global__ void __launch_bounds__(256) k_mx_deq8(DeqArgs a) {
    const float s2 = (FMT == MX_NVFP4) ? __ldg(a.global_scale) : 1.0f;
    const int64_t n_items = a.numel / 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n_items;
         base += stride * DQ_U) {
        uint2 w[DQ_U];
        uint32_t sb[DQ_U];
        float fs[DQ_U];
#pragma unroll
        for (int u = 0; u < DQ_U; ++u) {
            const int64_t it = base + u * stride;
            if (it < n_items) {
                if constexpr (FMT == MX_NVFP4 || FMT == MX_MXFP4) {
                    w[u].x = __ldg(reinterpret_cast<const uint32_t*>(a.codes) + it);
                    sb[u] = __ldg((const uint8_t*)a.scales + (FMT == MX_NVFP4 ? (it >> 1) : (it >> 2)));
                } else {
                    w[u] = __ldg(reinterpret_cast<const uint2*>(a.codes) + it);
                    if constexpr (FMT == MX_MXFP8) {
                        sb[u] = __ldg((const uint8_t*)a.scales + (it >> 2));
                    } else {
                        fs[u] = __ldg((const float*)a.scales + fp8_block_index<BR, FD>(a, it));
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < DQ_U; ++u) {
            const int64_t it = base + u * stride;
            if (it >= n_items) continue;
            float o[8];
            if constexpr (FMT == MX_NVFP4) {
                e2m1x8_mul(w[u].x, f2_bcast(__fmul_rn(e4m3_to_f32(sb[u]), s2)), o);
            } else if constexpr (FMT == MX_MXFP4) {
                e2m1x8_mul(w[u].x, f2_bcast(e8m0_mul(sb[u])), o);
            } else {
                e4m3x8_mul(w[u].x, w[u].y, f2_bcast(FMT == MX_MXFP8 ? e8m0_mul(sb[u]) : fs[u]), o);
            }
            st_vals8<T>((T*)a.y + it * 8, o);
        }
    }
}

// ------------------------------------------------------------ NVFP4 -> FP8
// predequant_to_fp8 (metrale QuantizedWeight): each element's NVFP4 value
// fl(e2m1(code) * fl(dec(sb) * s2)) encoded to E4M3 (round to nearest even,
// saturating). Items of 8 elements: 4 code bytes in, 8 E4M3 bytes out
// (consecutive lanes write consecutive 8 bytes).
__global__ void __launch_bounds__(256) k_nv_predeq8(const uint8_t* __restrict__ codes,
                                                    const uint8_t* __restrict__ scales,
                                                    const float* __restrict__ global_scale,
                                                    int64_t numel, uint8_t* __restrict__ out) {
    const float s2 = __ldg(global_scale);
    const int64_t n_items = numel / 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n_items;
         base += stride * DQ_U) {
        uint32_t w[DQ_U], sb[DQ_U];
#pragma unroll
        for (int u = 0; u < DQ_U; ++u) {
            const int64_t it = base + u * stride;
            if (it < n_items) {
                w[u] = __ldg(reinterpret_cast<const uint32_t*>(codes) + it);
                sb[u] = __ldg(scales + (it >> 1));
            }
        }
#pragma unroll
        for (int u = 0; u < DQ_U; ++u) {
            const int64_t it = base + u * stride;
            if (it >= n_items) continue;
            float o[8];
            e2m1x8_mul(w[u], f2_bcast(__fmul_rn(e4m3_to_f32(sb[u]), s2)), o);
            st8(out + it * 8, e4m3x4(o[0], o[1], o[2], o[3]), e4m3x4(o[4], o[5], o[6], o[7]));
        }
    }
}

// The same on 16-byte code chunks (32 elements, two scale blocks): one
// 16-byte code load and one 2-byte scale load per chunk, two 16-byte stores;
// PQ_U chunks loaded per thread before any is decoded. Needs numel % 32 == 0,
// codes and out 16-byte aligned and scales 2-byte aligned.
constexpr int PQ_U = 4;
__global__ void __launch_bounds__(256) k_nv_predeq16(const uint8_t* __restrict__ codes,
                                                     const uint8_t* __restrict__ scales,
                                                     const float* __restrict__ global_scale,
                                                     int64_t numel, uint8_t* __restrict__ out) {
    const float s2 = __ldg(global_scale);
    const int64_t n_items = numel / 32;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n_items;
         base += stride * PQ_U) {
        U4 w[PQ_U];
        uint32_t sb[PQ_U];
#pragma unroll
        for (int u = 0; u < PQ_U; ++u) {
            const int64_t it = base + u * stride;
            if (it < n_items) {
                w[u] = ld16_stream(codes + it * 16);
                sb[u] = __ldg(reinterpret_cast<const unsigned short*>(scales) + it);
            }
        }
#pragma unroll
        for (int u = 0; u < PQ_U; ++u) {
            const int64_t it = base + u * stride;
            if (it >= n_items) continue;
            const F2 m0 = f2_bcast(__fmul_rn(e4m3_to_f32(sb[u] & 0xFFu), s2));   // block 2 it
            const F2 m1 = f2_bcast(__fmul_rn(e4m3_to_f32(sb[u] >> 8), s2));      // block 2 it + 1
            float o[8];
            U4 r0, r1;
            e2m1x8_mul(w[u].x, m0, o);
            r0.x = e4m3x4(o[0], o[1], o[2], o[3]); r0.y = e4m3x4(o[4], o[5], o[6], o[7]);
            e2m1x8_mul(w[u].y, m0, o);
            r0.z = e4m3x4(o[0], o[1], o[2], o[3]); r0.w = e4m3x4(o[4], o[5], o[6], o[7]);
            e2m1x8_mul(w[u].z, m1, o);
            r1.x = e4m3x4(o[0], o[1], o[2], o[3]); r1.y = e4m3x4(o[4], o[5], o[6], o[7]);
            e2m1x8_mul(w[u].w, m1, o);
            r1.z = e4m3x4(o[0], o[1], o[2], o[3]); r1.w = e4m3x4(o[4], o[5], o[6], o[7]);
            st16(out + it * 32, r0);
            st16(out + it * 32 + 16, r1);
        }
    }
}

// Element-wise fallback (any alignment).
__global__ void __launch_bounds__(256) k_nv_predeq_scalar(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ scales,
                                                          const float* __restrict__ global_scale,
                                                          int64_t numel, uint8_t* __restrict__ out) {
    const float s2 = __ldg(global_scale);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < numel;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t byte = __ldg(codes + i / 2);
        const float2 f = e2m1x2_to_f32(byte);
        const float eff = __fmul_rn(e4m3_to_f32(__ldg(scales + i / 16)), s2);
        out[i] = (uint8_t)e4m3x2(__fmul_rn((i & 1) ? f.y : f.x, eff), 0.0f);
    }
}

// ------------------------------------------------------------ segment copies
// Up to four (src, dst, bytes) copies in one launch (concat_rows): 16-byte
// vectors over the aligned part of each segment, bytes for the rest.
struct CopySeg {
    const uint8_t* src;
    uint8_t* dst;
    int64_t bytes, nvec, vfirst, bfirst;
};
struct CopySegs {
    CopySeg s[4];
    int n;
    int64_t nvec, nbytes;     // vector units, byte units over all segments
};

__global__ void __launch_bounds__(256) k_copy_segs(CopySegs c) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // Four 16-byte vectors per thread and step, all four loads issued before
    // any store, so that one step keeps four times the bytes in flight.
    constexpr int U = 4;
    auto seg_of = [&](int64_t i) {
        int q = 0;
        while (q + 1 < c.n && i >= c.s[q + 1].vfirst) ++q;
        return q;
    };
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < c.nvec; i0 += U * stride) {
        U4 v[U];
        int qs[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            qs[u] = 0;
            if (i < c.nvec) {
                qs[u] = seg_of(i);
                v[u] = ld16_stream(c.s[qs[u]].src + (i - c.s[qs[u]].vfirst) * 16);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < c.nvec) st16(c.s[qs[u]].dst + (i - c.s[qs[u]].vfirst) * 16, v[u]);
        }
    }
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < c.nbytes; i += stride) {
        int q = 0;
        while (q + 1 < c.n && i >= c.s[q + 1].bfirst) ++q;
        const int64_t b = c.s[q].nvec * 16 + (i - c.s[q].bfirst);
        c.s[q].dst[b] = __ldg(c.s[q].src + b);
    }
}

// ------------------------------------------------------------ launchers
static bool al(const void* p, int n) { return ((uintptr_t)p % (uintptr_t)n) == 0; }

static unsigned grid_cap(int64_t need_blocks, int per_sm) {
    int64_t cap = (int64_t)sm_count() * per_sm;
    if (need_blocks < 1) need_blocks = 1;
    return (unsigned)(need_blocks < cap ? need_blocks : cap);
}

// Grid of at most one wave of 256-thread blocks of kernel K; the occupancy
// query runs once per kernel instantiation.
template <auto K>
static unsigned grid_occ_mx(int64_t need_blocks) {
    static const int bps = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, K, 256, 0) != cudaSuccess || n < 1) {
            (void)cudaGetLastError();
            n = 1;
        }
        return n;
    }();
    return grid_cap(need_blocks, bps);
}

template <class T, int FMT>
static cudaError_t launch_mx_quant_t(const MxArgs& a, bool vec, cudaStream_t st) {
    using S = MxShape<T, FMT>;
    if (vec) {
        const int64_t per_warp = (int64_t)S::SEGS * (32 / S::TEAM);
        const int64_t warps = (a.n_seg + per_warp - 1) / per_warp;
        auto k = k_mx_quant<T, FMT>;
        k<<<grid_occ_mx<k_mx_quant<T, FMT>>((warps + 7) / 8), 256, 0, st>>>(a);
    } else {
        k_mx_quant_scalar<T, FMT><<<grid_cap((a.n_seg + 255) / 256, 8), 256, 0, st>>>(a);
    }
    return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_mx_quant_f(DT dt, const MxArgs& a, bool vec, cudaStream_t st) {
    switch (dt) {
        case DT::F32: return launch_mx_quant_t<float, FMT>(a, vec, st);
        case DT::F16: return launch_mx_quant_t<__half, FMT>(a, vec, st);
        case DT::BF16: return launch_mx_quant_t<__nv_bfloat16, FMT>(a, vec, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t mx_quant(DT dt, int fmt, const void* x, int64_t rows, int64_t k, uint8_t* codes,
                     void* scales, const unsigned long long* amax_rec, float* global_scale,
                     int static_global, cudaStream_t st) {
    const int G = fmt == MX_FP8_1x128 ? 128 : (fmt == MX_NVFP4 ? 16 : 32);
    MxArgs a;
    a.x = x; a.n_seg = rows * (k / G); a.codes = codes; a.scales = scales;
    a.amax_rec = amax_rec; a.global_scale = global_scale; a.static_global = static_global;
    if (a.n_seg == 0) return cudaSuccess;
    const cudaError_t pe = mx_quant_pipe(dt, fmt, x, rows, k, codes, scales, amax_rec, global_scale,
                                         static_global, st);
    if (pe != cudaErrorNotSupported) return pe;
    const int VEC = dt == DT::F32 ? 4 : 8;
    const int cb = (fmt == MX_NVFP4 || fmt == MX_MXFP4) ? VEC / 2 : VEC;
    const bool vec = al(x, 16) && al(codes, cb);
    switch (fmt) {
        case MX_FP8_1x128: return launch_mx_quant_f<MX_FP8_1x128>(dt, a, vec, st);
        case MX_MXFP8: return launch_mx_quant_f<MX_MXFP8>(dt, a, vec, st);
        case MX_NVFP4: return launch_mx_quant_f<MX_NVFP4>(dt, a, vec, st);
        case MX_MXFP4: return launch_mx_quant_f<MX_MXFP4>(dt, a, vec, st);
    }
    return cudaErrorInvalidValue;
}

template <class T>
static cudaError_t launch_tile_t(const void* x, int64_t rows, int64_t cols, int br, uint8_t* e,
                                 float* s, cudaStream_t st) {
    constexpr int VEC = Traits<T>::VEC;
    const int64_t nbr = (rows + br - 1) / br, nbc = (cols + 127) / 128;
    const int64_t nb = nbr * nbc;
    if (nb == 0) return cudaSuccess;
    if (nb > 0x7FFFFFFFll) return cudaErrorInvalidValue;
    const bool vec = (cols % VEC == 0) && al(x, 16) && al(e, VEC);
    if (br == 128) {
        if (vec) k_fp8_tile<T, 128, 256, true><<<(unsigned)nb, 256, 0, st>>>((const T*)x, rows, cols, nbc, e, s);
        else k_fp8_tile<T, 128, 256, false><<<(unsigned)nb, 256, 0, st>>>((const T*)x, rows, cols, nbc, e, s);
    } else {
        if (vec) k_fp8_tile<T, 1, 32, true><<<(unsigned)nb, 32, 0, st>>>((const T*)x, rows, cols, nbc, e, s);
        else k_fp8_tile<T, 1, 128, false><<<(unsigned)nb, 128, 0, st>>>((const T*)x, rows, cols, nbc, e, s);
    }
    return cudaGetLastError();
}

cudaError_t fp8_tile_quant(DT dt, const void* x, int64_t rows, int64_t cols, int br, int bc,
                           uint8_t* e4m3, float* scale, cudaStream_t st) {
    if (bc != 128 || (br != 1 && br != 128)) return cudaErrorNotSupported;
    if (br == 128) {
        const cudaError_t pe = fp8_tile_pipe(dt, x, rows, cols, e4m3, scale, st);
        if (pe != cudaErrorNotSupported) return pe;
    }
    switch (dt) {
        case DT::F32: return launch_tile_t<float>(x, rows, cols, br, e4m3, scale, st);
        case DT::F16: return launch_tile_t<__half>(x, rows, cols, br, e4m3, scale, st);
        case DT::BF16: return launch_tile_t<__nv_bfloat16>(x, rows, cols, br, e4m3, scale, st);
        default: return cudaErrorNotSupported;
    }
}

template <class T, int FMT>
static cudaError_t launch_deq_t(const DeqArgs& a, cudaStream_t st) {
    const int cb = (FMT == MX_NVFP4 || FMT == MX_MXFP4) ? 4 : 8;      // code bytes per 8 elements
    const bool vec = (a.k % 8 == 0) && al(a.y, 16) && al(a.codes, cb);
    if (vec) {
        const int64_t blocks = (a.numel / 8 + 256 * DQ_U - 1) / (256 * DQ_U);
        if constexpr (FMT == MX_FP8_1x128) {
            if (a.br < 0) {
                k_mx_deq8<T, FMT, -1, true><<<grid_occ_mx<k_mx_deq8<T, FMT, -1, true>>(blocks), 256, 0, st>>>(a);
            } else if (a.br == 1 && a.k % 128 == 0) {
                k_mx_deq8<T, FMT, 0, true><<<grid_occ_mx<k_mx_deq8<T, FMT, 0, true>>(blocks), 256, 0, st>>>(a);
            } else if (a.br == 1) {
                if (a.use_fd) k_mx_deq8<T, FMT, 1, true><<<grid_occ_mx<k_mx_deq8<T, FMT, 1, true>>(blocks), 256, 0, st>>>(a);
                else k_mx_deq8<T, FMT, 1, false><<<grid_occ_mx<k_mx_deq8<T, FMT, 1, false>>(blocks), 256, 0, st>>>(a);
            } else {
                if (a.use_fd) k_mx_deq8<T, FMT, 128, true><<<grid_occ_mx<k_mx_deq8<T, FMT, 128, true>>(blocks), 256, 0, st>>>(a);
                else k_mx_deq8<T, FMT, 128, false><<<grid_occ_mx<k_mx_deq8<T, FMT, 128, false>>(blocks), 256, 0, st>>>(a);
            }
        } else {
            k_mx_deq8<T, FMT, 0, true><<<grid_occ_mx<k_mx_deq8<T, FMT, 0, true>>(blocks), 256, 0, st>>>(a);
        }
    } else {
        auto k = k_mx_deq<T, FMT, false>;
        k<<<grid_occ_mx<k_mx_deq<T, FMT, false>>((a.numel + 255) / 256), 256, 0, st>>>(a);
    }
    return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_deq_f(DT dt, const DeqArgs& a, cudaStream_t st) {
    switch (dt) {
        case DT::F32: return launch_deq_t<float, FMT>(a, st);
        case DT::F16: return launch_deq_t<__half, FMT>(a, st);
        case DT::BF16: return launch_deq_t<__nv_bfloat16, FMT>(a, st);
        default: return cudaErrorNotSupported;
    }
}

static DeqArgs make_deq(const uint8_t* codes, const void* scales, const float* gs, int64_t rows,
                        int64_t k, void* y) {
    DeqArgs a;
    a.codes = codes; a.scales = scales; a.global_scale = gs;
    a.rows = rows; a.k = k; a.br = 1; a.bc = 128; a.nbc = 1;
    a.numel = rows * k;
    a.use_fd = (a.numel < ((int64_t)1 << 32) && k > 0) ? 1 : 0;
    a.fk = make_fastdiv(a.use_fd ? (uint32_t)k : 1u);
    a.y = y;
    return a;
}

cudaError_t mx_dequant(DT ydt, int fmt, const uint8_t* codes, const void* scales,
                       const float* global_scale, int64_t rows, int64_t k, void* y,
                       cudaStream_t st) {
    DeqArgs a = make_deq(codes, scales, global_scale, rows, k, y);
    if (a.numel == 0) return cudaSuccess;
    if (fmt == MX_NVFP4) return launch_deq_f<MX_NVFP4>(ydt, a, st);
    if (fmt == MX_MXFP8) return launch_deq_f<MX_MXFP8>(ydt, a, st);
    if (fmt == MX_MXFP4) return launch_deq_f<MX_MXFP4>(ydt, a, st);
    return cudaErrorInvalidValue;
}

cudaError_t fp8_block_dequant(DT ydt, const uint8_t* e4m3, const float* scale, int64_t rows,
                              int64_t cols, int br, int bc, void* y, cudaStream_t st) {
    DeqArgs a = make_deq(e4m3, scale, nullptr, rows, cols, y);
    a.br = br; a.bc = bc; a.nbc = (cols + bc - 1) / bc;
    if (a.numel == 0) return cudaSuccess;
    return launch_deq_f<MX_FP8_1x128>(ydt, a, st);
}

cudaError_t fp8_tensor_dequant(DT ydt, const uint8_t* e4m3, const float* scale, int64_t n, void* y,
                               cudaStream_t st) {
    // One row of n elements; a block of one row and n columns (the scalar
    // path's index) or the single-scale index (the vector path).
    DeqArgs a = make_deq(e4m3, scale, nullptr, 1, n, y);
    a.br = (n % 8 == 0) ? -1 : 1;
    a.bc = n > 0 ? n : 1;
    a.nbc = 1;
    if (a.numel == 0) return cudaSuccess;
    return launch_deq_f<MX_FP8_1x128>(ydt, a, st);
}

cudaError_t nvfp4_predequant_fp8(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                                 int64_t rows, int64_t k, uint8_t* out, cudaStream_t st) {
    const int64_t numel = rows * k;
    if (numel == 0) return cudaSuccess;
    if (numel % 32 == 0 && k % 16 == 0 && al(codes, 16) && al(out, 16) && al(scales, 2)) {
        const int64_t blocks = (numel / 32 + 256 * PQ_U - 1) / (256 * PQ_U);
        k_nv_predeq16<<<grid_occ_mx<k_nv_predeq16>(blocks), 256, 0, st>>>(codes, scales, global_scale, numel, out);
    } else if (k % 16 == 0 && al(codes, 4) && al(out, 8)) {
        const int64_t blocks = (numel / 8 + 256 * DQ_U - 1) / (256 * DQ_U);
        k_nv_predeq8<<<grid_occ_mx<k_nv_predeq8>(blocks), 256, 0, st>>>(codes, scales, global_scale, numel, out);
    } else {
        k_nv_predeq_scalar<<<grid_occ_mx<k_nv_predeq_scalar>((numel + 255) / 256), 256, 0, st>>>(
            codes, scales, global_scale, numel, out);
    }
    return cudaGetLastError();
}

cudaError_t copy_segments(const void* const* src, void* const* dst, const int64_t* bytes, int n,
                          cudaStream_t st) {
    CopySegs c{};
    c.n = 0;
    for (int i = 0; i < n && i < 4; ++i) {
        CopySeg g;
        g.src = (const uint8_t*)src[i];
        g.dst = (uint8_t*)dst[i];
        g.bytes = bytes[i];
        const bool vec = al(g.src, 16) && al(g.dst, 16);
        g.nvec = vec ? g.bytes / 16 : 0;
        g.vfirst = c.nvec;
        g.bfirst = c.nbytes;
        c.nvec += g.nvec;
        c.nbytes += g.bytes - g.nvec * 16;
        c.s[c.n++] = g;
    }
    const int64_t work = c.nvec > c.nbytes ? c.nvec : c.nbytes;
    if (work == 0) return cudaSuccess;
    k_copy_segs<<<grid_cap((work + 255) / 256, 8), 256, 0, st>>>(c);
    return cudaGetLastError();
}

}  // namespace bq
