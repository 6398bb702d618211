// Range reductions of 16-byte vectors shared by the pipelined quantizers and
// the GEMM prologue: packed two-lane max / min for 16-bit types, with or
// without NaN propagation, folded by a reduction tree.
#pragma once

#include <type_traits>

#include "bq_device.cuh"

namespace bq {

// Range of one 16-byte vector, accumulated without widening: for 16-bit types
// two lanes per instruction (max.xorsign.abs keeps the larger magnitude), for
// f32 one. PROP = true propagates a NaN into the accumulator (to detect one);
// PROP = false skips NaN operands (the range the formats define).
template <class T, bool ABS, bool PROP>
__device__ __forceinline__ void range_acc(const U4& r, uint32_t& ph, uint32_t& pl, float& hi,
                                          float& nlo) {
    if constexpr (sizeof(T) == 2) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                if (ABS) {
                    if (PROP) asm("max.NaN.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                    else asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                } else if (PROP) {
                    asm("max.NaN.bf16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                    asm("min.NaN.bf16x2 %0, %0, %1;" : "+r"(pl) : "r"(w[i]));
                } else {
                    asm("max.bf16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                    asm("min.bf16x2 %0, %0, %1;" : "+r"(pl) : "r"(w[i]));
                }
            } else {
                if (ABS) {
                    if (PROP) asm("max.NaN.xorsign.abs.f16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                    else asm("max.xorsign.abs.f16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                } else if (PROP) {
                    asm("max.NaN.f16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                    asm("min.NaN.f16x2 %0, %0, %1;" : "+r"(pl) : "r"(w[i]));
                } else {
                    asm("max.f16x2 %0, %0, %1;" : "+r"(ph) : "r"(w[i]));
                    asm("min.f16x2 %0, %0, %1;" : "+r"(pl) : "r"(w[i]));
                }
            }
        }
    } else {
        const float v[4] = {__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z),
                            __uint_as_float(r.w)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (PROP) {
                if (ABS) {
                    asm("max.NaN.f32 %0, %0, %1;" : "+f"(hi) : "f"(fabsf(v[i])));
                } else {
                    asm("max.NaN.f32 %0, %0, %1;" : "+f"(hi) : "f"(v[i]));
                    asm("max.NaN.f32 %0, %0, %1;" : "+f"(nlo) : "f"(-v[i]));
                }
            } else if (ABS) {
                hi = fmaxf(hi, fabsf(v[i]));
            } else {
                hi = fmaxf(hi, v[i]);
                nlo = fmaxf(nlo, -v[i]);
            }
        }
    }
}
// Two-lane 16-bit range steps: the larger magnitude (ABS, sign meaningless),
// or max / min; PROP propagates a NaN operand instead of skipping it.
template <class T, bool ABS, bool PROP>
__device__ __forceinline__ uint32_t pk_hi(uint32_t a, uint32_t b) {
    uint32_t r;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (ABS && PROP) asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else if (ABS) asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else if (PROP) asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    } else {
        if (ABS && PROP) asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else if (ABS) asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else if (PROP) asm("max.NaN.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    }
    return r;
}
template <class T, bool PROP>
__device__ __forceinline__ uint32_t pk_lo(uint32_t a, uint32_t b) {
    uint32_t r;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (PROP) asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    } else {
        if (PROP) asm("min.NaN.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else asm("min.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    }
    return r;
}
template <bool PROP>
__device__ __forceinline__ float f_hi(float a, float b) {
    if constexpr (PROP) {
        float r;
        asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
        return r;
    } else {
        return fmaxf(a, b);
    }
}
// Range of N 16-byte vectors folded into the accumulators of range_acc by a
// reduction tree: depth 2 + ceil(log2 N) instead of a serial chain of 4N
// dependent operations. Same result as N calls of range_acc.
template <class T, bool ABS, bool PROP, int N>
__device__ __forceinline__ void range_tree(const U4* r, uint32_t& ph, uint32_t& pl, float& hi,
                                           float& nlo) {
    if constexpr (sizeof(T) == 2) {
        uint32_t h[N], l[N];
#pragma unroll
        for (int j = 0; j < N; ++j) {
            h[j] = pk_hi<T, ABS, PROP>(pk_hi<T, ABS, PROP>(r[j].x, r[j].y), pk_hi<T, ABS, PROP>(r[j].z, r[j].w));
            if (!ABS) l[j] = pk_lo<T, PROP>(pk_lo<T, PROP>(r[j].x, r[j].y), pk_lo<T, PROP>(r[j].z, r[j].w));
        }
#pragma unroll
        for (int st = 1; st < N; st *= 2)
#pragma unroll
            for (int i = 0; i + st < N; i += 2 * st) {
                h[i] = pk_hi<T, ABS, PROP>(h[i], h[i + st]);
                if (!ABS) l[i] = pk_lo<T, PROP>(l[i], l[i + st]);
            }
        ph = pk_hi<T, ABS, PROP>(ph, h[0]);
        if (!ABS) pl = pk_lo<T, PROP>(pl, l[0]);
    } else {
        float h[N], l[N];
#pragma unroll
        for (int j = 0; j < N; ++j) {
            const float a = __uint_as_float(r[j].x), b = __uint_as_float(r[j].y);
            const float c = __uint_as_float(r[j].z), d = __uint_as_float(r[j].w);
            if (ABS) {
                h[j] = f_hi<PROP>(f_hi<PROP>(fabsf(a), fabsf(b)), f_hi<PROP>(fabsf(c), fabsf(d)));
            } else {
                h[j] = f_hi<PROP>(f_hi<PROP>(a, b), f_hi<PROP>(c, d));
                l[j] = f_hi<PROP>(f_hi<PROP>(-a, -b), f_hi<PROP>(-c, -d));
            }
        }
#pragma unroll
        for (int st = 1; st < N; st *= 2)
#pragma unroll
            for (int i = 0; i + st < N; i += 2 * st) {
                h[i] = f_hi<PROP>(h[i], h[i + st]);
                if (!ABS) l[i] = f_hi<PROP>(l[i], l[i + st]);
            }
        hi = f_hi<PROP>(hi, h[0]);
        if (!ABS) nlo = f_hi<PROP>(nlo, l[0]);
    }
}
// Packed accumulators -> (max(0, max x), max(0, -min x)) or (amax, 0).
template <class T, bool ABS>
__device__ __forceinline__ void range_finish(uint32_t ph, uint32_t pl, float& hi, float& nlo) {
    if constexpr (sizeof(T) == 2) {
        float h0, h1, l0, l1;
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
            unpack_bf16x2(ph, h0, h1);
            unpack_bf16x2(pl, l0, l1);
        } else {
            unpack_f16x2(ph, h0, h1);
            unpack_f16x2(pl, l0, l1);
        }
        if (ABS) {
            hi = fmaxf(fabsf(h0), fabsf(h1));
            nlo = 0.0f;
        } else {
            hi = fmaxf(fmaxf(h0, h1), 0.0f);
            nlo = fmaxf(fmaxf(-l0, -l1), 0.0f);
        }
    }
}
// As range_finish after a NaN-propagating accumulation; true if a NaN was met
// (then hi / nlo are not the range).
template <class T, bool ABS>
__device__ __forceinline__ bool range_finish_nan(uint32_t ph, uint32_t pl, float& hi, float& nlo) {
    if constexpr (sizeof(T) == 2) {
        // A 16-bit NaN: exponent all ones and a non-zero mantissa.
        constexpr uint32_t EXP = std::is_same<T, __nv_bfloat16>::value ? 0x7F80u : 0x7C00u;
        const uint32_t a0 = ph & 0x7FFFu, a1 = (ph >> 16) & 0x7FFFu;
        bool nan = a0 > EXP || a1 > EXP;
        if (!ABS) {
            const uint32_t b0 = pl & 0x7FFFu, b1 = (pl >> 16) & 0x7FFFu;
            nan = nan || b0 > EXP || b1 > EXP;
        }
        range_finish<T, ABS>(ph, pl, hi, nlo);
        return nan;
    } else {
        return (hi != hi) || (nlo != nlo);
    }
}

}  // namespace bq
