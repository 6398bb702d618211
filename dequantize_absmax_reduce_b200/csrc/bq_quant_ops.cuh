// Per-group arithmetic shared by the quantize kernels: scale / zero-point
// derivation of the integer formats, the MXFP8 shared exponent, and the code
// emitters for one 16-byte vector of values.
#pragma once

#include "bq_device.cuh"
#include "bq_internal.h"

namespace bq {

// ------------------------------------------------------------ group params
struct GroupF { float s; int zp; };
struct GroupD { float s; int zp; };

// Scale and zero-point from a group's range (f32 arithmetic). Symmetric:
// s = fl(amax / qmax). Asymmetric: s = fl(fl(max' - min') / (qmax - qmin)),
// zp = clamp(qmin - round(fl(min' / s)), qmin, qmax). 0 -> 1.
__device__ __forceinline__ GroupF derive_f(float hi, float nlo, const IntCfg& c) {
    GroupF g;
    if (c.symmetric) {
        float s = __fdiv_rn(fmaxf(hi, nlo), (float)c.qmax);
        if (s == 0.0f) s = 1.0f;
        g.s = s;
        g.zp = 0;
    } else {
        const float span = __fadd_rn(hi, nlo);
        float s = __fdiv_rn(span, (float)(c.qmax - c.qmin));
        if (s == 0.0f) s = 1.0f;
        const float m = __fdiv_rn(-nlo, s);
        const float r = c.rhaz ? roundf(m) : rintf(m);
        float z = __fsub_rn((float)c.qmin, r);
        z = fminf(fmaxf(z, (float)c.qmin), (float)c.qmax);   // NaN -> qmin
        g.s = s;
        g.zp = (int)z;
    }
    return g;
}
// Same in f64 for f64 inputs; the stored scale is still f32.
__device__ __forceinline__ GroupD derive_d(double hi, double nlo, const IntCfg& c) {
    GroupD g;
    if (c.symmetric) {
        float s = __double2float_rn(fmax(hi, nlo) / (double)c.qmax);
        if (s == 0.0f) s = 1.0f;
        g.s = s;
        g.zp = 0;
    } else {
        const double span = hi + nlo;
        float s = __double2float_rn(span / (double)(c.qmax - c.qmin));
        if (s == 0.0f) s = 1.0f;
        const double m = -nlo / (double)s;
        const double r = c.rhaz ? round(m) : rint(m);
        double z = (double)c.qmin - r;
        z = fmin(fmax(z, (double)c.qmin), (double)c.qmax);
        g.s = s;
        g.zp = (int)z;
    }
    return g;
}

__device__ __forceinline__ int load_zp(const void* zp, int64_t g, int q_signed) {
    if (!zp) return 0;
    const uint8_t b = __ldg((const uint8_t*)zp + g);
    return q_signed ? (int)(int8_t)b : (int)b;
}


// Group sizes of the microscaled formats.
template <int FMT> struct MxG;
template <> struct MxG<MX_FP8_1x128> { static constexpr int G = 128; };
template <> struct MxG<MX_MXFP8> { static constexpr int G = 32; };
template <> struct MxG<MX_NVFP4> { static constexpr int G = 16; };
template <> struct MxG<MX_MXFP4> { static constexpr int G = 32; };


__device__ __forceinline__ void st2(void* p, uint32_t a) {
    asm volatile("st.global.u16 [%0], %1;" :: "l"(p), "h"((uint16_t)a) : "memory");
}

// MX shared exponent: E = clamp(floor(log2 a) - emax, -127, 127), emax the
// largest exponent of the element format (8 for E4M3 / MXFP8, 2 for E2M1 /
// MXFP4), from the bits of a >= 0 (a subnormal a counts its leading zeros;
// infinity is 2^128; a = 0 gives -127).
__device__ __forceinline__ int mx_exponent(float a, int emax = 8) {
    const uint32_t b = __float_as_uint(a);
    const int ex = (int)(b >> 23);
    int fl2;
    if (ex == 0) {
        const uint32_t m = b & 0x7FFFFFu;
        fl2 = (m == 0) ? -1000 : (31 - __clz((int)m)) - 149;
    } else if (ex == 255) {
        fl2 = 128;
    } else {
        fl2 = ex - 127;
    }
    return min(max(fl2 - emax, -127), 127);
}


// Codes of one 16-byte vector (v: its VEC values) written at dst.
template <class T, int FMT, bool FAST>
__device__ __forceinline__ void mx_emit(const float* v, const Recip& R, float mul, bool zero,
                                        uint8_t* dst) {
    constexpr int VEC = Traits<T>::VEC;
    float t[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        if constexpr (FMT == MX_MXFP8 || FMT == MX_MXFP4) {
            t[i] = __fmul_rn(v[i], mul);
        } else {
            const float d = FAST ? div_chain(v[i], R) : div_any(v[i], R);
            t[i] = with_quotient_sign(d, v[i], R.s);
        }
    }
    if constexpr (FMT == MX_NVFP4 || FMT == MX_MXFP4) {
        if constexpr (VEC == 8) {
            const float (&t8)[8] = *reinterpret_cast<const float(*)[8]>(t);
            st4(dst, zero ? 0u : e2m1x8(t8));
        } else {
            float t8[8] = {t[0], t[1], t[2], t[3], 0.f, 0.f, 0.f, 0.f};
            st2(dst, zero ? 0u : (e2m1x8(t8) & 0xFFFFu));
        }
    } else {
        if constexpr (VEC == 8) {
            st8(dst, e4m3x4(t[0], t[1], t[2], t[3]), e4m3x4(t[4], t[5], t[6], t[7]));
        } else {
            st4(dst, e4m3x4(t[0], t[1], t[2], t[3]));
        }
    }
}


// ------------------------------------------------------------ fast emitters
// Per-vector encoders on f32 pairs (one .f32x2 instruction per two values).
// The caller guarantees, for the whole group: a positive scale in the range
// where the division chain is exact (Recip::fast), no NaN among the group's
// values (hence none among the quotients: |x| <= the group's finite range),
// and, for integer codes, that no clamp can bind. Under those conditions each
// emitter writes the same bits as the general one.

// Integer codes (QUANT: the low byte of magic + k + zp) or fake-quantized
// values (FAKE: fl(k * s)), k = round-half-even(fl(x / s)).
template <class T, int OP, bool ASYM, class R2T>
__device__ __forceinline__ void emit_int_fast(const U4& raw, const R2T& R2, F2 magic2, F2 zp2,
                                              F2 s2, uint8_t* q, int packed, T* y) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int NP = VEC / 2;
    F2 x[NP];
    widen_pairs<T>(raw, x);
    if constexpr (OP == OP_QUANT) {
        uint32_t c[VEC];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            F2 t = f2_add(div_chain2(x[p], R2), magic2);
            if (ASYM) t = f2_add(t, zp2);            // exact: both integers in the unit-spaced range
            f2_split_bits(t, c[2 * p], c[2 * p + 1]);
        }
        st_codes<VEC>(q, c, packed);
    } else {
        float o[VEC];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const F2 t = f2_add(div_chain2(x[p], R2), magic2);
            f2_split(f2_mul(f2_sub(t, magic2), s2), o[2 * p], o[2 * p + 1]);
        }
        st16(y, pack_vec<T>(o));
    }
}

// Sign bits of a vector's values, one per byte (bit 7 of byte i = sign of
// value i) for the first four values (HALF = 0) or the next four (HALF = 1).
template <class T, int HALF>
__device__ __forceinline__ uint32_t sign_bytes(const U4& raw) {
    if constexpr (sizeof(T) == 2) {
        return (HALF == 0 ? __byte_perm(raw.x, raw.y, 0x7531) : __byte_perm(raw.z, raw.w, 0x7531)) &
               0x80808080u;
    } else {
        return __byte_perm(__byte_perm(raw.x, raw.y, 0x0073), __byte_perm(raw.z, raw.w, 0x0073), 0x5410) &
               0x80808080u;
    }
}

// E4M3 codes of fl(x / s). The chain gives +0 for a zero quotient of a
// negative x; the sign bit of x, OR-ed into each byte afterwards, restores
// -0 there and changes nothing else (non-zero codes already carry it, and no
// value is NaN).
// The codes of one vector as words (VEC / 4 of them: byte i = value i).
template <class T, class R2T>
__device__ __forceinline__ uint2 fp8_words_fast(const U4& raw, const R2T& R2) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int NP = VEC / 2;
    F2 x[NP];
    widen_pairs<T>(raw, x);
    float t[VEC];
#pragma unroll
    for (int p = 0; p < NP; ++p) f2_split(div_chain2(x[p], R2), t[2 * p], t[2 * p + 1]);
    uint2 w;
    w.x = e4m3x4(t[0], t[1], t[2], t[3]) | sign_bytes<T, 0>(raw);
    if constexpr (VEC == 8) w.y = e4m3x4(t[4], t[5], t[6], t[7]) | sign_bytes<T, 1>(raw);
    else w.y = 0u;
    return w;
}
template <class T, class R2T>
__device__ __forceinline__ void emit_fp8_fast(const U4& raw, const R2T& R2, uint8_t* dst) {
    const uint2 w = fp8_words_fast<T>(raw, R2);
    if constexpr (Traits<T>::VEC == 8) st8(dst, w.x, w.y);
    else st4(dst, w.x);
}
// E4M3 codes of fl(x / s) for any values and scale (the general encoder of
// the FP8 block formats: IEEE division where the chain cannot be used, the
// sign of a zero quotient restored), eight values into two words.
template <bool FAST>
__device__ __forceinline__ uint2 fp8_words_general8(const float (&v)[8], const Recip& R) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float d = FAST ? div_chain(v[i], R) : div_any(v[i], R);
        t[i] = with_quotient_sign(d, v[i], R.s);
    }
    return make_uint2(e4m3x4(t[0], t[1], t[2], t[3]), e4m3x4(t[4], t[5], t[6], t[7]));
}

// E2M1 codes of fl(x / s), the sign of each quotient taken from x (no NaN
// among the values: the caller's guarantee above).
template <class T, class R2T>
__device__ __forceinline__ void emit_nv_fast(const U4& raw, const R2T& R2, uint8_t* dst) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int NP = VEC / 2;
    F2 x[NP];
    widen_pairs<T>(raw, x);
    float t[8];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        uint32_t q0, q1, x0, x1;
        f2_split_bits(div_chain2(x[p], R2), q0, q1);
        f2_split_bits(x[p], x0, x1);
        t[2 * p] = __uint_as_float((q0 & 0x7FFFFFFFu) | (x0 & 0x80000000u));
        t[2 * p + 1] = __uint_as_float((q1 & 0x7FFFFFFFu) | (x1 & 0x80000000u));
    }
    if constexpr (VEC == 8) {
        st4(dst, e2m1x8_finite(t));
    } else {
        t[4] = t[5] = t[6] = t[7] = 0.0f;
        st2(dst, e2m1x8_finite(t) & 0xFFFFu);
    }
}

// MXFP8 codes E4M3(fl(x * 2^-E)): a product, exact for every input (NaN and
// infinities included), so it needs no guard.
template <class T>
__device__ __forceinline__ void emit_mx_fast(const U4& raw, F2 mul2, uint8_t* dst) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int NP = VEC / 2;
    F2 x[NP];
    widen_pairs<T>(raw, x);
    float t[VEC];
#pragma unroll
    for (int p = 0; p < NP; ++p) f2_split(f2_mul(x[p], mul2), t[2 * p], t[2 * p + 1]);
    if constexpr (VEC == 8) {
        st8(dst, e4m3x4(t[0], t[1], t[2], t[3]), e4m3x4(t[4], t[5], t[6], t[7]));
    } else {
        st4(dst, e4m3x4(t[0], t[1], t[2], t[3]));
    }
}

// MXFP4 codes E2M1(fl(x * 2^-E)): a product (exact, sign kept for zeros and
// underflows). The caller guarantees no NaN among the values (a NaN takes
// the general encoder, which gives it code 0).
template <class T>
__device__ __forceinline__ void emit_mx4_fast(const U4& raw, F2 mul2, uint8_t* dst) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int NP = VEC / 2;
    F2 x[NP];
    widen_pairs<T>(raw, x);
    float t[8];
#pragma unroll
    for (int p = 0; p < NP; ++p) f2_split(f2_mul(x[p], mul2), t[2 * p], t[2 * p + 1]);
    if constexpr (VEC == 8) {
        st4(dst, e2m1x8_finite(t));
    } else {
        t[4] = t[5] = t[6] = t[7] = 0.0f;
        st2(dst, e2m1x8_finite(t) & 0xFFFFu);
    }
}

// Integer codes (QUANT) or fake-quantized values (FAKE) of one vector of
// VEC values. SYM_DYN: symmetric scale derived from this group's own range.
// When that scale is also a normal number (FAST: 2^-64 <= s <= 2^64) it is
// within 2^-24 of amax/qmax, so |x/s| <= qmax (1 + 2^-23) rounds to at most
// qmax and only the lower clamp (which also takes a NaN to qmin) can bind.
template <class T, int OP, bool FAST, bool SYM_DYN>
__device__ __forceinline__ void emit_int(const float* v, const Recip& R, const IntParams& ip,
                                         uint8_t* q, int packed, T* y) {
    constexpr int VEC = Traits<T>::VEC;
    float t[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        const float qv = FAST ? div_chain(v[i], R) : div_slow(v[i], R.s);
        if constexpr (SYM_DYN && FAST) t[i] = __fadd_rn(fmaxf(qv, ip.lo), kMagic);
        else t[i] = rounded_rne(qv, ip);
    }
    if constexpr (OP == OP_QUANT) {
        uint32_t cw[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) cw[i] = code_from_rounded(t[i], SYM_DYN ? 0 : ip.zp);
        st_codes<VEC>(q, cw, packed);
    } else {
        float o[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) o[i] = dequant_from_rounded(t[i], R.s);
        st16(y, pack_vec<T>(o));
    }
}

}  // namespace bq
