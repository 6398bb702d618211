// Device helpers shared by the bq kernels: element types, 16-byte memory
// access, correctly rounded division, integer-code rounding and the FP8 / FP4
// encoders. sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <type_traits>

namespace bq {

// ---------------------------------------------------------------- launch order
// Programmatic dependent launch (sm_90 and later). A kernel launched with the
// programmatic-serialization attribute (launch_pdl) may start while the
// kernel before it on the stream is still running: pdl_wait() blocks until
// that kernel has completed and its writes are visible (it returns at once in
// a kernel launched the ordinary way), and pdl_trigger() lets the next such
// kernel start once every block of this grid has called it or exited. The
// first kernel of every library call is launched the ordinary way, so a call
// never overlaps the caller's earlier work; a kernel launched with the
// attribute touches nothing an earlier kernel of the same call writes before
// its pdl_wait().
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*k)(KArgs...), unsigned grid, unsigned block, size_t smem,
                              cudaStream_t st, Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, args...);
}

// ---------------------------------------------------------------- elements
// Acc is the arithmetic type: f32 for f32/f16/bf16 storage, f64 for f64.
template <class T> struct Traits;
template <> struct Traits<float>          { using Acc = float;  static constexpr int VEC = 4; };
template <> struct Traits<__half>         { using Acc = float;  static constexpr int VEC = 8; };
template <> struct Traits<__nv_bfloat16>  { using Acc = float;  static constexpr int VEC = 8; };
template <> struct Traits<double>         { using Acc = double; static constexpr int VEC = 2; };

struct alignas(16) U4 { uint32_t x, y, z, w; };

// Read-only 16-byte load through L1 (neighbouring lanes share sectors).
__device__ __forceinline__ U4 ld16_nc(const void* p) {
    U4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
// Streaming 16-byte load: read once, keep it out of L1.
__device__ __forceinline__ U4 ld16_stream(const void* p) {
    U4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st16(void* p, const U4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st8(void* p, uint32_t a, uint32_t b) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(p), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st4(void* p, uint32_t a) {
    asm volatile("st.global.u32 [%0], %1;" :: "l"(p), "r"(a) : "memory");
}

// Unpack one 16-byte vector into VEC arithmetic values (exact widening).
__device__ __forceinline__ void unpack(const U4& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}
__device__ __forceinline__ void unpack_f16x2(uint32_t w, float& lo, float& hi) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    float2 f = __half22float2(h);
    lo = f.x; hi = f.y;
}
template <class T> __device__ __forceinline__ void unpack8(const U4& u, float (&v)[8]);
template <> __device__ __forceinline__ void unpack8<__nv_bfloat16>(const U4& u, float (&v)[8]) {
    unpack_bf16x2(u.x, v[0], v[1]); unpack_bf16x2(u.y, v[2], v[3]);
    unpack_bf16x2(u.z, v[4], v[5]); unpack_bf16x2(u.w, v[6], v[7]);
}
template <> __device__ __forceinline__ void unpack8<__half>(const U4& u, float (&v)[8]) {
    unpack_f16x2(u.x, v[0], v[1]); unpack_f16x2(u.y, v[2], v[3]);
    unpack_f16x2(u.z, v[4], v[5]); unpack_f16x2(u.w, v[6], v[7]);
}
__device__ __forceinline__ void unpack(const U4& u, double (&v)[2]) {
    v[0] = __hiloint2double((int)u.y, (int)u.x);
    v[1] = __hiloint2double((int)u.w, (int)u.z);
}

// Generic: VEC values from one 16-byte vector.
template <class T>
__device__ __forceinline__ void load_vec(const U4& u, typename Traits<T>::Acc (&v)[Traits<T>::VEC]) {
    if constexpr (sizeof(T) == 2) unpack8<T>(u, v); else unpack(u, v);
}

// Scalar element load / store with round-to-nearest-even narrowing.
template <class T> __device__ __forceinline__ typename Traits<T>::Acc ld1(const T* p);
template <> __device__ __forceinline__ float ld1<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ double ld1<double>(const double* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld1<__half>(const __half* p) {
    return __half2float(__ldg(p));
}
template <> __device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p) {
    unsigned short b = __ldg(reinterpret_cast<const unsigned short*>(p));
    return __uint_as_float(((uint32_t)b) << 16);
}

template <class T> __device__ __forceinline__ T to_out(typename Traits<T>::Acc v);
template <> __device__ __forceinline__ float to_out<float>(float v) { return v; }
template <> __device__ __forceinline__ double to_out<double>(double v) { return v; }
template <> __device__ __forceinline__ __half to_out<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Pack VEC arithmetic values into one 16-byte vector of T (RNE narrowing).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <class T>
__device__ __forceinline__ U4 pack_vec(const typename Traits<T>::Acc (&v)[Traits<T>::VEC]) {
    U4 u;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        u.x = pack_bf16x2(v[0], v[1]); u.y = pack_bf16x2(v[2], v[3]);
        u.z = pack_bf16x2(v[4], v[5]); u.w = pack_bf16x2(v[6], v[7]);
    } else if constexpr (std::is_same<T, __half>::value) {
        u.x = pack_f16x2(v[0], v[1]); u.y = pack_f16x2(v[2], v[3]);
        u.z = pack_f16x2(v[4], v[5]); u.w = pack_f16x2(v[6], v[7]);
    } else if constexpr (std::is_same<T, float>::value) {
        u.x = __float_as_uint(v[0]); u.y = __float_as_uint(v[1]);
        u.z = __float_as_uint(v[2]); u.w = __float_as_uint(v[3]);
    } else {
        u.x = (uint32_t)__double2loint(v[0]); u.y = (uint32_t)__double2hiint(v[0]);
        u.z = (uint32_t)__double2loint(v[1]); u.w = (uint32_t)__double2hiint(v[1]);
    }
    return u;
}

// ---------------------------------------------------------------- division
// fl(x / s) for a per-group divisor s, correctly rounded, from the correctly
// rounded reciprocal y = RN(1/s) and two remainder corrections:
//   q0 = RN(x*y); q1 = RN(q0 + RN(x - s*q0)*y)  -> within one ulp of x/s;
//   q2 = RN(q1 + (x - s*q1)*y)                  -> RN(x/s)
// The last step is Markstein's theorem (P. Markstein, IBM J. Res. Dev. 34(1),
// 1990; Muller et al., Handbook of Floating-Point Arithmetic, ch. 4): with y
// within half an ulp of 1/s and q1 within one ulp of x/s, the remainder
// x - s*q1 is exact in an FMA and RN(q1 + r*y) = RN(x/s). The hypotheses
// need no overflow and a remainder above the subnormal range; `fast` holds
// when 2^-64 <= |s| <= 2^64, which covers every quotient that can decide a
// code (|x/s| >= 2^-12 needs |x| >= 2^-76). Outside that range, and for
// x/s that overflow (only possible when x is not bounded by the group range),
// callers use the IEEE division __fdiv_rn.
struct Recip {
    float s, y;
    bool fast;
};
__device__ __forceinline__ Recip make_recip(float s) {
    Recip r;
    r.s = s;
    r.y = __frcp_rn(s);
    const float a = fabsf(s);
    r.fast = (a >= 0x1p-64f) && (a <= 0x1p64f);
    return r;
}
// Correct when r.fast and |x| is bounded by the group range (no overflow).
__device__ __forceinline__ float div_chain(float x, const Recip& r) {
    const float q0 = __fmul_rn(x, r.y);
    const float e0 = __fmaf_rn(-r.s, q0, x);
    const float q1 = __fmaf_rn(e0, r.y, q0);
    const float e1 = __fmaf_rn(-r.s, q1, x);
    return __fmaf_rn(e1, r.y, q1);
}
// IEEE division kept out of line: it is the rare path, and inlining it into
// unrolled loops only costs registers and instruction cache.
static __device__ __noinline__ float div_slow(float x, float s) { return __fdiv_rn(x, s); }
// Any x: falls back to IEEE division when the chain produced a NaN
// (an infinite or overflowing operand); a NaN x stays NaN either way.
__device__ __forceinline__ float div_any(float x, const Recip& r) {
    if (!r.fast) return div_slow(x, r.s);
    float q = div_chain(x, r);
    if (q != q) q = div_slow(x, r.s);
    return q;
}
// Sign of a quotient of zero: x/s keeps the sign of x * s. The chain returns
// +0 for x = -0; encoders that keep the sign of zero restore it here.
__device__ __forceinline__ float with_quotient_sign(float q, float x, float s) {
    return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) |
                           ((__float_as_uint(x) ^ __float_as_uint(s)) & 0x80000000u));
}

// ---------------------------------------------------------------- f32 pairs
// sm_100 issues add / sub / mul / fma on two f32 lanes held in one 64-bit
// register pair (PTX .f32x2); each lane is rounded exactly as the scalar
// instruction rounds it (round-to-nearest-even, subnormals kept). The fast
// per-element paths run their arithmetic on such pairs: the same bits as the
// scalar sequence, half the issue slots.
typedef unsigned long long F2;
__device__ __forceinline__ F2 f2_pack(float lo, float hi) {
    F2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(F2 v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ void f2_split_bits(F2 v, uint32_t& lo, uint32_t& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ F2 f2_bcast(float v) { return f2_pack(v, v); }
__device__ __forceinline__ F2 f2_add(F2 a, F2 b) {
    F2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ F2 f2_sub(F2 a, F2 b) {
    F2 r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ F2 f2_mul(F2 a, F2 b) {
    F2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ F2 f2_fma(F2 a, F2 b, F2 c) {
    F2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
// The two 16-bit floats of one word (low half first), widened exactly.
__device__ __forceinline__ F2 f2_widen_bf16x2(uint32_t w) {
    F2 r;
    asm("{\n\t.reg .b32 lo, hi;\n\t"
        "shl.b32 lo, %1, 16;\n\t"
        "and.b32 hi, %1, 0xFFFF0000;\n\t"
        "mov.b64 %0, {lo, hi};\n\t}"
        : "=l"(r) : "r"(w));
    return r;
}
__device__ __forceinline__ F2 f2_widen_f16x2(uint32_t w) {
    F2 r;
    asm("{\n\t.reg .b16 a, b;\n\t.reg .f32 lo, hi;\n\t"
        "mov.b32 {a, b}, %1;\n\t"
        "cvt.f32.f16 lo, a;\n\t"
        "cvt.f32.f16 hi, b;\n\t"
        "mov.b64 %0, {lo, hi};\n\t}"
        : "=l"(r) : "r"(w));
    return r;
}
// One 16-byte vector as VEC/2 pairs, in element order.
template <class T>
__device__ __forceinline__ void widen_pairs(const U4& u, F2 (&x)[Traits<T>::VEC / 2]) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        x[0] = f2_widen_bf16x2(u.x); x[1] = f2_widen_bf16x2(u.y);
        x[2] = f2_widen_bf16x2(u.z); x[3] = f2_widen_bf16x2(u.w);
    } else if constexpr (std::is_same<T, __half>::value) {
        x[0] = f2_widen_f16x2(u.x); x[1] = f2_widen_f16x2(u.y);
        x[2] = f2_widen_f16x2(u.z); x[3] = f2_widen_f16x2(u.w);
    } else {
        x[0] = f2_pack(__uint_as_float(u.x), __uint_as_float(u.y));
        x[1] = f2_pack(__uint_as_float(u.z), __uint_as_float(u.w));
    }
}
// div_chain on both lanes of a pair: the same five roundings per lane.
struct Recip2 {
    F2 y, ns;   // (RN(1/s), RN(1/s)), (-s, -s)
};
__device__ __forceinline__ F2 div_chain2(F2 x, const Recip2& r) {
    const F2 q0 = f2_mul(x, r.y);
    const F2 e0 = f2_fma(r.ns, q0, x);
    const F2 q1 = f2_fma(e0, r.y, q0);
    const F2 e1 = f2_fma(r.ns, q1, x);
    return f2_fma(e1, r.y, q1);
}
// fl(x / s) on pairs in four roundings, from a two-term reciprocal: with
// y = RN(1/s), the residual e = 1 - s*y is exact in an FMA and
// 1/s = y (1 + e + e^2 + ...), |e| <= 2^-23, so y + ylo, ylo = RN(e * y),
// is 1/s to a relative 2^-45. Then q0 = RN(x*y + RN(x*ylo)) (one FMA) lies
// within 2^-44 |x/s| + half an ulp of x/s, i.e. within one ulp, and one
// remainder correction RN(q0 + (x - s*q0) * y) is RN(x/s) (Markstein's
// theorem, the hypotheses of div_chain's last step; the remainder is exact
// in an FMA). Same domain as div_chain: Recip::fast and no overflow.
struct Recip2T {
    F2 y, ylo, ns;   // RN(1/s), RN((1 - s*y) * y), -s, on both lanes
};
__device__ __forceinline__ Recip2T make_recip2(const Recip& r) {
    Recip2T p;
    const float e = __fmaf_rn(-r.s, r.y, 1.0f);
    p.y = f2_bcast(r.y);
    p.ylo = f2_bcast(__fmul_rn(e, r.y));
    p.ns = f2_bcast(-r.s);
    return p;
}
__device__ __forceinline__ F2 div_chain2(F2 x, const Recip2T& r) {
    const F2 q0 = f2_fma(x, r.y, f2_mul(x, r.ylo));
    const F2 e0 = f2_fma(r.ns, q0, x);
    return f2_fma(e0, r.y, q0);
}

// ---------------------------------------------------------------- int codes
// Rounding v (an exact f32 quotient) to an integer code with nearest-even:
// for |v| <= 2^22, fl(v + 1.5*2^23) has unit spacing, so the addition itself
// rounds v to the nearest integer (ties to even) and round(v) sits in the low
// mantissa bits. The zero-point is added afterwards as an integer, so the
// tie rule applies to round(v) itself, not to round(v) + zp.
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23

struct IntParams {
    float lo, hi;      // code range shifted by the zero-point: qmin - zp, qmax - zp
    int zp;
};
__device__ __forceinline__ IntParams make_int_params(int qmin, int qmax, int zp) {
    IntParams p;
    p.lo = (float)(qmin - zp);
    p.hi = (float)(qmax - zp);
    p.zp = zp;
    return p;
}
// fl(round(clamp(v)) + 1.5*2^23): round(v) clamped to [qmin-zp, qmax-zp], as
// the low mantissa bits of the result. A NaN v clamps to qmin - zp.
__device__ __forceinline__ float rounded_rne(float v, const IntParams& p) {
    v = fminf(fmaxf(v, p.lo), p.hi);            // fmaxf(NaN, lo) = lo
    return __fadd_rn(v, kMagic);
}
// Ties away from zero.
__device__ __forceinline__ float rounded_rhaz(float v, const IntParams& p) {
    v = fminf(fmaxf(v, p.lo), p.hi);
    const float t = truncf(v);
    const float d = __fsub_rn(v, t);             // exact
    const float k = (fabsf(d) >= 0.5f) ? __fadd_rn(t, copysignf(1.0f, v)) : t;
    return __fadd_rn(k, kMagic);
}
template <bool RHAZ>
__device__ __forceinline__ float rounded_of(float v, const IntParams& p) {
    if constexpr (RHAZ) return rounded_rhaz(v, p); else return rounded_rne(v, p);
}
// Low byte = the code clamp(round(v) + zp, qmin, qmax).
__device__ __forceinline__ uint32_t code_from_rounded(float t, int zp) {
    return __float_as_uint(t) + (uint32_t)zp;
}
// The dequantized value fl((q - zp) * s) from the rounded form.
__device__ __forceinline__ float dequant_from_rounded(float t, float s) {
    return __fmul_rn(__fsub_rn(t, kMagic), s);
}
// round(v) as a float, for the STE mask; v is clamped to [lo-1, hi+1] first
// so that the result stays exact (a NaN v gives lo - 1: masked).
template <bool RHAZ>
__device__ __forceinline__ float round_for_mask(float v, const IntParams& p) {
    v = fminf(fmaxf(v, p.lo - 1.0f), p.hi + 1.0f);
    if constexpr (RHAZ) {
        const float t = truncf(v);
        const float d = __fsub_rn(v, t);
        return (fabsf(d) >= 0.5f) ? __fadd_rn(t, copysignf(1.0f, v)) : t;
    } else {
        return __fsub_rn(__fadd_rn(v, kMagic), kMagic);
    }
}

// f64 versions (f64 inputs): IEEE f64 division and rounding.
__device__ __forceinline__ double round_rne_d(double v) { return rint(v); }
__device__ __forceinline__ double round_rhaz_d(double v) { return round(v); }

// Pack four low bytes into one word: byte i of the result = low byte of w[i].
__device__ __forceinline__ uint32_t pack4_lowbytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d);

// ---------------------------------------------------------------- code storage
// Integer codes are one byte each, or (packed) two 4-bit codes per byte with
// element 2j in the low nibble of byte j. Vectors of codes always start at an
// even element, so a packed vector covers whole bytes.
__device__ __forceinline__ uint8_t* code_ptr(uint8_t* q, int64_t e, int packed) {
    return q + (packed ? (e >> 1) : e);
}
__device__ __forceinline__ const uint8_t* code_ptr(const uint8_t* q, int64_t e, int packed) {
    return q + (packed ? (e >> 1) : e);
}
// Low nibbles of the four bytes of w as two bytes (bytes 0, 1 of the result).
__device__ __forceinline__ uint32_t nib_pack4(uint32_t w) {
    uint32_t t = w & 0x0F0F0F0Fu;
    t |= t >> 4;                                   // bytes 0 and 2 hold the pairs
    return __byte_perm(t, 0u, 0x4420);
}
// Bytes 0, 1 of x as four 4-bit codes widened to bytes (sign-extended when
// q_signed).
__device__ __forceinline__ uint32_t nib_spread(uint32_t x, int q_signed) {
    const uint32_t y = __byte_perm(x, 0u, 0x1100);
    uint32_t w = (y & 0x000F000Fu) | ((y >> 4) & 0x0F000F00u);
    if (q_signed) w = __vsub4(w ^ 0x08080808u, 0x08080808u);
    return w;
}
template <int W>
__device__ __forceinline__ void st_codes(uint8_t* q, const uint32_t (&c)[W], int packed);
template <int W>
__device__ __forceinline__ void ld_codes(const uint8_t* q, int packed, int q_signed,
                                         uint32_t (&w)[(W + 3) / 4]);

__device__ __forceinline__ uint32_t pack4_lowbytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    const uint32_t ab = __byte_perm(a, b, 0x0040);   // [a0, b0, a0, a0]
    const uint32_t cd = __byte_perm(c, d, 0x0040);   // [c0, d0, ...]
    return __byte_perm(ab, cd, 0x5410);              // [a0, b0, c0, d0]
}

// W codes (the low bytes of c[]) at q (from code_ptr): W bytes, or W/2 bytes
// of two 4-bit codes.
template <int W>
__device__ __forceinline__ void st_codes(uint8_t* q, const uint32_t (&c)[W], int packed) {
    if constexpr (W == 8) {
        const uint32_t lo = pack4_lowbytes(c[0], c[1], c[2], c[3]);
        const uint32_t hi = pack4_lowbytes(c[4], c[5], c[6], c[7]);
        if (packed) st4(q, nib_pack4(lo) | (nib_pack4(hi) << 16));
        else st8(q, lo, hi);
    } else if constexpr (W == 4) {
        const uint32_t w = pack4_lowbytes(c[0], c[1], c[2], c[3]);
        if (packed) *reinterpret_cast<unsigned short*>(q) = (unsigned short)nib_pack4(w);
        else st4(q, w);
    } else if constexpr (W == 2) {
        if (packed) {
            q[0] = (uint8_t)((c[0] & 0xFu) | ((c[1] & 0xFu) << 4));
        } else {
            q[0] = (uint8_t)c[0];
            q[1] = (uint8_t)c[1];
        }
    } else {
        q[0] = (uint8_t)c[0];     // single codes: never packed (the callers' shapes rule it out)
    }
}
// W codes at q (from code_ptr) as bytes, four per word; packed 4-bit codes
// are widened to bytes (sign-extended when q_signed).
template <int W>
__device__ __forceinline__ void ld_codes(const uint8_t* q, int packed, int q_signed,
                                         uint32_t (&w)[(W + 3) / 4]) {
    if (packed) {
        if constexpr (W == 8) {
            const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(q));
            w[0] = nib_spread(v & 0xFFFFu, q_signed);
            w[1] = nib_spread(v >> 16, q_signed);
        } else if constexpr (W == 4) {
            w[0] = nib_spread(__ldg(reinterpret_cast<const unsigned short*>(q)), q_signed);
        } else if constexpr (W == 2) {
            w[0] = nib_spread(__ldg(q), q_signed);
        } else {
            w[0] = __ldg(q);
        }
        return;
    }
    if constexpr (W == 8) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(q));
        w[0] = v.x; w[1] = v.y;
    } else if constexpr (W == 4) {
        w[0] = __ldg(reinterpret_cast<const uint32_t*>(q));
    } else if constexpr (W == 2) {
        w[0] = __ldg(reinterpret_cast<const unsigned short*>(q));
    } else {
        w[0] = __ldg(q);
    }
}

// ---------------------------------------------------------------- FP8 / FP4
// E4M3 (OCP FP8, max 448, no infinities), round to nearest even, saturating.
// Two values per instruction; `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    return e4m3x2(a, b) | (e4m3x2(c, d) << 16);
}
// E2M1 (OCP FP4), round to nearest even, saturating to +-6: eight values
// into one word, value i in nibble i (low nibble first). For NaN-free
// inputs only: the conversion instruction gives a NaN the code of +6.
__device__ __forceinline__ uint32_t e2m1x8_finite(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}
// E2M1 of any f32: E2M1 has no NaN, so a NaN of either sign encodes as +0
// (code 0); every other value as e2m1x8_finite.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = isnan(v[i]) ? 0.0f : v[i];
    return e2m1x8_finite(t);
}
// Decode two E4M3 bytes (low byte first) to f32 exactly (via f16, which
// holds every E4M3 value).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two));
    __half2 hh = *reinterpret_cast<__half2*>(&h);
    return __half22float2(hh);
}
// Decode one byte of two E2M1 codes (low nibble first) to f32.
__device__ __forceinline__ float2 e2m1x2_to_f32(uint32_t byte) {
    uint32_t h;
    asm("{\n\t.reg .b8 lo, hi;\n\t"
        "mov.b16 {lo, hi}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, lo;\n\t}"
        : "=r"(h) : "h"((uint16_t)byte));
    __half2 hh = *reinterpret_cast<__half2*>(&h);
    return __half22float2(hh);
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) { return e4m3x2_to_f32(byte & 0xFF).x; }

// 2^e as f32 for e in [-149, 127], exact.
__device__ __forceinline__ float exp2i(int e) {
    return (e >= -126) ? __uint_as_float((uint32_t)(e + 127) << 23)
                       : __uint_as_float(1u << (e + 149));
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max(float v, int width = 32) {
    for (int o = width / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o, width));
    return v;
}
__device__ __forceinline__ double warp_max(double v, int width = 32) {
    for (int o = width / 2; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o, width));
    return v;
}

// Range record bits: IEEE bits of a non-negative value, zero-extended.
__device__ __forceinline__ unsigned long long range_bits(float v) {
    return (unsigned long long)__float_as_uint(v);
}
__device__ __forceinline__ unsigned long long range_bits(double v) {
    return (unsigned long long)__double_as_longlong(v);
}
__device__ __forceinline__ void range_from_bits(unsigned long long b, float& v) {
    v = __uint_as_float((uint32_t)b);
}
__device__ __forceinline__ void range_from_bits(unsigned long long b, double& v) {
    v = __longlong_as_double((long long)b);
}

// ---------------------------------------------------------------- fast divide
// Unsigned 32-bit division by a runtime-invariant d (Granlund & Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, §4):
// with l = ceil(log2 d) and m = floor(2^32 * (2^l - d) / d) + 1,
// n / d = (t + ((n - t) >> 1)) >> (l - 1) where t = mulhi(m, n), for l >= 1.
struct FastDiv {
    uint32_t d, m, l;
};
inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d) ++l;
    f.l = l;
    f.m = (uint32_t)(((1ull << 32) * ((1ull << l) - d)) / d + 1);
    return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
    if (f.l == 0) return n;                      // d == 1
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> 1)) >> (f.l - 1);
}

}  // namespace bq
