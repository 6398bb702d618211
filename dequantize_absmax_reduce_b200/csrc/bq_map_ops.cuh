// Element-wise quantize-family arithmetic with per-group parameters, shared by
// the element kernels of bq_int.cu and the pipelined ones of bq_pipe.cu.
#pragma once

#include <type_traits>

#include "bq_quant_ops.cuh"

namespace bq {

// ------------------------------------------------------------ element-wise
struct MapArgs {
    const void* a;      // x, q or dy
    const void* b;      // dy (backwards)
    int64_t numel, G, n_seg;
    FastDiv fd;         // divide by G when numel < 2^32
    int use_fd;
    IntCfg cfg;
    const float* scale_in;
    const void* zp_in;
    const unsigned long long* ranges;
    float* scale_out;
    uint8_t* zp_out;
    void* out;
};

// Per-group state cached by a thread while it walks its elements.
// x_lo / x_hi: the STE mask 1[qmin < round(fl(x/s)) + zp < qmax] as the input
// interval x_lo <= x <= x_hi (exact, see mask_thresholds); valid when mfast.
struct GState {
    int64_t seg;
    float s;
    int zp;
    Recip R;
    IntParams ip;
    float x_lo, x_hi;
    bool mfast;         // x_lo / x_hi hold the mask
    bool fast;          // mfast and a fast-range scale: branch-free backward path
};

// fl(x/s) for a fast-range s and |x| below 2^100 (no overflow in the chain).
__device__ __forceinline__ float quot(float x, const Recip& R) { return div_chain(x, R); }

// The STE mask as an interval of x. For s > 0, fl(x/s) is non-decreasing in
// x, so {x : round(fl(x/s)) > lo} = {x : fl(x/s) >= a'} is [x_lo, +inf) and
// {x : round(fl(x/s)) < hi} = (-inf, x_hi]; a' (b') is the half-integer
// lo + 1/2 (hi - 1/2) or its neighbour one ulp inward, by the tie rule. Each
// threshold starts at RN(a' s) and moves one ulp at a time while the exact
// quotient says it should (a handful of steps at most). Returns false when
// the scale or the thresholds fall outside the range where this holds; the
// caller then divides per element.
template <bool RHAZ>
__device__ __forceinline__ bool mask_thresholds(const Recip& R, const IntParams& ip, float* x_lo,
                                                float* x_hi) {
    if (!R.fast || !(R.s > 0.0f)) return false;
    const float a = ip.lo + 0.5f, b = ip.hi - 0.5f;          // exact half-integers
    // rne: a tie at a rounds up iff lo + 1 is even; rhaz: iff a > 0.
    const bool a_incl = RHAZ ? (a > 0.0f) : ((((int)ip.lo + 1) & 1) == 0);
    const bool b_incl = RHAZ ? (b < 0.0f) : ((((int)ip.hi - 1) & 1) == 0);
    const float ap = a_incl ? a : nextafterf(a, INFINITY);
    const float bp = b_incl ? b : nextafterf(b, -INFINITY);
    float xl = __fmul_rn(ap, R.s), xh = __fmul_rn(bp, R.s);
    if (!(fabsf(xl) >= 0x1p-90f && fabsf(xl) <= 0x1p90f && fabsf(xh) >= 0x1p-90f && fabsf(xh) <= 0x1p90f))
        return false;
    // x_lo: smallest x with quot(x) >= ap.
    bool ok = false;
    if (quot(xl, R) >= ap) {
        for (int i = 0; i < 8; ++i) {
            const float d = nextafterf(xl, -INFINITY);
            if (quot(d, R) >= ap) xl = d; else { ok = true; break; }
        }
    } else {
        for (int i = 0; i < 8; ++i) {
            xl = nextafterf(xl, INFINITY);
            if (quot(xl, R) >= ap) { ok = true; break; }
        }
    }
    if (!ok) return false;
    ok = false;
    // x_hi: largest x with quot(x) <= bp.
    if (quot(xh, R) <= bp) {
        for (int i = 0; i < 8; ++i) {
            const float u = nextafterf(xh, INFINITY);
            if (quot(u, R) <= bp) xh = u; else { ok = true; break; }
        }
    } else {
        for (int i = 0; i < 8; ++i) {
            xh = nextafterf(xh, -INFINITY);
            if (quot(xh, R) <= bp) { ok = true; break; }
        }
    }
    if (!ok) return false;
    *x_lo = xl;
    *x_hi = xh;
    return true;
}

// The same thresholds found by a whole warp at once: lanes 0..15 test the 16
// candidates RN(a' s) - 8 ulp .. + 7 ulp for the lower bound, lanes 16..31 the
// same around RN(b' s) for the upper one, and a ballot picks the boundary.
// Every lane of the warp must call it with the same arguments.
template <bool RHAZ>
__device__ __forceinline__ bool mask_thresholds_warp(const Recip& R, const IntParams& ip,
                                                     float* x_lo, float* x_hi) {
    const int lane = threadIdx.x & 31;
    if (!R.fast || !(R.s > 0.0f)) return false;
    const float a = ip.lo + 0.5f, b = ip.hi - 0.5f;
    const bool a_incl = RHAZ ? (a > 0.0f) : ((((int)ip.lo + 1) & 1) == 0);
    const bool b_incl = RHAZ ? (b < 0.0f) : ((((int)ip.hi - 1) & 1) == 0);
    const float ap = a_incl ? a : nextafterf(a, INFINITY);
    const float bp = b_incl ? b : nextafterf(b, -INFINITY);
    const bool upper = lane >= 16;
    const float target = upper ? bp : ap;
    const float x0 = __fmul_rn(target, R.s);
    const bool in_range = fabsf(x0) >= 0x1p-90f && fabsf(x0) <= 0x1p90f;
    // x0 + k ulp in value order (x0 != 0 and no sign change within 8 ulp).
    const int k = (lane & 15) - 8;
    const int step = (x0 > 0.0f) ? k : -k;
    const float cand = __int_as_float(__float_as_int(x0) + step);
    const float qv = quot(cand, R);
    const bool pred = upper ? (qv <= bp) : (qv >= ap);
    const unsigned bal = __ballot_sync(0xffffffffu, pred && in_range);
    const unsigned ok_all = __ballot_sync(0xffffffffu, in_range);
    if (ok_all != 0xffffffffu) return false;
    // The quotient is exact and monotone in the candidate, so the true lanes
    // of each half are contiguous: an up-set below (lanes 0..15), a down-set
    // above (lanes 16..31). Each boundary must fall strictly inside its half.
    const unsigned lo_bits = bal & 0xFFFFu, hi_bits = bal >> 16;
    if (lo_bits == 0u || (lo_bits & 1u)) return false;        // k = -8 true or none true
    if (hi_bits == 0u || (hi_bits & 0x8000u)) return false;   // k = +7 true or none true
    const int first_lo = __ffs(lo_bits) - 1;                  // lane of the smallest true
    const int last_hi = 31 - __clz(hi_bits);                   // largest true, within the half
    const float xl = __shfl_sync(0xffffffffu, cand, first_lo);
    const float xh = __shfl_sync(0xffffffffu, cand, 16 + last_hi);
    *x_lo = xl;
    *x_hi = xh;
    return true;
}

// Group state from a known scale and zero-point (static parameters).
template <class T, bool MASK, bool RHAZ>
__device__ __forceinline__ void group_set(const MapArgs& a, int64_t seg, float s, int zp, GState& st) {
    using Acc = typename Traits<T>::Acc;
    st.seg = seg;
    st.s = s;
    st.zp = zp;
    st.R = make_recip(s);
    st.ip = make_int_params(a.cfg.qmin, a.cfg.qmax, zp);
    st.mfast = false;
    if constexpr (MASK && !std::is_same<Acc, double>::value)
        st.mfast = mask_thresholds<RHAZ>(st.R, st.ip, &st.x_lo, &st.x_hi);
    st.fast = st.mfast && st.R.fast;
}

template <class T, int PSRC, bool MASK = false, bool RHAZ = false>
__device__ __forceinline__ void load_group(const MapArgs& a, int64_t seg, bool writer, GState& st) {
    using Acc = typename Traits<T>::Acc;
    st.seg = seg;
    if (PSRC == PS_RANGE) {
        Acc hi, nlo;
        range_from_bits(a.ranges[2 * seg], hi);
        range_from_bits(a.ranges[2 * seg + 1], nlo);
        if constexpr (std::is_same<Acc, double>::value) {
            const GroupD g = derive_d(hi, nlo, a.cfg);
            st.s = g.s; st.zp = g.zp;
        } else {
            const GroupF g = derive_f(hi, nlo, a.cfg);
            st.s = g.s; st.zp = g.zp;
        }
        if (writer) {
            a.scale_out[seg] = st.s;
            if (a.zp_out) a.zp_out[seg] = (uint8_t)st.zp;
        }
    } else {
        st.s = __ldg(a.scale_in + seg);
        st.zp = a.cfg.symmetric ? 0 : load_zp(a.zp_in, seg, a.cfg.q_signed);
    }
    st.R = make_recip(st.s);
    st.ip = make_int_params(a.cfg.qmin, a.cfg.qmax, st.zp);
    st.mfast = false;
    if constexpr (MASK && !std::is_same<Acc, double>::value)
        st.mfast = mask_thresholds<RHAZ>(st.R, st.ip, &st.x_lo, &st.x_hi);
    st.fast = st.mfast && st.R.fast;
}

// As load_group, with the mask thresholds searched by the whole warp; every
// lane of the warp must be in the same group.
template <class T, int PSRC, bool RHAZ = false>
__device__ __forceinline__ void load_group_warp_mask(const MapArgs& a, int64_t seg, bool writer,
                                                     GState& st) {
    load_group<T, PSRC, false, RHAZ>(a, seg, writer, st);
    st.mfast = mask_thresholds_warp<RHAZ>(st.R, st.ip, &st.x_lo, &st.x_hi);
    st.fast = st.mfast && st.R.fast;
}

// Backward element with a fast group (thresholds valid, normal scale): no
// branches. QBWD: dx = (dy * RN(1/s)) * m; FBWD: dx = dy * m.
template <int OP>
__device__ __forceinline__ float elem_bwd_fast(float xa, float xb, const GState& st) {
    const float m = (xa >= st.x_lo && xa <= st.x_hi) ? 1.0f : 0.0f;
    if constexpr (OP == OP_QBWD) return __fmul_rn(__fmul_rn(xb, st.R.y), m);
    else return __fmul_rn(xb, m);
}

// One element, f32 arithmetic. Returns the output value (float ops) or the
// code byte (QUANT) in the low byte of *code.
template <int OP, bool RHAZ>
__device__ __forceinline__ float elem_f(float xa, float xb, const GState& st, uint32_t* code) {
    if constexpr (OP == OP_QUANT || OP == OP_FAKE) {
        const float v = div_any(xa, st.R);
        const float t = rounded_of<RHAZ>(v, st.ip);
        *code = code_from_rounded(t, st.ip.zp);
        if constexpr (OP == OP_FAKE) return dequant_from_rounded(t, st.s);
        return 0.0f;
    } else if constexpr (OP == OP_QBWD || OP == OP_FBWD) {
        // Mask 1[qmin < round(fl(x/s)) + zp < qmax]: the interval test on x
        // (NaN fails both comparisons), or the exact quotient per element.
        float m;
        if (st.mfast) {
            m = (xa >= st.x_lo && xa <= st.x_hi) ? 1.0f : 0.0f;
        } else {
            const float k = round_for_mask<RHAZ>(div_any(xa, st.R), st.ip);
            m = (k > st.ip.lo && k < st.ip.hi) ? 1.0f : 0.0f;
        }
        if constexpr (OP == OP_QBWD) {
            // Gradient dy * RN(1/s): within one ulp of fl(dy/s) (the STE
            // tolerance); the IEEE quotient when the scale is outside the
            // fast range.
            const float g = st.R.fast ? __fmul_rn(xb, st.R.y)
                                      : with_quotient_sign(div_slow(xb, st.s), xb, st.s);
            return __fmul_rn(g, m);
        } else {
            return __fmul_rn(xb, m);
        }
    } else if constexpr (OP == OP_DBWD) {
        return __fmul_rn(xa, st.s);
    } else {
        return 0.0f;
    }
}

// f64 arithmetic (f64 tensors).
template <int OP, bool RHAZ>
__device__ __forceinline__ double elem_d(double xa, double xb, const GState& st, uint32_t* code) {
    const double s = (double)st.s;
    const double lo = (double)st.ip.lo, hi = (double)st.ip.hi;
    if constexpr (OP == OP_QUANT || OP == OP_FAKE) {
        const double v = xa / s;
        double k = RHAZ ? round(v) : rint(v);
        k = fmin(fmax(k, lo), hi);                  // NaN -> lo
        *code = (uint32_t)((int)k + st.zp);
        if constexpr (OP == OP_FAKE) return (double)((int)k) * s;   // (q - zp) as an integer: +0, never -0
        return 0.0;
    } else if constexpr (OP == OP_QBWD || OP == OP_FBWD) {
        const double v = xa / s;
        double k = RHAZ ? round(v) : rint(v);
        if (v != v) k = lo;
        const double m = (k > lo && k < hi) ? 1.0 : 0.0;
        if constexpr (OP == OP_QBWD) return (xb / s) * m;
        else return xb * m;
    } else if constexpr (OP == OP_DBWD) {
        return xa * s;
    } else {
        return 0.0;
    }
}

// Dequantize one code: (q - zp) * s. The byte goes into the low mantissa of
// 2^23 so that one f32 subtraction gives q - zp exactly.
__device__ __forceinline__ float deq_code_f(uint32_t word, int i, const GState& st, int q_signed) {
    if (q_signed) word ^= 0x80808080u;
    const uint32_t sel = (uint32_t)i | (4u << 4) | (5u << 8) | (7u << 12);
    const float f = __uint_as_float(__byte_perm(word, 0x4B000000u, sel));
    const float off = 8388608.0f + (float)((q_signed ? 128 : 0) + st.zp);
    return __fmul_rn(__fsub_rn(f, off), st.s);
}


}  // namespace bq
