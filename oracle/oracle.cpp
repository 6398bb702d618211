// CPU oracle for scaled quantize / dequantize — TEST INFRASTRUCTURE ONLY.
//
// Plain, slow, single-threaded C++17. Only the tests, the smoke check and the
// benchmark's CPU-baseline leg may load it; the library never does. It shares
// no code, header, table or constant with the CUDA path.
//
// Sources (pages, with the section each function follows):
//   [baracuda]  docs.rs baracuda_kernels::quantize — module index: op list,
//               dtype coverage (input f32/f64/f16/bf16, output s8/u8), the
//               Straight-Through-Estimator backward dx = (dy/scale)*1[qmin<q<qmax]
//               with the mask recomputed from the saved input, the dequantize
//               backward plans (dq = dy*scale), fake_quantize "FP roundtrip",
//               and default_q_range (S8 [-128,127], U8 [0,255]).
//   [granularity] teenygrad teeny_quant/quant/granularity.rs — enum
//               Granularity {PerTensor, PerChannel{axis}, Group{axis,group_size}}
//               and axis_and_group_size(): PerChannel{axis} == (axis, 1).
//   [QuantizedWeight] docs.metrale.ai QuantizedWeight — NVFP4 layout: packed
//               E2M1 two per byte, FP8 scale per 16, f32 per-tensor
//               weight_scale_2; transpose_for_gemm(_gs) and the padded
//               transpose (stride = align_up(n, align), pad zeroed); the
//               multi-part transpose_concat_for_gemm(_gs, _padded),
//               concat_rows and predequant_to_fp8.
//   [smile.llm.quant] package summary — Fp8BlockGemm / Fp8BlockDequant
//               (E4M3, f32 scale per 1x128 activation group and per 128x128
//               weight tile, weight_scale_inv) and MxFp8 (E4M3, E8M0 scale per
//               32 consecutive elements along the reduction dimension) and
//               Fp8KvCodec (FP8 KV store / load with per-tensor scales).
//
// Precision. The pages fix no precision. Every result of this path ends in a
// discrete encoding (an integer code, an FP8/FP4 code, a bf16/f16/f32 value),
// and a code must be decided in the same precision on both sides, so each
// step is computed in f64 and rounded once to f32, which is exactly the IEEE
// f32 result of that step (f32 products are exact in f64; for quotients,
// sums and differences of f32 operands one f64 rounding followed by one f32
// rounding is innocuous because 53 >= 2*24+2: S. Figueroa, "When is double
// rounding innocuous?", SIGNUM Newsletter 30(3), 1995). For f64 inputs the
// steps stay in f64. No step is fused (built with -ffp-contract=off).
//
// Conventions the pages leave open (each is listed again in the design notes):
//   * group of Group{axis, gs}: x viewed as [outer, L, inner]; group g of
//     outer index o holds axis indices [g*gs, (g+1)*gs) and every inner index.
//   * symmetric scale s = fl(amax / qmax); asymmetric s = fl(fl(max'-min') /
//     (qmax-qmin)) with min' = min(min x, 0), max' = max(max x, 0) and
//     zp = clamp(qmin - rne(fl(min'/s)), qmin, qmax); a scale that comes out
//     as 0 is replaced by 1. Range reductions ignore NaN.
//   * q = clamp(rne(fl(x/s)) + zp, qmin, qmax); a NaN quotient gives qmin.
//   * dequantize y = RN_y(fl((q-zp)*s)); f64 outputs keep the exact product.
//   * E4M3 encode is round-to-nearest-even with saturation to +-448, NaN ->
//     0x7F; E2M1 encode is round-to-nearest-even with saturation to +-6 and
//     the sign bit kept, NaN -> 0x0 (+0: E2M1 has no NaN, and IEEE 754-2019
//     6.3 gives a NaN's sign bit no meaning, so the code carries no sign,
//     as E4M3's single NaN code carries none); E2M1 element 2j goes to the
//     low nibble of byte j.
//   * NVFP4: s2 = fl(A/2688) (2688 = 448*6), sb = E4M3(fl(a_b/fl(6*s2))),
//     eff = fl(dec(sb)*s2), code = E2M1(fl(x/eff)), all-zero codes when
//     eff == 0.
//   * MXFP8: E = clamp(floor(log2 a) - 8, -127, 127), byte = E + 127 (an
//     infinite a counts as 2^128), e = E4M3(fl(x * 2^-E)). MXFP4: the same
//     with 2 (the largest E2M1 exponent) in place of 8 and E2M1 codes.
//   * FP8 block: s = fl(a/448) (0 -> 1), e = E4M3(fl(x/s)), s is stored.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

namespace {

// ---------------------------------------------------------------------------
// Element types understood by the oracle (its own numbering).
// OR_S4 / OR_U4: 4-bit codes packed two per byte, element 2j in the low
// nibble of byte j (the nibble order of packed E2M1 on the QuantizedWeight
// page); their zero-points are stored one per byte (s8 / u8).
enum OrType { OR_F32 = 0, OR_F64 = 1, OR_F16 = 2, OR_BF16 = 3, OR_S8 = 4, OR_U8 = 5, OR_S4 = 6, OR_U4 = 7 };

// ---------------------------------------------------------------------------
// Small floating-point formats, decoded from their bit-field definitions:
// value = (-1)^s * 2^(e - bias) * (1 + m / 2^M) for e != 0 and
//         (-1)^s * 2^(1 - bias) * (m / 2^M)      for e == 0.
// f16 (IEEE binary16), bf16 (8-bit exponent, 7-bit fraction) and the OCP
// FP8 E4M3 / FP4 E2M1 element formats.
struct MiniFmt {
    int ebits, mbits, bias;
    bool ieee_special;   // all-ones exponent encodes inf (m == 0) / NaN
    bool e4m3_nan;       // only S.1111.111 is NaN, no infinities
    std::vector<double> pos;  // value of every non-negative finite code, in code order
    int max_code;             // largest finite positive code
};

double mini_decode_fields(const MiniFmt& f, uint32_t code) {
    const uint32_t emask = (1u << f.ebits) - 1, mmask = (1u << f.mbits) - 1;
    const int s = (code >> (f.ebits + f.mbits)) & 1;
    const uint32_t e = (code >> f.mbits) & emask, m = code & mmask;
    double v;
    if (f.ieee_special && e == emask) {
        v = (m == 0) ? INFINITY : NAN;
    } else if (f.e4m3_nan && e == emask && m == mmask) {
        v = NAN;
    } else if (e == 0) {
        v = std::ldexp((double)m, 1 - f.bias - f.mbits);
    } else {
        v = std::ldexp((double)((1u << f.mbits) + m), (int)e - f.bias - f.mbits);
    }
    return s ? -v : v;
}

MiniFmt make_fmt(int ebits, int mbits, int bias, bool ieee, bool e4m3) {
    MiniFmt f{ebits, mbits, bias, ieee, e4m3, {}, 0};
    const uint32_t npos = 1u << (ebits + mbits);
    for (uint32_t c = 0; c < npos; ++c) {
        double v = mini_decode_fields(f, c);
        if (!std::isfinite(v)) break;   // codes are monotonic; specials sit at the top
        f.pos.push_back(v);
        f.max_code = (int)c;
    }
    return f;
}

const MiniFmt& fmt_f16()  { static MiniFmt f = make_fmt(5, 10, 15, true, false); return f; }
const MiniFmt& fmt_bf16() { static MiniFmt f = make_fmt(8, 7, 127, true, false); return f; }
const MiniFmt& fmt_e4m3() { static MiniFmt f = make_fmt(4, 3, 7, false, true); return f; }
const MiniFmt& fmt_e2m1() { static MiniFmt f = make_fmt(2, 1, 1, false, false); return f; }

// Round-to-nearest-even of v onto the format's grid. `sat`: values beyond the
// largest finite magnitude give that magnitude (satfinite), otherwise IEEE
// overflow to infinity. The tie rule picks the code whose last mantissa bit
// is 0, i.e. the even code.
uint32_t mini_encode(const MiniFmt& f, double v, bool sat, uint32_t nan_code) {
    const uint32_t sign_bit = 1u << (f.ebits + f.mbits);
    if (std::isnan(v)) return nan_code;
    const uint32_t sgn = std::signbit(v) ? sign_bit : 0u;
    const double a = std::fabs(v);
    const double top = f.pos[f.max_code];
    uint32_t code;
    if (a >= top) {
        if (sat) {
            code = (uint32_t)f.max_code;
        } else {
            // The value after the largest finite one, with an unbounded exponent.
            const double next = top + (top - f.pos[f.max_code - 1]);
            const double mid = 0.5 * (top + next);
            code = (a >= mid) ? (uint32_t)(f.max_code + 1) : (uint32_t)f.max_code;  // max_code+1 = inf
        }
    } else {
        // Largest i with pos[i] <= a.
        size_t i = (size_t)(std::upper_bound(f.pos.begin(), f.pos.end(), a) - f.pos.begin()) - 1;
        if (f.pos[i] == a) {
            code = (uint32_t)i;
        } else {
            const double mid = 0.5 * (f.pos[i] + f.pos[i + 1]);  // exact in f64
            if (a < mid) code = (uint32_t)i;
            else if (a > mid) code = (uint32_t)(i + 1);
            else code = (i % 2 == 0) ? (uint32_t)i : (uint32_t)(i + 1);
        }
    }
    return code | sgn;
}

uint16_t enc_f16(double v)  { return (uint16_t)mini_encode(fmt_f16(), v, false, 0x7E00u); }
uint16_t enc_bf16(double v) { return (uint16_t)mini_encode(fmt_bf16(), v, false, 0x7FC0u); }
uint8_t  enc_e4m3(double v) { return (uint8_t)mini_encode(fmt_e4m3(), v, true, 0x7Fu); }
uint8_t  enc_e2m1(double v) {
    // No NaN in E2M1: a NaN of either sign becomes +0 (code 0x0).
    return (uint8_t)mini_encode(fmt_e2m1(), v, true, 0x0u);
}
double dec_f16(uint16_t c)  { return mini_decode_fields(fmt_f16(), c); }
double dec_bf16(uint16_t c) { return mini_decode_fields(fmt_bf16(), c); }
double dec_e4m3(uint8_t c)  { return mini_decode_fields(fmt_e4m3(), c); }
double dec_e2m1(uint8_t c)  { return mini_decode_fields(fmt_e2m1(), c & 0xF); }
// E8M0 (OCP MX scale): 2^(b - 127); 0xFF is NaN.
double dec_e8m0(uint8_t b)  { return b == 0xFF ? NAN : std::ldexp(1.0, (int)b - 127); }

// One IEEE f32 rounding of an f64 value (x86-64 SSE conversion, IEEE 754).
double r32(double v) { return (double)(float)v; }

// ---------------------------------------------------------------------------
// Element access.
bool is_float_type(int t) { return t == OR_F32 || t == OR_F64 || t == OR_F16 || t == OR_BF16; }

double load_f(const void* p, int t, int64_t i) {
    switch (t) {
        case OR_F32: { float v; std::memcpy(&v, (const char*)p + 4 * i, 4); return v; }
        case OR_F64: { double v; std::memcpy(&v, (const char*)p + 8 * i, 8); return v; }
        case OR_F16: { uint16_t c; std::memcpy(&c, (const char*)p + 2 * i, 2); return dec_f16(c); }
        case OR_BF16: { uint16_t c; std::memcpy(&c, (const char*)p + 2 * i, 2); return dec_bf16(c); }
    }
    return NAN;
}
// Store a value that is already exact in f32 (or f64 for OR_F64) with one
// round-to-nearest-even into the destination type.
void store_f(void* p, int t, int64_t i, double v) {
    switch (t) {
        case OR_F32: { float f = (float)v; std::memcpy((char*)p + 4 * i, &f, 4); break; }
        case OR_F64: { std::memcpy((char*)p + 8 * i, &v, 8); break; }
        case OR_F16: { uint16_t c = enc_f16(v); std::memcpy((char*)p + 2 * i, &c, 2); break; }
        case OR_BF16: { uint16_t c = enc_bf16(v); std::memcpy((char*)p + 2 * i, &c, 2); break; }
    }
}
int64_t load_i(const void* p, int t, int64_t i) {
    if (t == OR_S4 || t == OR_U4) {
        const int nib = (((const uint8_t*)p)[i / 2] >> (4 * (i % 2))) & 0xF;
        return (t == OR_S4 && nib >= 8) ? nib - 16 : nib;
    }
    return t == OR_S8 ? (int64_t)((const int8_t*)p)[i] : (int64_t)((const uint8_t*)p)[i];
}
void store_i(void* p, int t, int64_t i, int64_t v) {
    if (t == OR_S4 || t == OR_U4) {
        uint8_t& b = ((uint8_t*)p)[i / 2];
        const int sh = 4 * (int)(i % 2);
        b = (uint8_t)((b & ~(0xF << sh)) | (((int)v & 0xF) << sh));
        return;
    }
    if (t == OR_S8) ((int8_t*)p)[i] = (int8_t)v; else ((uint8_t*)p)[i] = (uint8_t)v;
}
bool is_int_type(int t) { return t == OR_S8 || t == OR_U8 || t == OR_S4 || t == OR_U4; }
// Zero-points of a code type: one byte per group (s8 for signed codes).
int zp_type(int q_t) { return (q_t == OR_S8 || q_t == OR_S4) ? OR_S8 : OR_U8; }

// ---------------------------------------------------------------------------
// Rounding a real value to an integer.
// rne: nearest integer, ties to the even one. rhaz: ties away from zero.
double round_rne(double v) {
    if (!std::isfinite(v)) return v;
    double f = std::floor(v);
    double d = v - f;                  // exact: 0 <= d < 1
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (std::fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}
double round_rhaz(double v) {
    if (!std::isfinite(v)) return v;
    double f = std::floor(v);
    double d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return v > 0 ? f + 1.0 : f;        // halves move away from zero
}

// ---------------------------------------------------------------------------
// [granularity] Granularity -> (axis, group_size); PerTensor has none.
// Group g of outer index o covers axis indices [g*gs, (g+1)*gs) and all inner
// indices: with x viewed as [outer, L, inner] the element (o, l, i) sits at
// (o*L + l)*inner + i.
// Column groups (GRAN_COLUMN): the Group granularity read as blocks of gs
// consecutive indices along `axis` at one fixed index of the dimensions after
// it (the [K, N]-stored weight of a GPTQ-style quantizer grouped along K):
// group (o, b, i) holds the elements (o, l, i) for l in [b*gs, (b+1)*gs), and
// groups are numbered (o*(L/gs) + b)*inner + i, i.e. a scale array of shape
// [outer, L/gs, inner].
enum OrGran { GRAN_TENSOR = 0, GRAN_CHANNEL = 1, GRAN_GROUP = 2, GRAN_TOKEN = 3, GRAN_COLUMN = 4 };

struct Layout {
    int64_t outer = 1, L = 1, inner = 1, gs = 1;   // groups per outer = L / gs
    bool column = false;                           // one group per inner index
    bool ok = true;
    int64_t n_groups() const { return outer * (gs ? L / gs : 0) * (column ? inner : 1); }
    int64_t group_elems() const { return column ? gs : gs * inner; }
    int64_t numel() const { return outer * L * inner; }
};

Layout make_layout(int ndim, const int64_t* shape, int gran, int axis, int64_t gs) {
    Layout lay;
    if (ndim < 0 || ndim > 8) { lay.ok = false; return lay; }
    int64_t numel = 1;
    for (int d = 0; d < ndim; ++d) { if (shape[d] < 0) lay.ok = false; numel *= shape[d]; }
    if (gran == GRAN_TENSOR) {
        // One group holding every element.
        lay.outer = 1; lay.L = 1; lay.inner = numel; lay.gs = 1;
        return lay;
    }
    if (gran == GRAN_TOKEN) {
        // One group per row of the last dimension.
        if (ndim < 1) { lay.ok = false; return lay; }
        lay.outer = numel / std::max<int64_t>(shape[ndim - 1], 1);
        if (shape[ndim - 1] == 0) lay.outer = 0;
        lay.L = shape[ndim - 1]; lay.inner = 1; lay.gs = shape[ndim - 1];
        if (lay.gs == 0) { lay.gs = 1; lay.L = 0; }
        return lay;
    }
    if (axis < 0 || axis >= ndim) { lay.ok = false; return lay; }
    if (gran == GRAN_CHANNEL) gs = 1;          // PerChannel{axis} -> (axis, 1)
    if (gran != GRAN_CHANNEL && gran != GRAN_GROUP && gran != GRAN_COLUMN) { lay.ok = false; return lay; }
    if (gs < 1) { lay.ok = false; return lay; }
    lay.column = (gran == GRAN_COLUMN);
    lay.outer = 1; lay.inner = 1;
    for (int d = 0; d < axis; ++d) lay.outer *= shape[d];
    for (int d = axis + 1; d < ndim; ++d) lay.inner *= shape[d];
    lay.L = shape[axis];
    lay.gs = gs;
    if (lay.L % gs != 0) lay.ok = false;       // group_size must divide the axis
    return lay;
}

template <class F>
void for_each_in_group(const Layout& lay, int64_t group, F&& fn) {
    const int64_t per_outer = lay.L / lay.gs;
    if (lay.column) {
        const int64_t i = group % lay.inner, ob = group / lay.inner;
        const int64_t o = ob / per_outer, b = ob % per_outer;
        for (int64_t l = b * lay.gs; l < (b + 1) * lay.gs; ++l) fn((o * lay.L + l) * lay.inner + i);
        return;
    }
    const int64_t o = group / per_outer, g = group % per_outer;
    for (int64_t l = g * lay.gs; l < (g + 1) * lay.gs; ++l)
        for (int64_t i = 0; i < lay.inner; ++i)
            fn((o * lay.L + l) * lay.inner + i);
}

struct QParams {
    int x_t, q_t;
    int symmetric;
    int64_t qmin, qmax;
    int rhaz;
};

bool default_range(int q_t, int64_t* qmin, int64_t* qmax) {
    // [baracuda] default_q_range: S8 -> [-128, 127], U8 -> [0, 255].
    if (q_t == OR_S8) { *qmin = -128; *qmax = 127; return true; }
    if (q_t == OR_U8) { *qmin = 0; *qmax = 255; return true; }
    // s4 / u4 (deferred to a later milestone on the baracuda page): the
    // two's-complement and unsigned 4-bit ranges.
    if (q_t == OR_S4) { *qmin = -8; *qmax = 7; return true; }
    if (q_t == OR_U4) { *qmin = 0; *qmax = 15; return true; }
    return false;
}

// Range of a group: max(0, max x) and max(0, -min x), NaN ignored.
void group_range(const void* x, int x_t, const Layout& lay, int64_t g, double* hi, double* neg_lo) {
    double mx = 0.0, mn = 0.0;
    for_each_in_group(lay, g, [&](int64_t idx) {
        double v = load_f(x, x_t, idx);
        if (std::isnan(v)) return;
        if (v > mx) mx = v;
        if (v < mn) mn = v;
    });
    *hi = mx; *neg_lo = -mn;
}

// [baracuda] scale (and zero-point) of one group from its range.
// wide = f64 arithmetic (f64 inputs); otherwise every step is rounded to f32.
void derive_scale(const QParams& P, bool wide, double hi, double neg_lo, float* s_out, int64_t* zp_out) {
    auto rnd = [&](double v) { return wide ? v : r32(v); };
    if (P.symmetric) {
        double a = std::max(hi, neg_lo);                 // max |x|
        float s = (float)(a / (double)P.qmax);
        if (s == 0.0f) s = 1.0f;
        *s_out = s; *zp_out = 0;
    } else {
        double mx = hi, mn = -neg_lo;                    // max' >= 0, min' <= 0
        double span = rnd(mx - mn);
        float s = (float)(span / (double)(P.qmax - P.qmin));
        if (s == 0.0f) s = 1.0f;
        double r = P.rhaz ? round_rhaz(rnd(mn / (double)s)) : round_rne(rnd(mn / (double)s));
        double zp = (double)P.qmin - r;
        if (std::isnan(zp)) zp = (double)P.qmin;
        zp = std::min(std::max(zp, (double)P.qmin), (double)P.qmax);
        *s_out = s; *zp_out = (int64_t)zp;
    }
}

// [baracuda] q = clamp(round(x/s) + zp, qmin, qmax); unclamped code for the STE mask.
double quant_unclamped(const QParams& P, bool wide, double x, float s, int64_t zp) {
    double v = wide ? x / (double)s : r32(x / (double)s);
    if (std::isnan(v)) return (double)P.qmin;
    double k = P.rhaz ? round_rhaz(v) : round_rne(v);
    return k + (double)zp;
}
int64_t quant_one(const QParams& P, bool wide, double x, float s, int64_t zp) {
    double k = quant_unclamped(P, wide, x, s, zp);
    k = std::min(std::max(k, (double)P.qmin), (double)P.qmax);
    return (int64_t)k;
}
// [baracuda] dequantize: (q - zp) * scale in f32 (exact product in f64 for f64 outputs).
double dequant_one(int64_t q, int64_t zp, float s, int y_t) {
    double prod = (double)(q - zp) * (double)s;          // exact in f64
    return y_t == OR_F64 ? prod : r32(prod);
}

bool check_params(QParams& P, int64_t qmin, int64_t qmax) {
    if (!is_float_type(P.x_t)) return false;
    if (!is_int_type(P.q_t)) return false;
    int64_t dmin, dmax;
    default_range(P.q_t, &dmin, &dmax);
    if (qmin == 0 && qmax == 0) { qmin = dmin; qmax = dmax; }
    if (qmin < dmin || qmax > dmax || qmin >= qmax) return false;
    if (P.symmetric && (P.q_t == OR_U8 || P.q_t == OR_U4 || qmax <= 0)) return false;
    P.qmin = qmin; P.qmax = qmax;
    return true;
}

}  // namespace

// ===========================================================================
// Exported entry points (ctypes). Return 0 on success, 1 on invalid input.
extern "C" {

// ---- codecs over arrays (f64 in / codes out, and back) --------------------
// fmt: 0 f16, 1 bf16, 2 e4m3, 3 e2m1 (one code per byte), 4 e8m0 (decode only)
int or_encode(int fmt, const double* v, int64_t n, void* out) {
    for (int64_t i = 0; i < n; ++i) {
        switch (fmt) {
            case 0: ((uint16_t*)out)[i] = enc_f16(v[i]); break;
            case 1: ((uint16_t*)out)[i] = enc_bf16(v[i]); break;
            case 2: ((uint8_t*)out)[i] = enc_e4m3(v[i]); break;
            case 3: ((uint8_t*)out)[i] = enc_e2m1(v[i]); break;
            default: return 1;
        }
    }
    return 0;
}
// The same encoders over a run of f32 bit patterns: value i is the f32 whose
// bits are first + i (count <= 2^32 - first), so a caller can sweep every f32.
int or_encode_f32_bits(int fmt, uint32_t first, int64_t count, void* out) {
    if (fmt < 0 || fmt > 3 || count < 0 || (uint64_t)first + (uint64_t)count > (1ull << 32)) return 1;
    for (int64_t i = 0; i < count; ++i) {
        const uint32_t bits = first + (uint32_t)i;
        float f;
        std::memcpy(&f, &bits, 4);
        const double v = f;
        switch (fmt) {
            case 0: ((uint16_t*)out)[i] = enc_f16(v); break;
            case 1: ((uint16_t*)out)[i] = enc_bf16(v); break;
            case 2: ((uint8_t*)out)[i] = enc_e4m3(v); break;
            default: ((uint8_t*)out)[i] = enc_e2m1(v); break;
        }
    }
    return 0;
}
int or_decode(int fmt, const void* codes, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) {
        switch (fmt) {
            case 0: out[i] = dec_f16(((const uint16_t*)codes)[i]); break;
            case 1: out[i] = dec_bf16(((const uint16_t*)codes)[i]); break;
            case 2: out[i] = dec_e4m3(((const uint8_t*)codes)[i]); break;
            case 3: out[i] = dec_e2m1(((const uint8_t*)codes)[i]); break;
            case 4: out[i] = dec_e8m0(((const uint8_t*)codes)[i]); break;
            default: return 1;
        }
    }
    return 0;
}
// Round each value to an integer (ties to even, or away from zero when rhaz).
int or_round_int(const double* v, int64_t n, int rhaz, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = rhaz ? round_rhaz(v[i]) : round_rne(v[i]);
    return 0;
}

int or_default_q_range(int q_t, int64_t* qmin, int64_t* qmax) {
    return default_range(q_t, qmin, qmax) ? 0 : 1;
}

// [granularity] layout query: number of groups and elements per group.
int or_group_count(int ndim, const int64_t* shape, int gran, int axis, int64_t gs,
                   int64_t* n_groups, int64_t* group_elems) {
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok) return 1;
    *n_groups = lay.n_groups();
    *group_elems = lay.group_elems();
    return 0;
}

// [granularity] range of every group: hi = max(0, max x), neg_lo = max(0, -min x).
int or_group_range(const void* x, int x_t, int ndim, const int64_t* shape, int gran, int axis,
                   int64_t gs, double* hi, double* neg_lo) {
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok || !is_float_type(x_t)) return 1;
    for (int64_t g = 0; g < lay.n_groups(); ++g) group_range(x, x_t, lay, g, &hi[g], &neg_lo[g]);
    return 0;
}

// [baracuda] quantize_per_{tensor,channel,token,group}.
// scale_mode 0: derive scale/zp from each group's range and write them.
// scale_mode 1: read scale/zp (static).
// scale_mode 2: derive from the ranges given in range_hi/range_neg_lo (one per
//               group), e.g. ranges combined across shards.
int or_quantize(const void* x, int x_t, int ndim, const int64_t* shape, int gran, int axis,
                int64_t gs, int q_t, int symmetric, int64_t qmin, int64_t qmax, int rhaz,
                int scale_mode, const double* range_hi, const double* range_neg_lo,
                void* q, float* scale, void* zp) {
    QParams P{x_t, q_t, symmetric, 0, 0, rhaz};
    if (!check_params(P, qmin, qmax)) return 1;
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok) return 1;
    const bool wide = (x_t == OR_F64);
    for (int64_t g = 0; g < lay.n_groups(); ++g) {
        float s; int64_t z;
        if (scale_mode == 1) {
            s = scale[g];
            z = (zp && !symmetric) ? load_i(zp, zp_type(q_t), g) : 0;
        } else {
            double hi, nlo;
            if (scale_mode == 2) { hi = range_hi[g]; nlo = range_neg_lo[g]; }
            else group_range(x, x_t, lay, g, &hi, &nlo);
            derive_scale(P, wide, hi, nlo, &s, &z);
            scale[g] = s;
            if (zp) store_i(zp, zp_type(q_t), g, z);
        }
        for_each_in_group(lay, g, [&](int64_t idx) {
            store_i(q, q_t, idx, quant_one(P, wide, load_f(x, x_t, idx), s, z));
        });
    }
    return 0;
}

// [baracuda] dequantize_per_{tensor,channel,token,group}: y = (q - zp) * scale.
int or_dequantize(const void* q, int q_t, const float* scale, const void* zp, int ndim,
                  const int64_t* shape, int gran, int axis, int64_t gs, void* y, int y_t) {
    if (!is_int_type(q_t)) return 1;
    if (!is_float_type(y_t)) return 1;
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok) return 1;
    for (int64_t g = 0; g < lay.n_groups(); ++g) {
        const float s = scale[g];
        const int64_t z = zp ? load_i(zp, zp_type(q_t), g) : 0;
        for_each_in_group(lay, g, [&](int64_t idx) {
            store_f(y, y_t, idx, dequant_one(load_i(q, q_t, idx), z, s, y_t));
        });
    }
    return 0;
}

// [baracuda] fake_quantize: quantize then dequantize back to the input dtype
// ("FP roundtrip"). scale_mode as in or_quantize.
int or_fake_quantize(const void* x, int x_t, int ndim, const int64_t* shape, int gran, int axis,
                     int64_t gs, int q_t, int symmetric, int64_t qmin, int64_t qmax, int rhaz,
                     int scale_mode, const double* range_hi, const double* range_neg_lo,
                     float* scale, void* zp, void* y) {
    QParams P{x_t, q_t, symmetric, 0, 0, rhaz};
    if (!check_params(P, qmin, qmax)) return 1;
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok) return 1;
    const bool wide = (x_t == OR_F64);
    for (int64_t g = 0; g < lay.n_groups(); ++g) {
        float s; int64_t z;
        if (scale_mode == 1) {
            s = scale[g];
            z = (zp && !symmetric) ? load_i(zp, zp_type(q_t), g) : 0;
        } else {
            double hi, nlo;
            if (scale_mode == 2) { hi = range_hi[g]; nlo = range_neg_lo[g]; }
            else group_range(x, x_t, lay, g, &hi, &nlo);
            derive_scale(P, wide, hi, nlo, &s, &z);
            scale[g] = s;
            if (zp) store_i(zp, zp_type(q_t), g, z);
        }
        for_each_in_group(lay, g, [&](int64_t idx) {
            int64_t qq = quant_one(P, wide, load_f(x, x_t, idx), s, z);
            store_f(y, x_t, idx, dequant_one(qq, z, s, x_t));
        });
    }
    return 0;
}

// [baracuda] quantize_*_backward (Straight-Through Estimator):
// dx = (dy / scale) * 1[qmin < q < qmax], q recomputed from the saved x
// before clamping. kind 0: quantize backward (dy/scale, masked);
// kind 1: fake_quantize backward (dy, masked).
int or_ste_backward(int kind, const void* x, const void* dy, int x_t, const float* scale,
                    const void* zp, int ndim, const int64_t* shape, int gran, int axis,
                    int64_t gs, int q_t, int symmetric, int64_t qmin, int64_t qmax, int rhaz,
                    void* dx) {
    QParams P{x_t, q_t, symmetric, 0, 0, rhaz};
    if (!check_params(P, qmin, qmax)) return 1;
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok) return 1;
    const bool wide = (x_t == OR_F64);
    auto rnd = [&](double v) { return wide ? v : r32(v); };
    for (int64_t g = 0; g < lay.n_groups(); ++g) {
        const float s = scale[g];
        const int64_t z = (zp && !symmetric) ? load_i(zp, zp_type(q_t), g) : 0;
        for_each_in_group(lay, g, [&](int64_t idx) {
            double k = quant_unclamped(P, wide, load_f(x, x_t, idx), s, z);
            double m = ((double)P.qmin < k && k < (double)P.qmax) ? 1.0 : 0.0;
            double d = load_f(dy, x_t, idx);
            double base = (kind == 0) ? rnd(d / (double)s) : d;
            store_f(dx, x_t, idx, rnd(base * m));
        });
    }
    return 0;
}

// [baracuda] dequantize_*_backward: dq = dy * scale (straight-through).
int or_dequantize_backward(const void* dy, int dy_t, const float* scale, int ndim,
                           const int64_t* shape, int gran, int axis, int64_t gs, void* dq) {
    if (!is_float_type(dy_t)) return 1;
    Layout lay = make_layout(ndim, shape, gran, axis, gs);
    if (!lay.ok) return 1;
    const bool wide = (dy_t == OR_F64);
    for (int64_t g = 0; g < lay.n_groups(); ++g) {
        const float s = scale[g];
        for_each_in_group(lay, g, [&](int64_t idx) {
            double p = load_f(dy, dy_t, idx) * (double)s;
            store_f(dq, dy_t, idx, wide ? p : r32(p));
        });
    }
    return 0;
}

// Tensor amax (max |x|, NaN ignored), as used by per-tensor scaling and the
// NVFP4 per-tensor scale [QuantizedWeight weight_scale_2].
int or_tensor_amax(const void* x, int x_t, int64_t n, double* amax) {
    if (!is_float_type(x_t)) return 1;
    double a = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double v = std::fabs(load_f(x, x_t, i));
        if (v > a) a = v;                     // false for NaN
    }
    *amax = a;
    return 0;
}

// ---- NVFP4 [QuantizedWeight]: E2M1 packed 2/byte, E4M3 scale per 16 along K,
// f32 per-tensor scale s2. x is [n, k] row-major, k % 16 == 0.
int or_nvfp4_quantize(const void* x, int x_t, int64_t n, int64_t k, uint8_t* packed,
                      uint8_t* sc, float* s2_io, int static_s2) {
    if (x_t != OR_F32 && x_t != OR_F16 && x_t != OR_BF16) return 1;
    if (n < 0 || k < 0 || k % 16 != 0) return 1;
    float s2;
    if (static_s2) {
        s2 = *s2_io;
    } else {
        double A;
        or_tensor_amax(x, x_t, n * k, &A);
        s2 = (float)(A / 2688.0);               // 2688 = 448 * 6
        if (s2 == 0.0f) s2 = 1.0f;
        *s2_io = s2;
    }
    const double six_s2 = r32(6.0 * (double)s2);
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t b = 0; b < k / 16; ++b) {
            const int64_t base = r * k + b * 16;
            double ab = 0.0;
            for (int j = 0; j < 16; ++j) {
                double v = std::fabs(load_f(x, x_t, base + j));
                if (v > ab) ab = v;
            }
            const uint8_t sb = enc_e4m3(r32(ab / six_s2));
            sc[r * (k / 16) + b] = sb;
            const double eff = r32(dec_e4m3(sb) * (double)s2);
            for (int j = 0; j < 16; j += 2) {
                uint8_t c[2];
                for (int t = 0; t < 2; ++t) {
                    double xv = load_f(x, x_t, base + j + t);
                    c[t] = (eff == 0.0) ? 0 : enc_e2m1(r32(xv / eff));
                }
                packed[(base + j) / 2] = (uint8_t)(c[0] | (c[1] << 4));   // low nibble first
            }
        }
    }
    return 0;
}

int or_nvfp4_dequantize(const uint8_t* packed, const uint8_t* sc, float s2, int64_t n, int64_t k,
                        void* y, int y_t) {
    if (y_t != OR_F32 && y_t != OR_F16 && y_t != OR_BF16) return 1;
    if (n < 0 || k < 0 || k % 16 != 0) return 1;
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t c = 0; c < k; ++c) {
            const int64_t idx = r * k + c;
            const double eff = r32(dec_e4m3(sc[r * (k / 16) + c / 16]) * (double)s2);
            const uint8_t byte = packed[idx / 2];
            const uint8_t code = (idx % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            store_f(y, y_t, idx, r32(dec_e2m1(code) * eff));
        }
    }
    return 0;
}

// ---- MXFP8 [smile.llm.quant MxFp8]: E4M3 elements, E8M0 scale per 32
// consecutive elements along the reduction (last) dimension.
int or_mxfp8_quantize(const void* x, int x_t, int64_t rows, int64_t k, uint8_t* e4m3,
                      uint8_t* e8m0) {
    if (x_t != OR_F32 && x_t != OR_F16 && x_t != OR_BF16) return 1;
    if (rows < 0 || k < 0 || k % 32 != 0) return 1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < k / 32; ++b) {
            const int64_t base = r * k + b * 32;
            double a = 0.0;
            for (int j = 0; j < 32; ++j) {
                double v = std::fabs(load_f(x, x_t, base + j));
                if (v > a) a = v;
            }
            // floor(log2 a) - 8, where 8 = floor(log2 448), the largest E4M3 exponent.
            int fl2;
            if (a == 0.0) fl2 = -1000;
            else if (std::isinf(a)) fl2 = 128;
            else { int e; std::frexp(a, &e); fl2 = e - 1; }
            int E = std::min(std::max(fl2 - 8, -127), 127);
            e8m0[r * (k / 32) + b] = (uint8_t)(E + 127);
            const double inv = std::ldexp(1.0, -E);      // exact power of two
            for (int j = 0; j < 32; ++j)
                e4m3[base + j] = enc_e4m3(r32(load_f(x, x_t, base + j) * inv));
        }
    }
    return 0;
}

int or_mxfp8_dequantize(const uint8_t* e4m3, const uint8_t* e8m0, int64_t rows, int64_t k,
                        void* y, int y_t) {
    if (y_t != OR_F32 && y_t != OR_F16 && y_t != OR_BF16) return 1;
    if (rows < 0 || k < 0 || k % 32 != 0) return 1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k; ++c) {
            const int64_t idx = r * k + c;
            store_f(y, y_t, idx, r32(dec_e4m3(e4m3[idx]) * dec_e8m0(e8m0[r * (k / 32) + c / 32])));
        }
    return 0;
}

// ---- MXFP4 [QuantizedWeight: "E8M0 for native MXFP4"; OCP MX rule as for
// MXFP8]: E2M1 elements packed two per byte (element 2j in the low nibble),
// one E8M0 scale per 32 consecutive elements along the last dimension.
// E = clamp(floor(log2 a) - 2, -127, 127) (2 = the largest E2M1 exponent; an
// infinite a counts as 2^128, a = 0 gives -127), byte E + 127,
// code = E2M1(fl(x * 2^-E)).
int or_mxfp4_quantize(const void* x, int x_t, int64_t rows, int64_t k, uint8_t* packed,
                      uint8_t* e8m0) {
    if (x_t != OR_F32 && x_t != OR_F16 && x_t != OR_BF16) return 1;
    if (rows < 0 || k < 0 || k % 32 != 0) return 1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < k / 32; ++b) {
            const int64_t base = r * k + b * 32;
            double a = 0.0;
            for (int j = 0; j < 32; ++j) {
                double v = std::fabs(load_f(x, x_t, base + j));
                if (v > a) a = v;
            }
            int fl2;
            if (a == 0.0) fl2 = -1000;
            else if (std::isinf(a)) fl2 = 128;
            else { int e; std::frexp(a, &e); fl2 = e - 1; }
            const int E = std::min(std::max(fl2 - 2, -127), 127);
            e8m0[r * (k / 32) + b] = (uint8_t)(E + 127);
            const double inv = std::ldexp(1.0, -E);      // exact power of two
            for (int j = 0; j < 32; j += 2) {
                const uint8_t c0 = enc_e2m1(r32(load_f(x, x_t, base + j) * inv));
                const uint8_t c1 = enc_e2m1(r32(load_f(x, x_t, base + j + 1) * inv));
                packed[(base + j) / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
    return 0;
}

int or_mxfp4_dequantize(const uint8_t* packed, const uint8_t* e8m0, int64_t rows, int64_t k,
                        void* y, int y_t) {
    if (y_t != OR_F32 && y_t != OR_F16 && y_t != OR_BF16) return 1;
    if (rows < 0 || k < 0 || k % 32 != 0) return 1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k; ++c) {
            const int64_t idx = r * k + c;
            const uint8_t byte = packed[idx / 2];
            const uint8_t code = (idx % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            store_f(y, y_t, idx, r32(dec_e2m1(code) * dec_e8m0(e8m0[r * (k / 32) + c / 32])));
        }
    return 0;
}

// ---- FP8 block scaling [smile.llm.quant Fp8BlockGemm / Fp8BlockDequant]:
// E4M3 elements, one f32 scale (the dequantize multiplier, weight_scale_inv)
// per br x bc block; blocks at the bottom / right edges may be partial.
// scale is [ceil(rows/br), ceil(cols/bc)] row-major.
int or_fp8_block_quantize(const void* x, int x_t, int64_t rows, int64_t cols, int64_t br,
                          int64_t bc, uint8_t* e4m3, float* scale) {
    if (x_t != OR_F32 && x_t != OR_F16 && x_t != OR_BF16) return 1;
    if (rows < 0 || cols < 0 || br < 1 || bc < 1) return 1;
    const int64_t nbr = (rows + br - 1) / br, nbc = (cols + bc - 1) / bc;
    for (int64_t I = 0; I < nbr; ++I)
        for (int64_t J = 0; J < nbc; ++J) {
            const int64_t r1 = std::min(rows, (I + 1) * br), c1 = std::min(cols, (J + 1) * bc);
            double a = 0.0;
            for (int64_t r = I * br; r < r1; ++r)
                for (int64_t c = J * bc; c < c1; ++c) {
                    double v = std::fabs(load_f(x, x_t, r * cols + c));
                    if (v > a) a = v;
                }
            float s = (float)(a / 448.0);
            if (s == 0.0f) s = 1.0f;
            scale[I * nbc + J] = s;
            for (int64_t r = I * br; r < r1; ++r)
                for (int64_t c = J * bc; c < c1; ++c)
                    e4m3[r * cols + c] = enc_e4m3(r32(load_f(x, x_t, r * cols + c) / (double)s));
        }
    return 0;
}

int or_fp8_block_dequantize(const uint8_t* e4m3, const float* scale, int64_t rows, int64_t cols,
                            int64_t br, int64_t bc, void* y, int y_t) {
    if (y_t != OR_F32 && y_t != OR_F16 && y_t != OR_BF16) return 1;
    if (rows < 0 || cols < 0 || br < 1 || bc < 1) return 1;
    const int64_t nbc = (cols + bc - 1) / bc;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            store_f(y, y_t, r * cols + c,
                    r32(dec_e4m3(e4m3[r * cols + c]) * (double)scale[(r / br) * nbc + c / bc]));
    return 0;
}

// ---- W8A8 block-FP8 matrix multiply [smile.llm.quant Fp8BlockGemm]: the
// activations a [m, k] are quantized on the fly to E4M3 with one f32 scale
// per 1x128 group (or_fp8_block_quantize with a 1 x 128 block); the weights
// are E4M3 [n, k] with one f32 scale per 128x128 tile (sw is
// [ceil(n/128), ceil(k/128)]); then
//   C[i, j] = sum over k-blocks b of sa[i, b] * sw[j / 128, b] * S(i, j, b),
//   S(i, j, b) = sum over the k in block b of dec(ea[i, k]) * dec(ew[j, k]).
// Every E4M3 value is an integer multiple of 2^-9 below 2^18 such units, so a
// product of two is a multiple of 2^-18 below 2^36 units and a block's 128
// products add exactly in binary64; the two scale products and the sum over
// blocks round in binary64. The pages fix no output precision: C is returned
// in binary64 (a tensor-core f32 accumulation is compared with it within a
// bound). ea / sa, when given, receive the activation codes and scales.
// The product alone, for activations already quantized: ea [m, k] E4M3 codes
// with sa [m, ceil(k/128)] scales.
int or_fp8_block_gemm_codes(const uint8_t* ea, const float* sa, const uint8_t* ew, const float* sw,
                            int64_t m, int64_t n, int64_t k, double* c) {
    if (m < 0 || n < 0 || k < 0) return 1;
    const int64_t nkb = (k + 127) / 128;
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t b = 0; b < nkb; ++b) {
                double blk = 0.0;
                for (int64_t kk = b * 128; kk < std::min(k, (b + 1) * 128); ++kk)
                    blk += dec_e4m3(ea[i * k + kk]) * dec_e4m3(ew[j * k + kk]);
                acc += (double)sa[i * nkb + b] * (double)sw[(j / 128) * nkb + b] * blk;
            }
            c[i * n + j] = acc;
        }
    return 0;
}

int or_fp8_block_gemm(const void* a, int a_t, const uint8_t* ew, const float* sw, int64_t m,
                      int64_t n, int64_t k, double* c, uint8_t* ea_out, float* sa_out) {
    if (a_t != OR_F32 && a_t != OR_F16 && a_t != OR_BF16) return 1;
    if (m < 0 || n < 0 || k < 0) return 1;
    const int64_t nkb = (k + 127) / 128;
    std::vector<uint8_t> ea((size_t)(m * k));
    std::vector<float> sa((size_t)(m * nkb));
    if (or_fp8_block_quantize(a, a_t, m, k, 1, 128, ea.data(), sa.data()) != 0) return 1;
    if (or_fp8_block_gemm_codes(ea.data(), sa.data(), ew, sw, m, n, k, c) != 0) return 1;
    if (ea_out) std::copy(ea.begin(), ea.end(), ea_out);
    if (sa_out) std::copy(sa.begin(), sa.end(), sa_out);
    return 0;
}

// ---- FP8 per-tensor codec [smile.llm.quant Fp8KvCodec: FP8 KV store / load
// with per-tensor scales]: one f32 scale for the whole tensor, the dequantize
// multiplier as in the FP8 block formats: s = fl(amax / 448) (0 -> 1, amax
// ignores NaN) or given; e = E4M3(fl(x / s)); load y = RN_y(fl(dec(e) * s)).
int or_fp8_tensor_quantize(const void* x, int x_t, int64_t n, uint8_t* e4m3, float* s_io,
                           int static_s) {
    if (x_t != OR_F32 && x_t != OR_F16 && x_t != OR_BF16) return 1;
    if (n < 0) return 1;
    float s;
    if (static_s) {
        s = *s_io;
    } else {
        double a;
        or_tensor_amax(x, x_t, n, &a);
        s = (float)(a / 448.0);
        if (s == 0.0f) s = 1.0f;
        *s_io = s;
    }
    for (int64_t i = 0; i < n; ++i) e4m3[i] = enc_e4m3(r32(load_f(x, x_t, i) / (double)s));
    return 0;
}

int or_fp8_tensor_dequantize(const uint8_t* e4m3, float s, int64_t n, void* y, int y_t) {
    if (y_t != OR_F32 && y_t != OR_F16 && y_t != OR_BF16) return 1;
    if (n < 0) return 1;
    for (int64_t i = 0; i < n; ++i) store_f(y, y_t, i, r32(dec_e4m3(e4m3[i]) * (double)s));
    return 0;
}

// ---- Packed weight / scale transpose [QuantizedWeight transpose_for_gemm(_gs),
// transpose_concat_for_gemm_padded]: w [n, k/2] -> w_t [k/2, stride],
// sc [n, k/gs] -> sc_t [k/gs, stride], stride = align_up(n, align), pad = 0.
int64_t or_align_up(int64_t n, int64_t align) { return (n + align - 1) / align * align; }

int or_packed_transpose(const uint8_t* w, const uint8_t* sc, int64_t n, int64_t k, int64_t gs,
                        int64_t align, uint8_t* w_t, uint8_t* sc_t, int64_t* stride_out) {
    if (n < 0 || k < 0 || align < 1 || k % 2 != 0) return 1;
    if (sc && (gs < 1 || k % gs != 0)) return 1;
    const int64_t stride = or_align_up(n, align);
    const int64_t kb = k / 2;
    for (int64_t i = 0; i < kb; ++i)
        for (int64_t j = 0; j < stride; ++j)
            w_t[i * stride + j] = (j < n) ? w[j * kb + i] : 0;
    if (sc) {
        const int64_t ng = k / gs;
        for (int64_t i = 0; i < ng; ++i)
            for (int64_t j = 0; j < stride; ++j)
                sc_t[i * stride + j] = (j < n) ? sc[j * ng + i] : 0;
    }
    *stride_out = stride;
    return 0;
}

// ---- Multi-part transpose [QuantizedWeight transpose_concat_for_gemm,
// transpose_concat_for_gemm_gs, transpose_concat_for_gemm_padded]: parts
// (w_i [n_i, k/2], sc_i [n_i, k/gs]) that share k; part i lands in columns
// [off_i, off_i + n_i) of w_t [k/2, stride] and sc_t [k/gs, stride], with
// off_i = n_0 + ... + n_{i-1} and stride = align_up(n_0 + ... + n_{p-1}, align);
// the pad columns are zero. No parts is an error (the page's rule). sc may be
// null (weights only); then every sc_i is ignored.
int or_packed_transpose_concat(int n_parts, const uint8_t* const* w, const uint8_t* const* sc,
                               const int64_t* n, int64_t k, int64_t gs, int64_t align,
                               uint8_t* w_t, uint8_t* sc_t, int64_t* stride_out) {
    if (n_parts < 1 || k < 0 || align < 1 || k % 2 != 0) return 1;
    if (sc && (gs < 1 || k % gs != 0)) return 1;
    int64_t total = 0;
    for (int p = 0; p < n_parts; ++p) {
        if (n[p] < 0) return 1;
        total += n[p];
    }
    const int64_t stride = or_align_up(total, align);
    const int64_t kb = k / 2, ng = sc ? k / gs : 0;
    for (int64_t i = 0; i < kb * stride; ++i) w_t[i] = 0;
    if (sc) for (int64_t i = 0; i < ng * stride; ++i) sc_t[i] = 0;
    int64_t off = 0;
    for (int p = 0; p < n_parts; ++p) {
        for (int64_t i = 0; i < kb; ++i)
            for (int64_t j = 0; j < n[p]; ++j) w_t[i * stride + off + j] = w[p][j * kb + i];
        if (sc)
            for (int64_t i = 0; i < ng; ++i)
                for (int64_t j = 0; j < n[p]; ++j) sc_t[i * stride + off + j] = sc[p][j * ng + i];
        off += n[p];
    }
    *stride_out = stride;
    return 0;
}

// ---- concat_rows [QuantizedWeight concat_rows]: two NVFP4 weights with the
// same k, [n1, k/2] + [n2, k/2] -> [n1 + n2, k/2] and their E4M3 scales
// (group 16) [n1, k/16] + [n2, k/16] -> [n1 + n2, k/16]. The two per-tensor
// scales must be bit-identical (else an error, 2); the result carries the
// first one.
int or_nvfp4_concat_rows(const uint8_t* w1, const uint8_t* sc1, float s2_1, int64_t n1,
                         const uint8_t* w2, const uint8_t* sc2, float s2_2, int64_t n2, int64_t k,
                         uint8_t* w_out, uint8_t* sc_out, float* s2_out) {
    if (n1 < 0 || n2 < 0 || k < 0 || k % 16 != 0) return 1;
    uint32_t b1, b2;
    std::memcpy(&b1, &s2_1, 4);
    std::memcpy(&b2, &s2_2, 4);
    if (b1 != b2) return 2;
    const int64_t kb = k / 2, ng = k / 16;
    for (int64_t i = 0; i < n1 * kb; ++i) w_out[i] = w1[i];
    for (int64_t i = 0; i < n2 * kb; ++i) w_out[n1 * kb + i] = w2[i];
    for (int64_t i = 0; i < n1 * ng; ++i) sc_out[i] = sc1[i];
    for (int64_t i = 0; i < n2 * ng; ++i) sc_out[n1 * ng + i] = sc2[i];
    *s2_out = s2_1;
    return 0;
}

// ---- predequant_to_fp8 [QuantizedWeight predequant_to_fp8]: an NVFP4 weight
// [n, k] as FP8 E4M3 [n, k] with the per-tensor scale applied: each element is
// the NVFP4 dequantized value fl(e2m1(code) * fl(dec(sb) * s2)) encoded to
// E4M3 (round to nearest even, saturating to +-448, NaN -> 0x7F).
int or_nvfp4_predequant_fp8(const uint8_t* packed, const uint8_t* sc, float s2, int64_t n,
                            int64_t k, uint8_t* e4m3) {
    if (n < 0 || k < 0 || k % 16 != 0) return 1;
    for (int64_t r = 0; r < n; ++r)
        for (int64_t c = 0; c < k; ++c) {
            const int64_t idx = r * k + c;
            const double eff = r32(dec_e4m3(sc[r * (k / 16) + c / 16]) * (double)s2);
            const uint8_t byte = packed[idx / 2];
            const uint8_t code = (idx % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            e4m3[idx] = enc_e4m3(r32(dec_e2m1(code) * eff));
        }
    return 0;
}

}  // extern "C"
