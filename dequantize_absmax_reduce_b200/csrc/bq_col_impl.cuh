// Column groups: the Group granularity (teenygrad granularity.rs, Group{axis,
// group_size}: one scale / zero-point per block of group_size consecutive
// indices along axis) read for a tensor stored [K, N] and grouped along K,
// the GPTQ / AWQ weight layout the baracuda quantize module names. x is
// viewed as [outer, L, inner] around the axis; group (o, b, i) holds the gs
// elements x[o, b*gs + r, i], r < gs, which lie `inner` elements apart;
// scale / zp are [outer, L/gs, inner] row-major.
//
// A CTA of 256 threads works on tiles of gs rows x CW columns of one (o, b).
// Lanes run across the columns (16-byte vectors, so that a warp load covers
// whole 128-byte row segments; single elements when the row width or an
// operand's alignment rules vectors out), lane groups down the rows. Dynamic
// scaling reduces each column's range down the rows (shuffles within a warp,
// shared memory across warps), derives the CW scales once and shares them;
// the codes are then encoded from registers (groups of at most
// COL_RPT * RS rows) or from a second, cached read of the tile. Static
// parameters are read per column from scale / zp.
#pragma once

#include <type_traits>

#include "bq_map_ops.cuh"

namespace bq {

// Range records of every column group (bq_group_range): the dynamic
// kernel's reduction with the two records written in place of the codes.
constexpr int COL_OP_RANGE = 16;

struct ColArgs {
    const void* a;          // x, q or dy
    const void* b;          // dy (STE backwards)
    const unsigned long long* ranges_in;   // FROM_RANGE: parameters derived from these records
    unsigned long long* ranges_out;        // COL_OP_RANGE: the records written
    int64_t inner, gs;      // row width (columns) and group length (rows)
    int64_t n_ct;           // column tiles per row
    int64_t n_tiles;        // outer * (L / gs) * n_ct
    IntCfg cfg;
    const float* scale_in;  // static parameters
    const void* zp_in;
    float* scale_out;       // dynamic parameters
    uint8_t* zp_out;
    void* out;              // q, y or dx
};

constexpr int COL_RPT = 4;  // rows a thread loads before computing

template <int W> struct ColGeom {
    static constexpr int CVN = (W == 1) ? 32 : 8;   // vectors across a tile row
    static constexpr int RS = 256 / CVN;            // lanes down the rows
    static constexpr int CW = CVN * W;              // columns per tile
    static constexpr int NW = 8;                    // warps
};

// One thread's W consecutive elements of a row: a 16-byte vector, or one
// element kept widened.
template <class T, int W> struct ColRaw { U4 u; };
template <class T> struct ColRaw<T, 1> { typename Traits<T>::Acc v; };

template <class T, int W>
__device__ __forceinline__ ColRaw<T, W> col_fetch(const T* p, bool cached) {
    ColRaw<T, W> r;
    if constexpr (W == 1) r.v = ld1<T>(p);
    else r.u = cached ? ld16_nc(p) : ld16_stream(p);
    return r;
}
template <class T, int W>
__device__ __forceinline__ void col_vals(const ColRaw<T, W>& r, typename Traits<T>::Acc (&v)[W]) {
    if constexpr (W == 1) v[0] = r.v;
    else load_vec<T>(r.u, v);
}
// Element k of a thread's W elements.
template <class T, int W>
__device__ __forceinline__ typename Traits<T>::Acc col_elem(const ColRaw<T, W>& r, int k) {
    if constexpr (W == 1) {
        return r.v;
    } else if constexpr (sizeof(T) == 2) {
        const uint32_t w = (k >> 1) == 0 ? r.u.x : (k >> 1) == 1 ? r.u.y : (k >> 1) == 2 ? r.u.z : r.u.w;
        float lo, hi;
        if constexpr (std::is_same<T, __nv_bfloat16>::value) unpack_bf16x2(w, lo, hi);
        else unpack_f16x2(w, lo, hi);
        return (k & 1) ? hi : lo;
    } else if constexpr (sizeof(T) == 4) {
        return __uint_as_float(k == 0 ? r.u.x : k == 1 ? r.u.y : k == 2 ? r.u.z : r.u.w);
    } else {
        return k == 0 ? __hiloint2double((int)r.u.y, (int)r.u.x) : __hiloint2double((int)r.u.w, (int)r.u.z);
    }
}
// One row's W outputs, packed as they are produced: code bytes (CODES), or
// values narrowed to T in pairs (16-bit T) or kept (f32 / f64).
template <class T, int W, bool CODES> struct ColOut {
    using Acc = typename Traits<T>::Acc;
    static constexpr bool HALF = sizeof(T) == 2 && W > 1;
    uint32_t cw[(W + 3) / 4];
    uint32_t h[HALF ? W / 2 : 1];
    Acc v[HALF ? 1 : W];
    float pend;
    __device__ __forceinline__ void set_code(int k, uint32_t code) {
        const uint32_t b = (code & 0xFFu) << (8 * (k % 4));
        cw[k / 4] = (k % 4 == 0) ? b : (cw[k / 4] | b);
    }
    __device__ __forceinline__ void set(int k, Acc o) {
        if constexpr (HALF) {
            if ((k & 1) == 0) {
                pend = o;
            } else {
                if constexpr (std::is_same<T, __nv_bfloat16>::value) h[k >> 1] = pack_bf16x2(pend, o);
                else h[k >> 1] = pack_f16x2(pend, o);
            }
        } else {
            v[k] = o;
        }
    }
    __device__ __forceinline__ void store_codes(uint8_t* q, int packed) const {
        if (packed) {
            if constexpr (W == 8) st4(q, nib_pack4(cw[0]) | (nib_pack4(cw[1]) << 16));
            else if constexpr (W == 4) *reinterpret_cast<unsigned short*>(q) = (unsigned short)nib_pack4(cw[0]);
            else if constexpr (W == 2) q[0] = (uint8_t)nib_pack4(cw[0]);
            else q[0] = (uint8_t)cw[0];          // single codes: never packed
        } else if constexpr (W == 8) {
            st8(q, cw[0], cw[1]);
        } else if constexpr (W == 4) {
            st4(q, cw[0]);
        } else {
#pragma unroll
            for (int i = 0; i < W; ++i) q[i] = (uint8_t)(cw[0] >> (8 * i));
        }
    }
    __device__ __forceinline__ void store(T* p) const {
        if constexpr (W == 1) {
            *p = to_out<T>(v[0]);
        } else if constexpr (HALF) {
            st16(p, U4{h[0], h[1], h[2], h[3]});
        } else {
            st16(p, pack_vec<T>(v));
        }
    }
};

// A column's parameters as a group state, from the scale, its correctly
// rounded reciprocal and the zero-point; the STE mask is decided per element
// from the exact quotient (no interval thresholds).
__device__ __forceinline__ GState col_state(const IntCfg& c, float s, float y, int zp) {
    GState st;
    st.seg = 0;
    st.s = s;
    st.zp = zp;
    st.R.s = s;
    st.R.y = y;
    const float m = fabsf(s);
    st.R.fast = (m >= 0x1p-64f) && (m <= 0x1p64f);
    st.ip = make_int_params(c.qmin, c.qmax, zp);
    st.x_lo = st.x_hi = 0.0f;
    st.mfast = false;
    st.fast = false;
    return st;
}

template <class A> __device__ __forceinline__ A acc_max(A a, A b) {
    if constexpr (std::is_same<A, double>::value) return fmax(a, b); else return fmaxf(a, b);
}
template <class A> __device__ __forceinline__ A acc_min(A a, A b) {
    if constexpr (std::is_same<A, double>::value) return fmin(a, b); else return fminf(a, b);
}

// Quantize / fake-quantize of one element whose quotient is known to be
// exact through the reciprocal chain (dynamic scaling: x lies in its group's
// range and the scale is in the fast range); a NaN quotient clamps to qmin.
template <int OP, bool RHAZ>
__device__ __forceinline__ float col_quant_chain(float x, const GState& st, uint32_t* code) {
    const float t = rounded_of<RHAZ>(div_chain(x, st.R), st.ip);
    *code = code_from_rounded(t, st.ip.zp);
    if constexpr (OP == OP_FAKE) return dequant_from_rounded(t, st.s);
    return 0.0f;
}

// OP: OP_QUANT / OP_FAKE (DYN: scale from each group's range, else static),
// OP_QBWD / OP_FBWD / OP_DBWD (static), OP_DEQ (codes in, T out).
// RES: the whole group fits one load batch (gs <= COL_RPT * RS), so dynamic
// scaling encodes from registers instead of re-reading the tile.
template <class T, int OP, bool DYN, bool RHAZ, int W, bool RES>
__global__ void __launch_bounds__(256) k_col(ColArgs a) {
    using Acc = typename Traits<T>::Acc;
    using G = ColGeom<W>;
    constexpr bool WIDE = std::is_same<Acc, double>::value;
    constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    constexpr int CVN = G::CVN, RS = G::RS, CW = G::CW, NW = G::NW;
    constexpr bool NEEDR = !WIDE && OP != OP_DEQ && OP != OP_DBWD;   // reciprocal used
    __shared__ Acc red_hi[DYN ? NW : 1][CW], red_lo[DYN ? NW : 1][CW];
    // The tile's column parameters (dynamic scaling), double-buffered by tile
    // parity: a thread writing tile t+2's entries has passed a barrier that
    // every reader of tile t's entries reached after reading them.
    __shared__ float col_s[DYN ? 2 : 1][CW], col_y[DYN ? 2 : 1][CW];
    __shared__ int col_z[DYN ? 2 : 1][CW];

    const int tid = threadIdx.x;
    const int cv = tid % CVN, rl = tid / CVN;
    const int wid = tid >> 5, lane = tid & 31;
    const int64_t inner = a.inner, gs = a.gs;
    int par = 0;

    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, par ^= 1) {
        const int64_t ct = tile % a.n_ct;
        const int64_t ob = tile / a.n_ct;                 // o * (L / gs) + b
        const int64_t c0 = ct * CW + (int64_t)cv * W;     // this thread's first column
        const bool col_ok = c0 < inner;                   // W columns (inner % W == 0 when W > 1)
        const int64_t row0 = ob * gs;                     // first row of the block, as o*L + b*gs

        ColRaw<T, W> raw[COL_RPT];

        if constexpr (DYN) {
            // ---- range of each of this thread's columns over its rows
            Acc hi[W], lo[W];
#pragma unroll
            for (int k = 0; k < W; ++k) hi[k] = lo[k] = (Acc)0;
            for (int64_t r0 = rl; r0 < gs; r0 += (int64_t)COL_RPT * RS) {
#pragma unroll
                for (int j = 0; j < COL_RPT; ++j) {
                    const int64_t r = r0 + (int64_t)j * RS;
                    if (col_ok && r < gs)
                        raw[j] = col_fetch<T, W>((const T*)a.a + (row0 + r) * inner + c0, !RES);
                }
#pragma unroll
                for (int j = 0; j < COL_RPT; ++j) {
                    const int64_t r = r0 + (int64_t)j * RS;
                    if (col_ok && r < gs) {
                        Acc v[W];
                        col_vals<T, W>(raw[j], v);
#pragma unroll
                        for (int k = 0; k < W; ++k) {          // NaN skipped by fmax / fmin
                            hi[k] = acc_max(hi[k], v[k]);
                            lo[k] = acc_min(lo[k], v[k]);
                        }
                    }
                }
            }
            // ---- reduce down the rows: lanes of one column within the warp, then warps
#pragma unroll
            for (int o = CVN; o < 32; o <<= 1) {
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    hi[k] = acc_max(hi[k], __shfl_xor_sync(0xffffffffu, hi[k], o));
                    lo[k] = acc_min(lo[k], __shfl_xor_sync(0xffffffffu, lo[k], o));
                }
            }
            if (lane < CVN) {
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    red_hi[wid][cv * W + k] = hi[k];
                    red_lo[wid][cv * W + k] = lo[k];
                }
            }
            __syncthreads();
            if (tid < CW) {
                Acc h = red_hi[0][tid], l = red_lo[0][tid];
#pragma unroll
                for (int w = 1; w < NW; ++w) {
                    h = acc_max(h, red_hi[w][tid]);
                    l = acc_min(l, red_lo[w][tid]);
                }
                float s;
                int z;
                if constexpr (WIDE) {
                    const GroupD g = derive_d(h, -l, a.cfg);
                    s = g.s; z = g.zp;
                } else {
                    const GroupF g = derive_f(h, -l, a.cfg);
                    s = g.s; z = g.zp;
                }
                col_s[par][tid] = s;
                col_z[par][tid] = z;
                if constexpr (NEEDR) col_y[par][tid] = __frcp_rn(s);
                const int64_t c = ct * CW + tid;
                if (c < inner) {
                    if constexpr (OP == COL_OP_RANGE) {
                        // max(0, max x) and max(0, -min x) as non-negative IEEE
                        // bits (a zero of either sign becomes +0), so that records
                        // combine with an integer MAX
                        a.ranges_out[2 * (ob * inner + c)] = range_bits(h + (Acc)0);
                        a.ranges_out[2 * (ob * inner + c) + 1] = range_bits((Acc)0 - l);
                    } else {
                        a.scale_out[ob * inner + c] = s;
                        if (a.zp_out) a.zp_out[ob * inner + c] = (uint8_t)z;
                    }
                }
            }
            __syncthreads();
        }
        if constexpr (OP == COL_OP_RANGE) continue;
        if (!col_ok) continue;      // no barrier below this point

        // ---- element pass over the block's rows, one column at a time (one
        // column's parameters live at once), outputs packed as they come
        const bool reuse = DYN && RES;
        for (int64_t r0 = rl; r0 < gs; r0 += (int64_t)COL_RPT * RS) {
            ColRaw<T, W> rb[TWO ? COL_RPT : 1];
            uint32_t cq[(OP == OP_DEQ) ? COL_RPT : 1][(W + 3) / 4];
            if (!reuse) {
#pragma unroll
                for (int j = 0; j < COL_RPT; ++j) {
                    const int64_t r = r0 + (int64_t)j * RS;
                    if (r >= gs) continue;
                    const int64_t e = (row0 + r) * inner + c0;
                    if constexpr (OP == OP_DEQ) {
                        ld_codes<W>(code_ptr((const uint8_t*)a.a, e, a.cfg.packed), a.cfg.packed,
                                    a.cfg.q_signed, cq[j]);
                    } else {
                        raw[j] = col_fetch<T, W>((const T*)a.a + e, false);
                        if constexpr (TWO) rb[j] = col_fetch<T, W>((const T*)a.b + e, false);
                    }
                }
            }
            ColOut<T, W, OP == OP_QUANT> res[COL_RPT];
#pragma unroll
            for (int k = 0; k < W; ++k) {
                const int c = cv * W + k;
                float sk, yk = 0.0f;
                int zk;
                if constexpr (DYN) {
                    sk = col_s[par][c];
                    if constexpr (NEEDR) yk = col_y[par][c];
                    zk = col_z[par][c];
                } else if (a.ranges_in) {
                    // Parameters from range records (FROM_RANGE), written out by
                    // the first lane of each column.
                    const int64_t g = ob * inner + c0 + k;
                    Acc h, n;
                    range_from_bits(a.ranges_in[2 * g], h);
                    range_from_bits(a.ranges_in[2 * g + 1], n);
                    if constexpr (WIDE) {
                        const GroupD gp = derive_d(h, n, a.cfg);
                        sk = gp.s; zk = gp.zp;
                    } else {
                        const GroupF gp = derive_f(h, n, a.cfg);
                        sk = gp.s; zk = gp.zp;
                    }
                    if constexpr (NEEDR) yk = __frcp_rn(sk);
                    if (rl == 0 && r0 == rl) {
                        a.scale_out[g] = sk;
                        if (a.zp_out) a.zp_out[g] = (uint8_t)zk;
                    }
                } else {
                    // Static parameters: each thread reads its own columns' (the
                    // rows of a block share them; L1 / L2 serve the repeats).
                    const int64_t g = ob * inner + c0 + k;
                    sk = __ldg(a.scale_in + g);
                    if constexpr (NEEDR) yk = __frcp_rn(sk);
                    zk = (OP == OP_DBWD || a.cfg.symmetric) ? 0 : load_zp(a.zp_in, g, a.cfg.q_signed);
                }
                const GState stk = col_state(a.cfg, sk, yk, zk);
#pragma unroll
                for (int j = 0; j < COL_RPT; ++j) {
                    if (r0 + (int64_t)j * RS >= gs) continue;
                    if constexpr (OP == OP_DEQ) {
                        const uint32_t b = (cq[j][k / 4] >> (8 * (k % 4))) & 0xFFu;
                        const int qv = a.cfg.q_signed ? (int)(int8_t)b : (int)b;
                        if constexpr (WIDE) res[j].set(k, (double)(qv - stk.zp) * (double)stk.s);
                        else res[j].set(k, __fmul_rn((float)(qv - stk.zp), stk.s));
                    } else {
                        const Acc xa = col_elem<T, W>(raw[j], k);
                        const Acc xb = TWO ? col_elem<T, W>(rb[TWO ? j : 0], k) : (Acc)0;
                        uint32_t code = 0;
                        Acc o;
                        if constexpr (WIDE) {
                            o = elem_d<OP, RHAZ>(xa, xb, stk, &code);
                        } else if constexpr (DYN) {
                            o = stk.R.fast ? col_quant_chain<OP, RHAZ>(xa, stk, &code)
                                           : elem_f<OP, RHAZ>(xa, 0.0f, stk, &code);
                        } else {
                            o = elem_f<OP, RHAZ>(xa, xb, stk, &code);
                        }
                        if constexpr (OP == OP_QUANT) res[j].set_code(k, code);
                        else res[j].set(k, o);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < COL_RPT; ++j) {
                const int64_t r = r0 + (int64_t)j * RS;
                if (r >= gs) continue;
                const int64_t e = (row0 + r) * inner + c0;
                if constexpr (OP == OP_QUANT) res[j].store_codes(code_ptr((uint8_t*)a.out, e, a.cfg.packed), a.cfg.packed);
                else res[j].store((T*)a.out + e);
            }
        }
    }
}

// Grid of at most one wave of kernel K (occupancy queried once per kernel).
template <auto K>
static unsigned col_grid(int64_t tiles) {
    static const int bps = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, K, 256, 0) != cudaSuccess || n < 1) {
            (void)cudaGetLastError();
            n = 1;
        }
        return n;
    }();
    const int64_t cap = (int64_t)sm_count() * bps;
    if (tiles < 1) tiles = 1;
    return (unsigned)(tiles < cap ? tiles : cap);
}

template <class T, int OP, bool DYN, bool RHAZ, int W, bool RES>
static cudaError_t col_launch_k(const ColArgs& a, cudaStream_t st) {
    constexpr auto K = k_col<T, OP, DYN, RHAZ, W, RES>;
    K<<<col_grid<K>(a.n_tiles), 256, 0, st>>>(a);
    return cudaGetLastError();
}

template <class T, int OP, bool DYN, bool RHAZ, int W>
static cudaError_t col_launch_w(const ColArgs& a, cudaStream_t st) {
    if constexpr (DYN) {
        if (a.gs <= (int64_t)COL_RPT * ColGeom<W>::RS) return col_launch_k<T, OP, DYN, RHAZ, W, true>(a, st);
    }
    return col_launch_k<T, OP, DYN, RHAZ, W, false>(a, st);
}

template <class T, int OP, bool DYN, bool RHAZ>
static cudaError_t col_launch_r(ColArgs a, bool vec, cudaStream_t st) {
    constexpr int V = Traits<T>::VEC;
    if (vec) {
        a.n_ct = (a.inner + ColGeom<V>::CW - 1) / ColGeom<V>::CW;
        a.n_tiles *= a.n_ct;
        return col_launch_w<T, OP, DYN, RHAZ, V>(a, st);
    }
    a.n_ct = (a.inner + ColGeom<1>::CW - 1) / ColGeom<1>::CW;
    a.n_tiles *= a.n_ct;
    return col_launch_w<T, OP, DYN, RHAZ, 1>(a, st);
}

// a.n_tiles holds outer * (L / gs) on entry; the launcher multiplies in the
// column tiles of the chosen width.
template <class T>
static cudaError_t col_entry(int op, int dyn, const ColArgs& a, bool vec, cudaStream_t st) {
    const bool rhaz = a.cfg.rhaz != 0;
    switch (op) {
        case OP_QUANT:
            if (dyn) return rhaz ? col_launch_r<T, OP_QUANT, true, true>(a, vec, st)
                                 : col_launch_r<T, OP_QUANT, true, false>(a, vec, st);
            return rhaz ? col_launch_r<T, OP_QUANT, false, true>(a, vec, st)
                        : col_launch_r<T, OP_QUANT, false, false>(a, vec, st);
        case OP_FAKE:
            if (dyn) return rhaz ? col_launch_r<T, OP_FAKE, true, true>(a, vec, st)
                                 : col_launch_r<T, OP_FAKE, true, false>(a, vec, st);
            return rhaz ? col_launch_r<T, OP_FAKE, false, true>(a, vec, st)
                        : col_launch_r<T, OP_FAKE, false, false>(a, vec, st);
        case OP_QBWD:
            return rhaz ? col_launch_r<T, OP_QBWD, false, true>(a, vec, st)
                        : col_launch_r<T, OP_QBWD, false, false>(a, vec, st);
        case OP_FBWD:
            return rhaz ? col_launch_r<T, OP_FBWD, false, true>(a, vec, st)
                        : col_launch_r<T, OP_FBWD, false, false>(a, vec, st);
        case OP_DEQ: return col_launch_r<T, OP_DEQ, false, false>(a, vec, st);
        case OP_DBWD: return col_launch_r<T, OP_DBWD, false, false>(a, vec, st);
        case COL_OP_RANGE: return col_launch_r<T, COL_OP_RANGE, true, false>(a, vec, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace bq

#define BQ_COL_ENTRY(TYPE, NAME)                                                               \
    cudaError_t col_groups_##NAME(int op, int dyn, const ColArgs& a, bool vec, cudaStream_t st) { \
        return col_entry<TYPE>(op, dyn, a, vec, st);                                            \
    }
