// Integer (s8 / u8) quantize, dequantize, fake-quantize and Straight-Through
// Estimator kernels for every granularity (baracuda_kernels::quantize module
// index: per_tensor, per_channel, per_token, per_group and their backwards;
// teenygrad granularity.rs for the groups).
//
// Every granularity reaches these kernels as a view of n_seg contiguous
// groups of G elements: with x viewed as [outer, L, inner], Group{axis, gs}
// holds axis indices [g*gs, (g+1)*gs) and every inner index, which is one
// contiguous run of gs*inner elements.
//
// Kernels:
//   k_int_dyn_warp / k_int_dyn_cta  one HBM pass for dynamic scales: a team
//       of lanes (part of a warp, a warp, or a CTA) holds a whole group in
//       registers, reduces its range, derives scale / zero-point and writes
//       the codes. 16-byte streaming loads.
//   k_int_map  element-wise with per-group parameters: static scales,
//       scales derived from range records (second pass of the two-pass path),
//       dequantize, and the three backwards.
//   k_tensor_range / k_seg_range  range records (max(0, max x),
//       max(0, -min x)) with integer atomicMax on the IEEE bits.
#include <type_traits>

#include "bq_device.cuh"
#include "bq_internal.h"
#include "bq_quant_ops.cuh"
#include "bq_map_ops.cuh"

namespace bq {

// ------------------------------------------------------------ dynamic, warp
struct DynArgs {
    const void* x;
    int64_t n_seg;
    int G;          // elements per group (multiple of VEC)
    int team;       // lanes per group (power of two <= 32), warp kernels
    IntCfg cfg;
    uint8_t* q;
    void* y;
    float* scale;
    uint8_t* zp;
};

// Codes (QUANT) or fake-quantized values (FAKE) of one 16-byte vector.
template <class T, int OP, bool FAST>
__device__ __forceinline__ void emit_vec(const U4& raw, const Recip& R, const IntParams& ip,
                                         int64_t off, const DynArgs& a) {
    constexpr int VEC = Traits<T>::VEC;
    float v[VEC];
    load_vec<T>(raw, v);
    float t[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        const float qv = FAST ? div_chain(v[i], R) : div_slow(v[i], R.s);
        t[i] = rounded_rne(qv, ip);
    }
    if constexpr (OP == OP_QUANT) {
        uint32_t cw[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) cw[i] = code_from_rounded(t[i], ip.zp);
        st_codes<VEC>(code_ptr(a.q, off, a.cfg.packed), cw, a.cfg.packed);
    } else {
        float o[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) o[i] = dequant_from_rounded(t[i], R.s);
        st16((T*)a.y + off, pack_vec<T>(o));
    }
}

template <class T>
__device__ __forceinline__ void range_vec(const U4& raw, bool sym, float& hi, float& nlo) {
    constexpr int VEC = Traits<T>::VEC;
    float v[VEC];
    load_vec<T>(raw, v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        if (sym) {
            hi = fmaxf(hi, fabsf(v[i]));
        } else {
            hi = fmaxf(hi, v[i]);
            nlo = fmaxf(nlo, -v[i]);
        }
    }
}

// Groups of up to team*NV vectors: `a.team` lanes per group, NV vectors per
// lane, SEGS groups per team per iteration (all their loads issued first).
template <class T, int OP, int NV, int SEGS, bool SYM>
__global__ void __launch_bounds__(256) k_int_dyn_warp(DynArgs a) {
    constexpr int VEC = Traits<T>::VEC;
    const T* __restrict__ x = (const T*)a.x;
    const int team = a.team;
    const int tpw = 32 / team;
    const int lane = threadIdx.x & 31;
    const int tm = lane / team;
    const int l = lane % team;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t per_chunk = (int64_t)SEGS * tpw;
    const int64_t n_chunks = (a.n_seg + per_chunk - 1) / per_chunk;

    for (int64_t c = gwarp; c < n_chunks; c += nwarps) {
        U4 raw[SEGS][NV];
#pragma unroll
        for (int r = 0; r < SEGS; ++r) {
            const int64_t seg = c * per_chunk + (int64_t)r * tpw + tm;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int e = (j * team + l) * VEC;
                if (seg < a.n_seg && e < a.G) raw[r][j] = ld16_nc(x + seg * a.G + e);
                else raw[r][j] = U4{0u, 0u, 0u, 0u};
            }
        }
#pragma unroll
        for (int r = 0; r < SEGS; ++r) {
            const int64_t seg = c * per_chunk + (int64_t)r * tpw + tm;
            float hi = 0.0f, nlo = 0.0f;
#pragma unroll
            for (int j = 0; j < NV; ++j) range_vec<T>(raw[r][j], SYM, hi, nlo);
            for (int o = team / 2; o > 0; o >>= 1) {
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
                if (!SYM) nlo = fmaxf(nlo, __shfl_xor_sync(0xffffffffu, nlo, o));
            }
            const GroupF g = derive_f(hi, nlo, a.cfg);
            const bool seg_ok = seg < a.n_seg;
            if (seg_ok && l == 0) {
                a.scale[seg] = g.s;
                if (a.zp) a.zp[seg] = (uint8_t)g.zp;
            }
            const IntParams ip = make_int_params(a.cfg.qmin, a.cfg.qmax, SYM ? 0 : g.zp);
            const Recip R = make_recip(g.s);
            if (R.fast) {
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    const int e = (j * team + l) * VEC;
                    if (seg_ok && e < a.G) emit_vec<T, OP, true>(raw[r][j], R, ip, seg * a.G + e, a);
                }
            } else {
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    const int e = (j * team + l) * VEC;
                    if (seg_ok && e < a.G) emit_vec<T, OP, false>(raw[r][j], R, ip, seg * a.G + e, a);
                }
            }
        }
    }
}

// A CTA of 256 threads per group, NV vectors per thread; while one group is
// reduced and written, the loads of the CTA's next group are in flight.
template <class T, int OP, int NV, bool SYM>
__device__ __forceinline__ void cta_load(const T* __restrict__ x, int64_t seg, int G, U4 (&raw)[NV]) {
    constexpr int VEC = Traits<T>::VEC;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int e = (j * 256 + (int)threadIdx.x) * VEC;
        raw[j] = (e < G) ? ld16_stream(x + seg * G + e) : U4{0u, 0u, 0u, 0u};
    }
}

template <class T, int OP, int NV, bool SYM>
__device__ __forceinline__ void cta_group(const U4 (&raw)[NV], int64_t seg, int par,
                                          float (*sh)[2][8], const DynArgs& a) {
    constexpr int VEC = Traits<T>::VEC;
    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
    float hi = 0.0f, nlo = 0.0f;
#pragma unroll
    for (int j = 0; j < NV; ++j) range_vec<T>(raw[j], SYM, hi, nlo);
    hi = warp_max(hi);
    if (!SYM) nlo = warp_max(nlo);
    if (lane == 0) { sh[par][0][wid] = hi; sh[par][1][wid] = nlo; }
    __syncthreads();
    hi = sh[par][0][0];
    nlo = sh[par][1][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        hi = fmaxf(hi, sh[par][0][w]);
        if (!SYM) nlo = fmaxf(nlo, sh[par][1][w]);
    }
    if (SYM) nlo = 0.0f;
    const GroupF g = derive_f(hi, nlo, a.cfg);
    if (tid == 0) {
        a.scale[seg] = g.s;
        if (a.zp) a.zp[seg] = (uint8_t)g.zp;
    }
    const IntParams ip = make_int_params(a.cfg.qmin, a.cfg.qmax, SYM ? 0 : g.zp);
    const Recip R = make_recip(g.s);
    if (R.fast) {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = (j * 256 + tid) * VEC;
            if (e < a.G) emit_vec<T, OP, true>(raw[j], R, ip, seg * a.G + e, a);
        }
    } else {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = (j * 256 + tid) * VEC;
            if (e < a.G) emit_vec<T, OP, false>(raw[j], R, ip, seg * a.G + e, a);
        }
    }
}

template <class T, int OP, int NV, bool SYM>
__global__ void __launch_bounds__(256) k_int_dyn_cta(DynArgs a) {
    __shared__ float sh[2][2][8];          // [parity][hi / nlo][warp]
    const T* __restrict__ x = (const T*)a.x;
    const int64_t G = gridDim.x;
    U4 A[NV], B[NV];
    int64_t seg = blockIdx.x;
    if (seg < a.n_seg) cta_load<T, OP, NV, SYM>(x, seg, a.G, A);
    for (; seg < a.n_seg; seg += 2 * G) {
        const int64_t s1 = seg + G, s2 = seg + 2 * G;
        if (s1 < a.n_seg) cta_load<T, OP, NV, SYM>(x, s1, a.G, B);
        cta_group<T, OP, NV, SYM>(A, seg, 0, sh, a);
        if (s2 < a.n_seg) cta_load<T, OP, NV, SYM>(x, s2, a.G, A);
        if (s1 < a.n_seg) cta_group<T, OP, NV, SYM>(B, s1, 1, sh, a);
    }
}

// Items of W elements (one 16-byte vector, or one element); each warp takes
// contiguous chunks of 32*U items, lane l the items l, l+32, ..., so every
// load instruction is coalesced and a lane's items rarely change group. All
// U items' loads are issued before any of them is computed.
template <class T, int OP, int PSRC, bool VECP, bool RHAZ>
__global__ void __launch_bounds__(256) k_int_map(MapArgs a) {
    using Acc = typename Traits<T>::Acc;
    constexpr bool WIDE = std::is_same<Acc, double>::value;
    constexpr int W = VECP ? Traits<T>::VEC : 1;
    constexpr int U = (OP == OP_DEQ) ? 8 : 4;
    constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_items = a.numel / W;
    const int64_t n_chunks = (n_items + 32 * U - 1) / (32 * U);
    GState st;
    st.seg = -1;
    for (int64_t c = gwarp; c < n_chunks; c += nwarps) {
        const int64_t it0 = c * 32 * U + lane;
        if constexpr (OP == OP_DEQ) {
            // codes: W bytes per item
            uint32_t cw[U][(W + 3) / 4];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t it = it0 + (int64_t)u * 32;
                if (it < n_items)
                    ld_codes<W>(code_ptr((const uint8_t*)a.a, it * W, a.cfg.packed), a.cfg.packed,
                                a.cfg.q_signed, cw[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t it = it0 + (int64_t)u * 32;
                if (it >= n_items) continue;
                const int64_t e0 = it * W;
                const int64_t seg = a.use_fd ? (int64_t)fdiv((uint32_t)e0, a.fd) : e0 / a.G;
                if (seg != st.seg) load_group<T, PSRC, false, RHAZ>(a, seg, false, st);
                Acc o[W];
                if constexpr (!WIDE && (W == 8 || W == 4)) {
#pragma unroll
                    for (int i = 0; i < W; ++i) o[i] = deq_code_f(cw[u][i / 4], i % 4, st, a.cfg.q_signed);
                } else {
#pragma unroll
                    for (int i = 0; i < W; ++i) {
                        const uint32_t b = (cw[u][0] >> (8 * i)) & 0xFFu;
                        const int qv = a.cfg.q_signed ? (int)(int8_t)b : (int)b;
                        if constexpr (WIDE) o[i] = (double)(qv - st.zp) * (double)st.s;
                        else o[i] = __fmul_rn((float)(qv - st.zp), st.s);
                    }
                }
                if constexpr (VECP) st16((T*)a.out + e0, pack_vec<T>(o));
                else ((T*)a.out)[e0] = to_out<T>(o[0]);
            }
        } else {
            U4 ra[U], rb[TWO ? U : 1];
            Acc sa[U], sb[TWO ? U : 1];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t it = it0 + (int64_t)u * 32;
                if (it < n_items) {
                    if constexpr (VECP) {
                        ra[u] = ld16_stream((const T*)a.a + it * W);
                        if constexpr (TWO) rb[u] = ld16_stream((const T*)a.b + it * W);
                    } else {
                        sa[u] = ld1<T>((const T*)a.a + it);
                        if constexpr (TWO) sb[u] = ld1<T>((const T*)a.b + it);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t it = it0 + (int64_t)u * 32;
                if (it >= n_items) continue;
                const int64_t e0 = it * W;
                const int64_t seg = a.use_fd ? (int64_t)fdiv((uint32_t)e0, a.fd) : e0 / a.G;
                if (seg != st.seg) load_group<T, PSRC, (OP == OP_QBWD || OP == OP_FBWD), RHAZ>(a, seg, e0 == seg * a.G, st);
                Acc xa[W], xb[W];
                if constexpr (VECP) {
                    load_vec<T>(ra[u], xa);
                    if constexpr (TWO) load_vec<T>(rb[u], xb);
                } else {
                    xa[0] = sa[u];
                    if constexpr (TWO) xb[0] = sb[u];
                }
                Acc o[W];
                uint32_t cw[W];
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    if constexpr (WIDE) o[i] = elem_d<OP, RHAZ>(xa[i], TWO ? xb[i] : 0.0, st, &cw[i]);
                    else o[i] = elem_f<OP, RHAZ>(xa[i], TWO ? xb[i] : 0.0f, st, &cw[i]);
                }
                if constexpr (OP == OP_QUANT) {
                    st_codes<W>(code_ptr((uint8_t*)a.out, e0, a.cfg.packed), cw, a.cfg.packed);
                } else {
                    if constexpr (VECP) st16((T*)a.out + e0, pack_vec<T>(o));
                    else ((T*)a.out)[e0] = to_out<T>(o[0]);
                }
            }
        }
    }
}

// ------------------------------------------------------------ ranges
template <class Acc>
__device__ __forceinline__ void acc_range(Acc v, bool sym, Acc& hi, Acc& nlo) {
    if (sym) {
        hi = fmax(hi, fabs(v));
    } else {
        hi = fmax(hi, v);
        nlo = fmax(nlo, -v);
    }
}

// Whole tensor: grid-stride 16-byte loads, CTA reduction, one atomicMax per
// CTA and slot. Unaligned head / tail elements go through scalar loads.
template <class T>
__global__ void __launch_bounds__(512) k_tensor_range(const T* __restrict__ x, int64_t n,
                                                      int64_t head, int sym,
                                                      unsigned long long* rec) {
    using Acc = typename Traits<T>::Acc;
    constexpr int VEC = Traits<T>::VEC;
    constexpr int UNR = 4;
    __shared__ Acc sh[2][16];
    Acc hi = 0, nlo = 0;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    if (tid < head) acc_range<Acc>(ld1<T>(x + tid), sym, hi, nlo);
    const T* body = x + head;
    const int64_t nb = n - head;
    const int64_t nvec = nb / VEC;
    int64_t i = tid;
    for (; i + (UNR - 1) * nthr < nvec; i += UNR * nthr) {
        U4 r[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) r[u] = ld16_stream(body + (i + u * nthr) * VEC);
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            Acc v[VEC];
            load_vec<T>(r[u], v);
#pragma unroll
            for (int k = 0; k < VEC; ++k) acc_range<Acc>(v[k], sym, hi, nlo);
        }
    }
    for (; i < nvec; i += nthr) {
        Acc v[VEC];
        load_vec<T>(ld16_stream(body + i * VEC), v);
#pragma unroll
        for (int k = 0; k < VEC; ++k) acc_range<Acc>(v[k], sym, hi, nlo);
    }
    const int64_t tail0 = nvec * VEC;
    if (tid < nb - tail0) acc_range<Acc>(ld1<T>(body + tail0 + tid), sym, hi, nlo);

    hi = warp_max(hi);
    nlo = warp_max(nlo);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { sh[0][w] = hi; sh[1][w] = nlo; }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int nw = blockDim.x >> 5;
        for (int k = 1; k < nw; ++k) { hi = fmax(hi, sh[0][k]); nlo = fmax(nlo, sh[1][k]); }
        atomicMax(rec, range_bits(hi));
        if (!sym) atomicMax(rec + 1, range_bits(nlo));
    }
}

// Many groups: the units (group, slice of UL elements) are split into one
// contiguous block per warp; a warp flushes its running range with
// atomicMax whenever the group changes and at the end.
template <class T, bool VECP>
__global__ void __launch_bounds__(256) k_seg_range(const T* __restrict__ x, int64_t n_seg,
                                                   int64_t G, int64_t upg, int64_t per_warp,
                                                   int sym, unsigned long long* ranges) {
    using Acc = typename Traits<T>::Acc;
    constexpr int W = VECP ? Traits<T>::VEC : 1;
    constexpr int UNR = 4;
    constexpr int64_t UL = 32 * W * UNR;
    const int lane = threadIdx.x & 31;
    const int64_t gwarp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t total = n_seg * upg;
    const int64_t u0 = gwarp * per_warp;
    const int64_t u1 = min(total, u0 + per_warp);
    int64_t cur = -1;
    Acc hi = 0, nlo = 0;
    for (int64_t u = u0; u < u1; ++u) {
        const int64_t seg = u / upg, part = u % upg;
        if (seg != cur) {
            if (cur >= 0) {
                const Acc h = warp_max(hi), nl = warp_max(nlo);
                if (lane == 0) {
                    atomicMax(ranges + 2 * cur, range_bits(h));
                    if (!sym) atomicMax(ranges + 2 * cur + 1, range_bits(nl));
                }
            }
            cur = seg;
            hi = 0; nlo = 0;
        }
        const int64_t base = seg * G + part * UL;
        const int64_t lim = min(UL, G - part * UL);
#pragma unroll
        for (int k = 0; k < UNR; ++k) {
            const int64_t e = (int64_t)(k * 32 + lane) * W;
            if (e < lim) {
                Acc v[W];
                if constexpr (VECP) load_vec<T>(ld16_stream(x + base + e), v);
                else v[0] = ld1<T>(x + base + e);
#pragma unroll
                for (int m = 0; m < W; ++m) acc_range<Acc>(v[m], sym, hi, nlo);
            }
        }
    }
    if (cur >= 0) {
        const Acc h = warp_max(hi), nl = warp_max(nlo);
        if (lane == 0) {
            atomicMax(ranges + 2 * cur, range_bits(h));
            if (!sym) atomicMax(ranges + 2 * cur + 1, range_bits(nl));
        }
    }
}

// Groups that hold no element (a zero-sized dimension after the axis): the
// range is empty, so the parameters are those of a zero range.
__global__ void k_empty_groups(int64_t n_seg, IntCfg cfg, float* scale, uint8_t* zp) {
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_seg;
         g += (int64_t)gridDim.x * blockDim.x) {
        const GroupF p = derive_f(0.0f, 0.0f, cfg);
        scale[g] = p.s;
        if (zp) zp[g] = (uint8_t)p.zp;
    }
}

__global__ void k_range_to_amax(const unsigned long long* rec, float* amax) {
    pdl_wait();
    float h, n;
    range_from_bits(rec[0], h);
    range_from_bits(rec[1], n);
    *amax = fmaxf(h, n);
}

// ------------------------------------------------------------ launchers
static int g_sms[64];

int sm_count() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    int v = __atomic_load_n(&g_sms[dev], __ATOMIC_RELAXED);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        __atomic_store_n(&g_sms[dev], v, __ATOMIC_RELAXED);
    }
    return v;
}

// Resident blocks per SM of a kernel at `threads` threads (occupancy API).
template <class K>
static int resident_blocks(K kernel, int threads) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = 1;
    }
    return n;
}

// Persistent grid: enough blocks for the work, at most one full wave.
template <class K>
static unsigned grid_occ(K kernel, int threads, int64_t need_blocks) {
    static const int bps = resident_blocks(kernel, threads);
    const int64_t cap = (int64_t)sm_count() * bps;
    if (need_blocks < 1) need_blocks = 1;
    return (unsigned)(need_blocks < cap ? need_blocks : cap);
}

static unsigned grid_for(int64_t work_items, int per_block, int blocks_per_sm) {
    int64_t need = (work_items + per_block - 1) / per_block;
    int64_t cap = (int64_t)sm_count() * blocks_per_sm;
    if (need < 1) need = 1;
    return (unsigned)(need < cap ? need : cap);
}

template <class T, int OP, int NV, int SEGS, bool SYM>
static void launch_warp(DynArgs a, int team, cudaStream_t st) {
    a.team = team;
    const int64_t per_warp = (int64_t)(32 / team) * SEGS;
    const int64_t warps = (a.n_seg + per_warp - 1) / per_warp;
    auto k = k_int_dyn_warp<T, OP, NV, SEGS, SYM>;
    k<<<grid_occ(k, 256, (warps + 7) / 8), 256, 0, st>>>(a);
}

template <class T, int OP, int NV, bool SYM>
static void launch_cta(const DynArgs& a, cudaStream_t st) {
    auto k = k_int_dyn_cta<T, OP, NV, SYM>;
    k<<<grid_occ(k, 256, a.n_seg), 256, 0, st>>>(a);
}

// Register-resident configurations by vectors per group U: small groups
// give each lane several vectors (fewer lanes share a group), large ones a
// CTA of 256 threads.
template <class T, int OP, bool SYM>
static cudaError_t launch_dyn_t(const DynArgs& a, cudaStream_t st) {
    constexpr int VEC = Traits<T>::VEC;
    const int64_t U = a.G / VEC;
    auto pow2 = [](int64_t v) { int t = 1; while (t < v) t <<= 1; return t; };
    if (U == 1)            launch_warp<T, OP, 1, 8, SYM>(a, 1, st);
    else if (U == 2)       launch_warp<T, OP, 2, 4, SYM>(a, 1, st);
    else if (U <= 128)     launch_warp<T, OP, 4, 2, SYM>(a, pow2((U + 3) / 4), st);
    else if (U <= 256)     launch_cta<T, OP, 1, SYM>(a, st);
    else if (U <= 512)     launch_cta<T, OP, 2, SYM>(a, st);
    else if (U <= 1024)    launch_cta<T, OP, 4, SYM>(a, st);
    else if (U <= 2048)    launch_cta<T, OP, 8, SYM>(a, st);
    else if (U <= 4096)    launch_cta<T, OP, 16, SYM>(a, st);
    else return cudaErrorNotSupported;
    return cudaGetLastError();
}

template <class T>
static cudaError_t launch_dyn_dt(int op, bool sym, const DynArgs& a, cudaStream_t st) {
    if (op == OP_QUANT) return sym ? launch_dyn_t<T, OP_QUANT, true>(a, st) : launch_dyn_t<T, OP_QUANT, false>(a, st);
    return sym ? launch_dyn_t<T, OP_FAKE, true>(a, st) : launch_dyn_t<T, OP_FAKE, false>(a, st);
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

cudaError_t int_dyn(DT dt, int op, const void* x, SegView sv, IntCfg cfg, void* q, void* y,
                    float* scale, void* zp, cudaStream_t st) {
    const cudaError_t pe = int_dyn_pipe(dt, op, x, sv, cfg, q, y, scale, zp, st);
    if (pe != cudaErrorNotSupported) return pe;
    if (dt == DT::F64 || cfg.rhaz) return cudaErrorNotSupported;
    if (op != OP_QUANT && op != OP_FAKE) return cudaErrorNotSupported;
    const int VEC = (dt == DT::F32) ? 4 : 8;
    if (sv.G % VEC != 0 || sv.G > (int64_t)4096 * VEC || !aligned16(x)) return cudaErrorNotSupported;
    if (op == OP_QUANT && ((uintptr_t)q % VEC) != 0) return cudaErrorNotSupported;
    if (op == OP_FAKE && !aligned16(y)) return cudaErrorNotSupported;
    if (sv.n_seg == 0) return cudaSuccess;
    DynArgs a;
    a.x = x; a.n_seg = sv.n_seg; a.G = (int)sv.G; a.team = 32; a.cfg = cfg;
    a.q = (uint8_t*)q; a.y = y; a.scale = scale; a.zp = (uint8_t*)zp;
    const bool sym = cfg.symmetric != 0;
    switch (dt) {
        case DT::F32: return launch_dyn_dt<float>(op, sym, a, st);
        case DT::F16: return launch_dyn_dt<__half>(op, sym, a, st);
        case DT::BF16: return launch_dyn_dt<__nv_bfloat16>(op, sym, a, st);
        default: return cudaErrorNotSupported;
    }
}

template <class T, int OP, int PSRC, bool VECP>
static cudaError_t launch_map4(const MapArgs& a, cudaStream_t st) {
    const int W = VECP ? Traits<T>::VEC : 1;
    const int U = (OP == OP_DEQ) ? 8 : 4;
    const int64_t chunks = (a.numel / W + 32 * U - 1) / (32 * U);
    if (a.cfg.rhaz) {
        auto k = k_int_map<T, OP, PSRC, VECP, true>;
        k<<<grid_occ(k, 256, (chunks + 7) / 8), 256, 0, st>>>(a);
    } else {
        auto k = k_int_map<T, OP, PSRC, VECP, false>;
        k<<<grid_occ(k, 256, (chunks + 7) / 8), 256, 0, st>>>(a);
    }
    return cudaGetLastError();
}

template <class T, int OP, int PSRC>
static cudaError_t launch_map3(const MapArgs& a, bool vecp, cudaStream_t st) {
    return vecp ? launch_map4<T, OP, PSRC, true>(a, st) : launch_map4<T, OP, PSRC, false>(a, st);
}

template <class T>
static cudaError_t launch_map_dt(int op, int psrc, const MapArgs& a, bool vecp, cudaStream_t st) {
    switch (op) {
        case OP_QUANT:
            return psrc == PS_RANGE ? launch_map3<T, OP_QUANT, PS_RANGE>(a, vecp, st)
                                    : launch_map3<T, OP_QUANT, PS_STATIC>(a, vecp, st);
        case OP_FAKE:
            return psrc == PS_RANGE ? launch_map3<T, OP_FAKE, PS_RANGE>(a, vecp, st)
                                    : launch_map3<T, OP_FAKE, PS_STATIC>(a, vecp, st);
        case OP_QBWD: return launch_map3<T, OP_QBWD, PS_STATIC>(a, vecp, st);
        case OP_FBWD: return launch_map3<T, OP_FBWD, PS_STATIC>(a, vecp, st);
        case OP_DEQ: return launch_map3<T, OP_DEQ, PS_STATIC>(a, vecp, st);
        case OP_DBWD: return launch_map3<T, OP_DBWD, PS_STATIC>(a, vecp, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t int_map(DT dt, int op, int psrc, const void* a_ptr, const void* b_ptr, SegView sv,
                    IntCfg cfg, const float* scale_in, const void* zp_in,
                    const unsigned long long* ranges, float* scale_out, void* zp_out, void* out,
                    cudaStream_t st) {
    if (sv.numel == 0) return cudaSuccess;
    MapArgs a;
    a.a = a_ptr; a.b = b_ptr;
    a.numel = sv.numel; a.G = sv.G; a.n_seg = sv.n_seg;
    a.use_fd = (sv.numel < ((int64_t)1 << 32)) ? 1 : 0;
    a.fd = make_fastdiv(a.use_fd ? (uint32_t)sv.G : 1u);
    a.cfg = cfg;
    a.scale_in = scale_in; a.zp_in = zp_in; a.ranges = ranges;
    a.scale_out = scale_out; a.zp_out = (uint8_t*)zp_out; a.out = out;
    const int esz = (dt == DT::F64) ? 8 : (dt == DT::F32 ? 4 : 2);
    const int VEC = 16 / esz;
    bool vecp = (sv.G % VEC == 0);
    if (op == OP_DEQ) {
        vecp = vecp && aligned16(out) && ((uintptr_t)a_ptr % VEC == 0);
    } else {
        vecp = vecp && aligned16(a_ptr);
        if (op == OP_QBWD || op == OP_FBWD) vecp = vecp && aligned16(b_ptr);
        if (op == OP_QUANT) vecp = vecp && ((uintptr_t)out % VEC == 0);
        else vecp = vecp && aligned16(out);
    }
    // Packed 4-bit codes are written and read a whole vector (whole bytes) at
    // a time; the callers only pass shapes and pointers that allow it.
    if (cfg.packed && !vecp && (op == OP_QUANT || op == OP_DEQ)) return cudaErrorNotSupported;
    if (vecp && !(cfg.packed && op == OP_QUANT)) {
        const cudaError_t pe = int_map_pipe(dt, op, a, st);
        if (pe != cudaErrorNotSupported) return pe;
    }
    switch (dt) {
        case DT::F32: return launch_map_dt<float>(op, psrc, a, vecp, st);
        case DT::F64: return launch_map_dt<double>(op, psrc, a, vecp, st);
        case DT::F16: return launch_map_dt<__half>(op, psrc, a, vecp, st);
        case DT::BF16: return launch_map_dt<__nv_bfloat16>(op, psrc, a, vecp, st);
    }
    return cudaErrorInvalidValue;
}

template <class T>
static cudaError_t launch_seg_range_t(const void* x, SegView sv, bool sym, unsigned long long* r,
                                      cudaStream_t st) {
    constexpr int VEC = Traits<T>::VEC;
    const bool vecp = (sv.G % VEC == 0) && aligned16(x);
    const int64_t UL = 32 * (vecp ? VEC : 1) * 4;
    const int64_t upg = (sv.G + UL - 1) / UL;
    const int64_t total = sv.n_seg * upg;
    const unsigned grid = grid_for(total * 32, 256, 8);
    const int64_t nwarps = (int64_t)grid * 8;
    const int64_t per_warp = (total + nwarps - 1) / nwarps;
    if (vecp) k_seg_range<T, true><<<grid, 256, 0, st>>>((const T*)x, sv.n_seg, sv.G, upg, per_warp, sym, r);
    else k_seg_range<T, false><<<grid, 256, 0, st>>>((const T*)x, sv.n_seg, sv.G, upg, per_warp, sym, r);
    return cudaGetLastError();
}

cudaError_t seg_range(DT dt, const void* x, SegView sv, bool sym, unsigned long long* ranges,
                      cudaStream_t st) {
    if (sv.n_seg == 0 || sv.G == 0) return cudaSuccess;
    switch (dt) {
        case DT::F32: return launch_seg_range_t<float>(x, sv, sym, ranges, st);
        case DT::F64: return launch_seg_range_t<double>(x, sv, sym, ranges, st);
        case DT::F16: return launch_seg_range_t<__half>(x, sv, sym, ranges, st);
        case DT::BF16: return launch_seg_range_t<__nv_bfloat16>(x, sv, sym, ranges, st);
    }
    return cudaErrorInvalidValue;
}

template <class T>
static cudaError_t launch_tensor_range_t(const void* x, int64_t n, bool sym,
                                         unsigned long long* rec, cudaStream_t st) {
    constexpr int VEC = Traits<T>::VEC;
    int64_t head = 0;
    const uintptr_t p = (uintptr_t)x;
    if (p % 16 != 0) {
        head = (int64_t)((16 - p % 16) / sizeof(T));
        if (head > n) head = n;
    }
    const int64_t nvec = (n - head) / VEC;
    const unsigned grid = grid_for(nvec / 4 + 1, 512, 2);
    k_tensor_range<T><<<grid, 512, 0, st>>>((const T*)x, n, head, sym ? 1 : 0, rec);
    return cudaGetLastError();
}

cudaError_t tensor_range(DT dt, const void* x, int64_t n, bool sym, unsigned long long* rec,
                         cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const cudaError_t pe = tensor_range_pipe(dt, x, n, sym, rec, st);
    if (pe != cudaErrorNotSupported) return pe;
    switch (dt) {
        case DT::F32: return launch_tensor_range_t<float>(x, n, sym, rec, st);
        case DT::F64: return launch_tensor_range_t<double>(x, n, sym, rec, st);
        case DT::F16: return launch_tensor_range_t<__half>(x, n, sym, rec, st);
        case DT::BF16: return launch_tensor_range_t<__nv_bfloat16>(x, n, sym, rec, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t empty_groups(int64_t n_seg, IntCfg cfg, float* scale, void* zp, cudaStream_t st) {
    if (n_seg == 0) return cudaSuccess;
    k_empty_groups<<<grid_for(n_seg, 256, 4), 256, 0, st>>>(n_seg, cfg, scale, (uint8_t*)zp);
    return cudaGetLastError();
}

__global__ void k_set_f32(float* p, float v) { *p = v; }

cudaError_t set_f32(float* p, float v, cudaStream_t st) {
    k_set_f32<<<1, 1, 0, st>>>(p, v);
    return cudaGetLastError();
}

cudaError_t range_to_amax(const unsigned long long* rec, float* amax, cudaStream_t st) {
    return launch_pdl(k_range_to_amax, 1u, 1u, 0, st, rec, amax);
}

// Lets the range kernel after it start at once (it waits for this one before
// its atomics).
__global__ void k_clear_records(unsigned long long* rec, int64_t n) {
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        rec[i] = 0ull;
}

cudaError_t clear_records(unsigned long long* rec, int64_t n, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    k_clear_records<<<grid_for(n, 256, 4), 256, 0, st>>>(rec, n);
    return cudaGetLastError();
}

}  // namespace bq
