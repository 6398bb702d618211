// Bulk-copy pipelined quantizers for contiguous groups with dynamic scales:
// per-token / per-channel / per-group integer quantize and fake-quantize
// (baracuda_kernels::quantize), FP8 1x128 and MXFP8 (smile llm.quant
// Fp8BlockGemm, MxFp8) and NVFP4 (metrale QuantizedWeight).
//
// A persistent CTA of 256 threads walks tiles of P whole groups. The tiles
// reach shared memory through cp.async.bulk (the Blackwell / Hopper bulk copy
// engine, no registers held while in flight) into a ring of STAGES slots,
// each completed on its own mbarrier; while the threads reduce and encode
// one tile, the next STAGES-1 are in flight. The CTA splits into 256/TEAM
// teams, one group per team, each thread holding NV 16-byte vectors of its
// group; teams of up to 32 lanes reduce with warp shuffles, larger teams
// also through shared memory. Codes go straight from registers to HBM.
//
// Every wait on an mbarrier is bounded: after about two seconds the kernel
// records the failure in g_pipe_error, waits (bounded again) for the copies
// it has in flight, and returns.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "bq_device.cuh"
#include "bq_internal.h"
#include "bq_quant_ops.cuh"
#include "bq_map_ops.cuh"
#include "bq_range.cuh"
#include "bq_pipe_args.h"

namespace bq {
namespace {   // one copy per dtype translation unit

// Set when a bounded wait gives up (one flag per translation unit).
__device__ unsigned int g_pipe_error;


// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// One thread: expect `bytes` on the barrier and start the bulk copy.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(1000u) : "memory");
    return ok != 0;
}
// Bounded wait: each try suspends for at most about a microsecond.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < (1u << 21); ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
__device__ __forceinline__ U4 ld_shared16(uint32_t addr) {
    U4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

// The general encoder of one vector (a clamp that can bind, a NaN, a scale
// outside the fast range), kept out of line: it is the rare path, and
// inlining it into the unrolled loops only adds instruction-cache pressure
// to the fast one.
template <class T, int OP, bool SYM>
__device__ __noinline__ void emit_int_general(U4 raw, Recip R, IntParams ip, uint8_t* q, int packed, T* y) {
    float v[Traits<T>::VEC];
    load_vec<T>(raw, v);
    if (R.fast) emit_int<T, OP, true, SYM>(v, R, ip, q, packed, y);
    else emit_int<T, OP, false, SYM>(v, R, ip, q, packed, y);
}

// ------------------------------------------------------------ the kernel
// Tuning constants (compile-time): ring depth of the dynamic quantizer for
// slots of up to 16 KB (NV <= 4) and 32 KB (NV >= 8); team width for groups of
// 9..16 vectors; ring depth of the group-tiled element kernels.
#ifndef BQ_SEG_STAGES_16K
#define BQ_SEG_STAGES_16K 3
#endif
#ifndef BQ_SEG_STAGES_32K
#define BQ_SEG_STAGES_32K 2
#endif
#ifndef BQ_SEG_TEAM_16
#define BQ_SEG_TEAM_16 4
#endif
#ifndef BQ_MAP_STAGES
#define BQ_MAP_STAGES 2
#endif

template <int NV> struct PipeStages { static constexpr int S = NV <= 4 ? BQ_SEG_STAGES_16K : BQ_SEG_STAGES_32K; };

template <class T, int PK, int TEAM, int NV, bool SYM, int NT>
__global__ void __launch_bounds__(NT) k_seg_pipe(PipeArgs a) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int NW = NT / 32;
    constexpr int SPAN = TEAM * NV * VEC;          // elements a team covers
    constexpr bool ABS = (PK != PK_INT_Q && PK != PK_INT_FAKE) || SYM;
    extern __shared__ __align__(128) uint8_t smem[];
    float* red = reinterpret_cast<float*>(smem);                     // [2][NW]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);         // [stages]
    uint8_t* ring = smem + 128;                                      // [stages][slot_bytes]
    const int tid = threadIdx.x;
    const int team = tid / TEAM, lane = tid % TEAM;
    const int wid = tid >> 5;
    constexpr int S = PipeStages<NV>::S;
    const int64_t grid = gridDim.x;
    const size_t esz = sizeof(T);
    const int G = a.G;
    const bool full_groups = (G == SPAN);
    // Teams narrower than 8 lanes read their vectors in an order rotated by
    // team, so that the 8 lanes of one 128-byte shared-memory phase (several
    // teams) land on distinct banks: vector j of a thread is vidx(j).
    constexpr int ROT_DIV = (TEAM * NV >= 8) ? 1 : 8 / (TEAM * NV);
    const int rot = (TEAM >= 8) ? 0 : team / ROT_DIV;
    auto vidx = [&](int j) { return (TEAM >= 8 || NV == 1) ? j : ((j + rot) & (NV - 1)); };

    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(smem_addr(&bars[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto tile_bytes = [&](int64_t tile) -> uint32_t {
        const int64_t segs = min((int64_t)a.P, a.n_seg - tile * a.P);
        return (uint32_t)(segs * G * esz);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            const int64_t tile = blockIdx.x + (int64_t)i * grid;
            if (tile >= a.n_tiles) break;
            bulk_load(smem_addr(ring + (size_t)i * a.slot_bytes),
                      (const uint8_t*)a.x + (size_t)tile * a.P * G * esz, tile_bytes(tile),
                      smem_addr(&bars[i]));
        }
    }

    // Launch constants.
    float s2 = 1.0f;
    Recip R6, Rq;
    const float qlo = (float)a.cfg.qmin, qhi = (float)a.cfg.qmax;
    if constexpr (PK == PK_NV) {
        if (a.static_global == 1) {
            s2 = *a.global_scale;
        } else {
            // The range kernel before this one may still be running (launch_pdl).
            pdl_wait();
            float h, n;
            range_from_bits(a.amax_rec[0], h);
            range_from_bits(a.amax_rec[1], n);
            s2 = __fdiv_rn(fmaxf(h, n), 2688.0f);
            if (s2 == 0.0f) s2 = 1.0f;
            if (blockIdx.x == 0 && tid == 0) *a.global_scale = s2;
        }
        R6 = make_recip(__fmul_rn(6.0f, s2));
    } else if constexpr (PK == PK_FP8) {
        Rq = make_recip(448.0f);
    } else if constexpr (PK == PK_INT_Q || PK == PK_INT_FAKE) {
        Rq = make_recip(SYM ? qhi : (float)(a.cfg.qmax - a.cfg.qmin));
    }

    int slot = 0;
    uint32_t parity = 0;
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += grid) {
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        const uint8_t* slot_ptr = ring + (size_t)slot * a.slot_bytes;
        const int64_t seg = tile * a.P + team;
        const bool seg_ok = seg < a.n_seg;
        const bool full = seg_ok && full_groups;

        // This thread's vectors of its group, straight from shared memory,
        // in the team's rotated order (vidx). (After a failed wait the slot
        // holds stale bytes; they are read but never used.)
        U4 raw[NV];
        const uint32_t gbase = smem_addr(slot_ptr + (size_t)team * G * esz) + (uint32_t)(lane * 16);
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = (vidx(j) * TEAM + lane) * VEC;
            raw[j] = (full || (seg_ok && e < G)) ? ld_shared16(gbase + (uint32_t)(vidx(j) * TEAM * 16))
                                                 : U4{0u, 0u, 0u, 0u};
        }
        // One barrier: every thread holds its vectors, so the slot is free
        // and is refilled with tile + S before this tile is encoded.
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                // Drain the copies still in flight into this CTA's ring.
                int s2 = slot;
                uint32_t p2 = parity;
                for (int i = 0; i < S; ++i) {
                    const int64_t t2 = tile + (int64_t)i * grid;
                    if (t2 >= a.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s2]), p2);
                    if (++s2 == S) { s2 = 0; p2 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < a.n_tiles) {
                fence_proxy_async();
                bulk_load(smem_addr(ring + (size_t)slot * a.slot_bytes),
                          (const uint8_t*)a.x + (size_t)next * a.P * G * esz, tile_bytes(next),
                          smem_addr(&bars[slot]));
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
        // Range with NaN propagation; a thread that met a NaN recomputes its
        // part ignoring NaN (the range the formats define) and its warp takes
        // the general encoders.
        uint32_t ph = 0u, pl = 0u;
        float hi = 0.0f, nlo = 0.0f;
        range_tree<T, ABS, true, NV>(raw, ph, pl, hi, nlo);
        const bool saw_nan = range_finish_nan<T, ABS>(ph, pl, hi, nlo);
        if (saw_nan) {
            ph = pl = 0u;
            hi = nlo = 0.0f;
            range_tree<T, ABS, false, NV>(raw, ph, pl, hi, nlo);
            range_finish<T, ABS>(ph, pl, hi, nlo);
        }
        const bool warp_nan = __any_sync(0xffffffffu, saw_nan);
        if constexpr (TEAM > 1) {
#pragma unroll
            for (int o = (TEAM < 32 ? TEAM : 32) / 2; o > 0; o >>= 1) {
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
                if (!ABS) nlo = fmaxf(nlo, __shfl_xor_sync(0xffffffffu, nlo, o));
            }
        }
        if constexpr (TEAM > 32) {
            constexpr int WPT = TEAM / 32;
            if ((tid & 31) == 0) { red[wid] = hi; red[NW + wid] = nlo; }
            __syncthreads();
            const int w0 = team * WPT;
            hi = red[w0];
            nlo = red[NW + w0];
#pragma unroll
            for (int w = 1; w < WPT; ++w) {
                hi = fmaxf(hi, red[w0 + w]);
                if (!ABS) nlo = fmaxf(nlo, red[NW + w0 + w]);
            }
        }
        // Vector j of this thread: valid, and its offset in the group.
        auto vok = [&](int j) { return full || (seg_ok && (vidx(j) * TEAM + lane) * VEC < G); };
        auto voff = [&](int j) { return vidx(j) * TEAM * VEC; };

        if constexpr (PK == PK_INT_Q || PK == PK_INT_FAKE) {
            constexpr int OP = (PK == PK_INT_Q) ? OP_QUANT : OP_FAKE;
            // Scale and zero-point: fl(amax/qmax) or fl(fl(max'-min')/(qmax-qmin)),
            // each quotient by the launch's divisor reciprocal (exact for a
            // normal dividend; IEEE division below 2^-100).
            float sc, zf = 0.0f, rz = 0.0f;
            Recip R;
            {
                const float num = SYM ? fmaxf(hi, nlo) : __fadd_rn(hi, nlo);
                sc = (num >= 0x1p-100f && num <= 0x1p100f) ? div_chain(num, Rq) : div_slow(num, Rq.s);
                if (sc == 0.0f) sc = 1.0f;
                R = make_recip(sc);
                if (!SYM) {
                    // fl(min'/s) through the group's reciprocal: |min'/s| <= qmax - qmin,
                    // so the chain cannot overflow, and it is exact wherever the
                    // rounding to an integer can depend on it (|min'/s| >= 1/2).
                    const float m = R.fast ? div_chain(-nlo, R) : __fdiv_rn(-nlo, sc);
                    rz = a.cfg.rhaz ? roundf(m) : rintf(m);
                    zf = fminf(fmaxf(__fsub_rn(qlo, rz), qlo), qhi);   // NaN -> qmin
                }
            }
            const int zp = (int)zf;
            if (seg_ok && lane == 0) {
                a.scale[seg] = sc;
                if (a.zp) a.zp[seg] = (uint8_t)zp;
            }
            IntParams ip;
            ip.lo = SYM ? qlo : __fsub_rn(qlo, zf);
            ip.hi = SYM ? qhi : __fsub_rn(qhi, zf);
            ip.zp = SYM ? 0 : zp;
            const int64_t qe = seg * G + lane * VEC;          // element offset of the codes
            const int pk = a.cfg.packed;
            T* yb = (T*)a.y + seg * G + lane * VEC;
            // Fast path: no NaN in the warp's groups, a normal scale, and no
            // clamp that can bind. Symmetric: |x/s| <= qmax (1 + 2^-23) rounds
            // into [-qmax, qmax], inside [qmin, qmax] when qmin <= -qmax.
            // Asymmetric: codes are monotone in x, the smallest is qmin when
            // the zero-point is unclamped, the largest is round(fl(max'/s)) + zp.
            bool noclamp;
            if constexpr (SYM) {
                noclamp = qlo <= -qhi;
            } else {
                const float kmax = R.fast ? __fsub_rn(__fadd_rn(div_chain(hi, R), kMagic), kMagic) : 0.0f;
                noclamp = (zf == __fsub_rn(qlo, rz)) && (__fadd_rn(kmax, zf) <= qhi);
            }
            if (seg_ok && R.fast && noclamp && !warp_nan) {
                const Recip2T R2 = make_recip2(R);
                const F2 magic2 = f2_bcast(kMagic), zp2 = f2_bcast(zf), s2v = f2_bcast(sc);
                // Whole groups: one branch-free block, so the vectors' division
                // chains interleave.
                if (full) {
#pragma unroll
                    for (int j = 0; j < NV; ++j)
                        emit_int_fast<T, OP, !SYM>(raw[j], R2, magic2, zp2, s2v, code_ptr(a.q, qe + voff(j), pk), pk, yb + voff(j));
                } else {
#pragma unroll
                    for (int j = 0; j < NV; ++j)
                        if (vok(j)) emit_int_fast<T, OP, !SYM>(raw[j], R2, magic2, zp2, s2v, code_ptr(a.q, qe + voff(j), pk), pk, yb + voff(j));
                }
            } else if (seg_ok) {
#pragma unroll
                for (int j = 0; j < NV; ++j)
                    if (vok(j)) emit_int_general<T, OP, SYM>(raw[j], R, ip, code_ptr(a.q, qe + voff(j), pk), pk, yb + voff(j));
            }
        } else {
            constexpr int FMT = (PK == PK_FP8) ? MX_FP8_1x128
                              : (PK == PK_MX ? MX_MXFP8 : (PK == PK_MX4 ? MX_MXFP4 : MX_NVFP4));
            constexpr int CB = (PK == PK_NV || PK == PK_MX4) ? VEC / 2 : VEC;     // code bytes per vector
            uint8_t* base = a.q + seg * (G / VEC) * CB + lane * CB;
            auto coff = [&](int j) { return vidx(j) * TEAM * CB; };
            if constexpr (PK == PK_FP8) {
                float s = (hi >= 0x1p-100f && hi <= 0x1p100f) ? div_chain(hi, Rq) : div_slow(hi, 448.0f);
                if (s == 0.0f) s = 1.0f;
                if (seg_ok && lane == 0) a.scale[seg] = s;
                const Recip R = make_recip(s);
                if (seg_ok && R.fast && !warp_nan) {
                    const Recip2T R2 = make_recip2(R);
                    if (full) {
#pragma unroll
                        for (int j = 0; j < NV; ++j) emit_fp8_fast<T>(raw[j], R2, base + coff(j));
                    } else {
#pragma unroll
                        for (int j = 0; j < NV; ++j)
                            if (vok(j)) emit_fp8_fast<T>(raw[j], R2, base + coff(j));
                    }
                } else if (seg_ok) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) {
                        if (!vok(j)) continue;
                        float v[VEC];
                        load_vec<T>(raw[j], v);
                        if (R.fast) mx_emit<T, FMT, true>(v, R, 0.f, false, base + coff(j));
                        else mx_emit<T, FMT, false>(v, R, 0.f, false, base + coff(j));
                    }
                }
            } else if constexpr (PK == PK_MX4) {
                const int E = mx_exponent(hi, 2);
                if (seg_ok && lane == 0) a.zp[seg] = (uint8_t)(E + 127);
                const float mul = exp2i(-E);
                const F2 mul2 = f2_bcast(mul);
                if (full && !warp_nan) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) emit_mx4_fast<T>(raw[j], mul2, base + coff(j));
                } else if (seg_ok && !warp_nan) {
#pragma unroll
                    for (int j = 0; j < NV; ++j)
                        if (vok(j)) emit_mx4_fast<T>(raw[j], mul2, base + coff(j));
                } else if (seg_ok) {
                    // A NaN in the warp's groups: the general encoder (NaN -> code 0).
                    const Recip R{};
#pragma unroll
                    for (int j = 0; j < NV; ++j) {
                        if (!vok(j)) continue;
                        float v[VEC];
                        load_vec<T>(raw[j], v);
                        mx_emit<T, FMT, true>(v, R, mul, false, base + coff(j));
                    }
                }
            } else if constexpr (PK == PK_MX) {
                const int E = mx_exponent(hi);
                if (seg_ok && lane == 0) a.zp[seg] = (uint8_t)(E + 127);
                const F2 mul2 = f2_bcast(exp2i(-E));
                if (full) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) emit_mx_fast<T>(raw[j], mul2, base + coff(j));
                } else if (seg_ok) {
#pragma unroll
                    for (int j = 0; j < NV; ++j)
                        if (vok(j)) emit_mx_fast<T>(raw[j], mul2, base + coff(j));
                }
            } else {
                const uint32_t sb = e4m3x2(div_any(hi, R6), 0.0f) & 0xFFu;
                if (seg_ok && lane == 0) a.zp[seg] = (uint8_t)sb;
                const float eff = __fmul_rn(e4m3_to_f32(sb), s2);
                const Recip R = make_recip(eff);
                // Fast: positive normal divisor, no NaN, quotients far from
                // overflow (|x| <= hi <= 2^64 eff).
                const bool fast = R.fast && eff > 0.0f && hi <= __fmul_rn(0x1p64f, eff) && !warp_nan;
                if (seg_ok && fast) {
                    const Recip2T R2 = make_recip2(R);
                    if (full) {
#pragma unroll
                        for (int j = 0; j < NV; ++j) emit_nv_fast<T>(raw[j], R2, base + coff(j));
                    } else {
#pragma unroll
                        for (int j = 0; j < NV; ++j)
                            if (vok(j)) emit_nv_fast<T>(raw[j], R2, base + coff(j));
                    }
                } else if (seg_ok) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) {
                        if (!vok(j)) continue;
                        float v[VEC];
                        load_vec<T>(raw[j], v);
                        mx_emit<T, FMT, false>(v, R, 0.f, eff == 0.0f, base + coff(j));
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------------ NVFP4, 16-bit inputs
// One thread per 16-element block (two 16-byte vectors), NV_BPT blocks per
// thread per tile. A block's codes divide by eff = fl(dec(sb) * s2), where sb
// is the block's E4M3 scale code: with only 256 codes, RN(1/eff) and the
// fast-path limits are tabulated once per CTA (NvEntry) instead of being
// derived once per block. Fast path (the same bits as the general encoder):
// no NaN in the block, eff a positive normal number in the exact range of
// the division chain, and |x| <= 2^64 eff (no quotient overflows).
constexpr int NV_BPT = 2;
#ifndef BQ_NV_STAGES
#define BQ_NV_STAGES 3
#endif
struct NvEntry {
    float y;      // RN(1 / eff)
    float ns;     // -eff
    float lim;    // 2^64 * eff
    uint32_t ok;  // eff > 0 and in the exact range of the chain
};

// E2M1 codes of one vector, fast path: fl(x / eff) by the chain on pairs,
// the sign of each quotient taken from x (restores -0 for x = -0).
template <class T>
__device__ __forceinline__ uint32_t nv_word_fast(const U4& raw, const Recip2& R2) {
    F2 x[4];
    widen_pairs<T>(raw, x);
    float t[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        uint32_t q0, q1, x0, x1;
        f2_split_bits(div_chain2(x[p], R2), q0, q1);
        f2_split_bits(x[p], x0, x1);
        t[2 * p] = __uint_as_float((q0 & 0x7FFFFFFFu) | (x0 & 0x80000000u));
        t[2 * p + 1] = __uint_as_float((q1 & 0x7FFFFFFFu) | (x1 & 0x80000000u));
    }
    return e2m1x8_finite(t);
}
// General path: IEEE division where the chain cannot be used; all-zero codes
// when eff == 0.
template <class T>
__device__ __forceinline__ uint32_t nv_word_general(const U4& raw, const Recip& R, bool zero) {
    float v[8];
    load_vec<T>(raw, v);
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = with_quotient_sign(div_any(v[i], R), v[i], R.s);
    return zero ? 0u : e2m1x8(t);
}

template <class T>
__global__ void __launch_bounds__(256) k_nv_quant(PipeArgs a) {
    static_assert(sizeof(T) == 2, "16-bit inputs");
    constexpr int S = BQ_NV_STAGES;
    constexpr int P = 256 * NV_BPT;                       // blocks per tile
    constexpr uint32_t SLOT = P * 32;                     // bytes per tile
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);
    NvEntry* table = reinterpret_cast<NvEntry*>(smem + 128);         // [256]
    uint8_t* ring = smem + 128 + 256 * sizeof(NvEntry);            // [S][SLOT]
    const int tid = threadIdx.x;
    const int64_t grid = gridDim.x;
    auto tile_bytes = [&](int64_t tile) -> uint32_t {
        return (uint32_t)(min((int64_t)P, a.n_seg - tile * P) * 32);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
        for (int i = 0; i < S; ++i) {
            const int64_t tile = blockIdx.x + (int64_t)i * grid;
            if (tile >= a.n_tiles) break;
            bulk_load(smem_addr(ring + (size_t)i * SLOT), (const uint8_t*)a.x + (size_t)tile * SLOT,
                      tile_bytes(tile), smem_addr(&bars[i]));
        }
    }
    // Per-tensor scale: given, or from the range record (written by the range
    // kernel that may still be running: launch_pdl).
    float s2;
    if (a.static_global == 1) {
        s2 = *a.global_scale;
    } else {
        pdl_wait();
        float h, n;
        range_from_bits(a.amax_rec[0], h);
        range_from_bits(a.amax_rec[1], n);
        s2 = __fdiv_rn(fmaxf(h, n), 2688.0f);
        if (s2 == 0.0f) s2 = 1.0f;
        if (blockIdx.x == 0 && tid == 0) *a.global_scale = s2;
    }
    const Recip R6 = make_recip(__fmul_rn(6.0f, s2));
    {
        const float eff = __fmul_rn(e4m3_to_f32((uint32_t)tid), s2);
        const Recip r = make_recip(eff);
        NvEntry e;
        e.y = r.y;
        e.ns = -eff;
        e.lim = __fmul_rn(0x1p64f, eff);
        e.ok = (r.fast && eff > 0.0f) ? 1u : 0u;
        table[tid] = e;
    }
    __syncthreads();

    // Two 16-byte vectors per block, read in an order rotated every four
    // lanes so that the eight lanes of one shared-memory phase hit distinct banks.
    const int rot = (tid >> 2) & 1;
    int slot = 0;
    uint32_t parity = 0;
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += grid) {
        const bool okw = mbar_wait(smem_addr(&bars[slot]), parity);
        const uint32_t sbase = smem_addr(ring + (size_t)slot * SLOT);
        // The thread's NV_BPT blocks go through each step together, so that
        // their serial per-block work (range, block scale, table) overlaps.
        const bool tile_full = (tile + 1) * P <= a.n_seg;
        U4 r0[NV_BPT], r1[NV_BPT];
        bool okb[NV_BPT], nan[NV_BPT];
        float hi[NV_BPT];
        uint32_t sb[NV_BPT];
#pragma unroll
        for (int g = 0; g < NV_BPT; ++g) {
            const int lb = g * 256 + tid;                     // block in the tile
            okb[g] = tile_full || tile * P + lb < a.n_seg;
            const uint32_t ba = sbase + (uint32_t)lb * 32u;
            r0[g] = okb[g] ? ld_shared16(ba + (uint32_t)(rot * 16)) : U4{0u, 0u, 0u, 0u};
            r1[g] = okb[g] ? ld_shared16(ba + (uint32_t)((rot ^ 1) * 16)) : U4{0u, 0u, 0u, 0u};
        }
        // One barrier: the blocks are in registers, the slot is refilled now.
        if (__syncthreads_or(!okw)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s3 = slot;
                uint32_t p3 = parity;
                for (int i = 0; i < S; ++i) {
                    if (tile + (int64_t)i * grid >= a.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s3]), p3);
                    if (++s3 == S) { s3 = 0; p3 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < a.n_tiles) {
                fence_proxy_async();
                bulk_load(smem_addr(ring + (size_t)slot * SLOT), (const uint8_t*)a.x + (size_t)next * SLOT,
                          tile_bytes(next), smem_addr(&bars[slot]));
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
#pragma unroll
        for (int g = 0; g < NV_BPT; ++g) {
            uint32_t ph = 0u, pl = 0u;
            float h = 0.0f, nlo = 0.0f;
            const U4 rr[2] = {r0[g], r1[g]};
            range_tree<T, true, true, 2>(rr, ph, pl, h, nlo);
            nan[g] = range_finish_nan<T, true>(ph, pl, h, nlo);
            if (nan[g]) {
                ph = 0u;
                range_tree<T, true, false, 2>(rr, ph, pl, h, nlo);
                range_finish<T, true>(ph, pl, h, nlo);
            }
            hi[g] = h;
        }
#pragma unroll
        for (int g = 0; g < NV_BPT; ++g) sb[g] = e4m3x2(div_any(hi[g], R6), 0.0f) & 0xFFu;
#pragma unroll
        for (int g = 0; g < NV_BPT; ++g) {
            if (!tile_full && !okb[g]) continue;
            const int64_t blk = tile * P + g * 256 + tid;
            a.zp[blk] = (uint8_t)sb[g];
            const NvEntry e = table[sb[g]];
            uint32_t w0, w1;     // codes of vectors r0, r1
            if (e.ok && hi[g] <= e.lim && !nan[g]) {
                Recip2 R2;
                R2.y = f2_bcast(e.y);
                R2.ns = f2_bcast(e.ns);
                w0 = nv_word_fast<T>(r0[g], R2);
                w1 = nv_word_fast<T>(r1[g], R2);
            } else {
                const float eff = -e.ns;
                const Recip R = make_recip(eff);
                w0 = nv_word_general<T>(r0[g], R, eff == 0.0f);
                w1 = nv_word_general<T>(r1[g], R, eff == 0.0f);
            }
            st8(a.q + blk * 8, rot ? w1 : w0, rot ? w0 : w1);
        }
    }
}

// ------------------------------------------------------------ FP8 128x128 tiles, 16-bit inputs
// One 128x128 tile per ring slot (32 KB), brought in by one 2D tensor copy
// (TMA, no multicast): the copy engine fetches the 128 row segments itself
// and fills the part of an edge tile outside the tensor with zeros, which
// leaves the tile's amax unchanged. Two passes over the slot: the amax (then
// one block reduction), then the codes; thread t owns the 16-byte vectors
// v = t, t + 256, ... of the tile (row v / 16, column chunk v % 16), so the
// shared loads are conflict-free and each row's codes leave as sixteen
// consecutive 8-byte stores.
#ifndef BQ_TILE_STAGES
#define BQ_TILE_STAGES 2
#endif

struct TileArgs {
    int64_t rows, cols, nbc, n_tiles;
    uint8_t* e4m3;
    float* scale;
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int c0, int c1,
                                            uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"((uint64_t)tm), "r"(c0), "r"(c1), "r"(bar) : "memory");
}

template <class T>
__global__ void __launch_bounds__(256) k_fp8_tile_tma(const __grid_constant__ CUtensorMap tm,
                                                      TileArgs a) {
    static_assert(sizeof(T) == 2, "16-bit inputs");
    constexpr int S = BQ_TILE_STAGES;
    constexpr uint32_t SLOT = 128 * 256;
    extern __shared__ __align__(128) uint8_t smem[];
    float* red = reinterpret_cast<float*>(smem);                  // [8] warp maxima
    uint32_t* rnan = reinterpret_cast<uint32_t*>(smem + 32);      // [8] warp saw a NaN
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);      // [S]
    uint8_t* ring = smem + 128;
    const int tid = threadIdx.x;
    const int64_t grid = gridDim.x;
    auto issue = [&](int64_t tile, int slot) {
        const int64_t bi = tile / a.nbc, bj = tile - bi * a.nbc;
        const uint32_t bar = smem_addr(&bars[slot]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(SLOT) : "memory");
        tma_load_2d(smem_addr(ring + (size_t)slot * SLOT), &tm, (int)(bj * 128), (int)(bi * 128), bar);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
        for (int i = 0; i < S; ++i) {
            const int64_t tile = blockIdx.x + (int64_t)i * grid;
            if (tile >= a.n_tiles) break;
            issue(tile, i);
        }
    }
    __syncthreads();
    const Recip Rq = make_recip(448.0f);
    int slot = 0;
    uint32_t parity = 0;
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += grid) {
        const bool okw = mbar_wait(smem_addr(&bars[slot]), parity);
        const uint32_t sbase = smem_addr(ring + (size_t)slot * SLOT);
        // Pass 1: the tile's amax (NaN propagated to detect one, then ignored).
        uint32_t ph = 0u, pl = 0u;
        float hi = 0.0f, nlo = 0.0f;
        bool nan = false;
        if (okw) {
            U4 rv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) rv[i] = ld_shared16(sbase + (uint32_t)(i * 256 + tid) * 16u);
            range_tree<T, true, true, 8>(rv, ph, pl, hi, nlo);
            nan = range_finish_nan<T, true>(ph, pl, hi, nlo);
            if (nan) {
                ph = 0u;
                range_tree<T, true, false, 8>(rv, ph, pl, hi, nlo);
                range_finish<T, true>(ph, pl, hi, nlo);
            }
        }
        hi = warp_max(hi);
        const bool wnan = __any_sync(0xffffffffu, nan);
        if ((tid & 31) == 0) {
            red[tid >> 5] = hi;
            rnan[tid >> 5] = wnan ? 1u : 0u;
        }
        if (__syncthreads_or(!okw)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s3 = slot;
                uint32_t p3 = parity;
                for (int i = 0; i < S; ++i) {
                    if (tile + (int64_t)i * grid >= a.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s3]), p3);
                    if (++s3 == S) { s3 = 0; p3 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        float am = red[0];
        uint32_t any_nan = rnan[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            am = fmaxf(am, red[w]);
            any_nan |= rnan[w];
        }
        float sc = (am >= 0x1p-100f && am <= 0x1p100f) ? div_chain(am, Rq) : div_slow(am, 448.0f);
        if (sc == 0.0f) sc = 1.0f;
        if (tid == 0) a.scale[tile] = sc;
        const Recip R = make_recip(sc);
        // Pass 2: codes of the valid part of the tile.
        const int64_t bi = tile / a.nbc, bj = tile - bi * a.nbc;
        const int nr = (int)min((int64_t)128, a.rows - bi * 128);
        const int nch = (int)((min((int64_t)128, a.cols - bj * 128)) / 8);
        const bool full = (nr == 128) && (nch == 16);
        uint8_t* obase = a.e4m3 + bi * 128 * a.cols + bj * 128;
        const bool fast = R.fast && !any_nan;
        const Recip2T R2 = make_recip2(R);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int v = i * 256 + tid;
            const int r = v >> 4, ch = v & 15;
            if (!full && (r >= nr || ch >= nch)) continue;
            const U4 raw = ld_shared16(sbase + (uint32_t)v * 16u);
            uint8_t* dst = obase + (int64_t)r * a.cols + ch * 8;
            if (fast) {
                emit_fp8_fast<T>(raw, R2, dst);
            } else {
                float vals[8];
                load_vec<T>(raw, vals);
                if (R.fast) mx_emit<T, MX_FP8_1x128, true>(vals, R, 0.f, false, dst);
                else mx_emit<T, MX_FP8_1x128, false>(vals, R, 0.f, false, dst);
            }
        }
        __syncthreads();
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < a.n_tiles) {
                fence_proxy_async();
                issue(next, slot);
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
    }
}

// ------------------------------------------------------------ FP8 per-tensor
// FP8 per-tensor store (smile llm.quant Fp8KvCodec): e = E4M3(fl(x / s)) with
// one f32 scale s for the whole tensor, given (*scale) or fl(amax / 448) from
// the range record written by the range kernel just before this one (launched
// to overlap it: the first copies go out before the wait). A vector with a
// NaN or an element beyond 2^64 s takes the general encoder.
struct Fp8TArgs {
    const void* x;
    int64_t n;
    uint8_t* e4m3;
    float* scale;
    const unsigned long long* rec;
    int from_rec;
};

// The same store, pipelined: chunks of FP8T_CHUNK bytes of x reach shared
// memory by bulk copy into a ring of FP8T_STAGES slots; each thread copies its
// vectors of a chunk to registers, one barrier frees the slot for the chunk S
// ahead, then the vectors are encoded. x 16-byte and e4m3 8-byte aligned.
constexpr int FP8T_CHUNK = 32768;
constexpr int FP8T_STAGES = 2;

template <class T>
__global__ void __launch_bounds__(256) k_fp8t_pipe(Fp8TArgs a) {
    constexpr int VEC = Traits<T>::VEC;
    constexpr int S = FP8T_STAGES;
    constexpr int NVT = FP8T_CHUNK / 16 / 256;            // vectors per thread per chunk
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);
    uint8_t* ring = smem + 128;
    const int tid = threadIdx.x;
    const int64_t grid = gridDim.x;
    const T* x = (const T*)a.x;
    const int64_t nvec = a.n / VEC;                        // whole 16-byte vectors
    const int64_t body = nvec * 16;
    const int64_t n_chunks = (body + FP8T_CHUNK - 1) / FP8T_CHUNK;
    auto chunk_bytes = [&](int64_t c) -> uint32_t {
        return (uint32_t)min((int64_t)FP8T_CHUNK, body - c * FP8T_CHUNK);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
        for (int i = 0; i < S; ++i) {
            const int64_t c = blockIdx.x + (int64_t)i * grid;
            if (c >= n_chunks) break;
            bulk_load(smem_addr(ring + (size_t)i * FP8T_CHUNK), (const uint8_t*)x + c * FP8T_CHUNK,
                      chunk_bytes(c), smem_addr(&bars[i]));
        }
    }
    __syncthreads();
    float s;
    if (a.from_rec) {
        pdl_wait();
        float h, nl;
        range_from_bits(a.rec[0], h);
        range_from_bits(a.rec[1], nl);
        s = __fdiv_rn(fmaxf(h, nl), 448.0f);
        if (s == 0.0f) s = 1.0f;
        if (blockIdx.x == 0 && tid == 0) *a.scale = s;
    } else {
        s = *a.scale;
    }
    const Recip R = make_recip(s);
    const bool fast_s = R.fast && s > 0.0f;
    const Recip2T R2 = make_recip2(R);
    const float lim = __fmul_rn(0x1p64f, s);
    int slot = 0;
    uint32_t parity = 0;
    for (int64_t c = blockIdx.x; c < n_chunks; c += grid) {
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        const uint32_t base = smem_addr(ring + (size_t)slot * FP8T_CHUNK);
        const int nv = (int)(chunk_bytes(c) / 16);
        U4 raw[NVT];
#pragma unroll
        for (int v = 0; v < NVT; ++v) {
            const int vi = v * 256 + tid;
            raw[v] = (vi < nv) ? ld_shared16(base + (uint32_t)vi * 16u) : U4{0u, 0u, 0u, 0u};
        }
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s3 = slot;
                uint32_t p3 = parity;
                for (int i = 0; i < S; ++i) {
                    if (c + (int64_t)i * grid >= n_chunks) break;
                    mbar_wait(smem_addr(&bars[s3]), p3);
                    if (++s3 == S) { s3 = 0; p3 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        if (tid == 0) {
            const int64_t next = c + (int64_t)S * grid;
            if (next < n_chunks) {
                fence_proxy_async();
                bulk_load(smem_addr(ring + (size_t)slot * FP8T_CHUNK), (const uint8_t*)x + next * FP8T_CHUNK,
                          chunk_bytes(next), smem_addr(&bars[slot]));
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
        const int64_t v0 = c * (FP8T_CHUNK / 16);            // first vector of the chunk
#pragma unroll
        for (int v = 0; v < NVT; ++v) {
            const int vi = v * 256 + tid;
            if (vi >= nv) continue;
            uint32_t ph = 0u, pl = 0u;
            float hi = 0.0f, nlo = 0.0f;
            range_tree<T, true, true, 1>(&raw[v], ph, pl, hi, nlo);
            const bool nan = range_finish_nan<T, true>(ph, pl, hi, nlo);
            uint8_t* dst = a.e4m3 + (v0 + vi) * VEC;
            if (fast_s && !nan && hi <= lim) {
                emit_fp8_fast<T>(raw[v], R2, dst);
            } else {
                float vals[VEC];
                load_vec<T>(raw[v], vals);
                mx_emit<T, MX_FP8_1x128, false>(vals, R, 0.f, false, dst);
            }
        }
    }
    // elements after the last whole vector
    if (blockIdx.x == 0 && tid < a.n - nvec * VEC) {
        const int64_t i = nvec * VEC + tid;
        const float v = ld1<T>(x + i);
        a.e4m3[i] = (uint8_t)(e4m3x2(with_quotient_sign(div_any(v, R), v, s), 0.0f) & 0xFFu);
    }
}

// Any alignment: one element per thread step.
template <class T>
__global__ void __launch_bounds__(256) k_fp8_tensor_scalar(Fp8TArgs a) {
    float s;
    if (a.from_rec) {
        pdl_wait();
        float h, nl;
        range_from_bits(a.rec[0], h);
        range_from_bits(a.rec[1], nl);
        s = __fdiv_rn(fmaxf(h, nl), 448.0f);
        if (s == 0.0f) s = 1.0f;
        if (blockIdx.x == 0 && threadIdx.x == 0) *a.scale = s;
    } else {
        s = *a.scale;
    }
    const Recip R = make_recip(s);
    const T* x = (const T*)a.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = ld1<T>(x + i);
        a.e4m3[i] = (uint8_t)(e4m3x2(with_quotient_sign(div_any(v, R), v, s), 0.0f) & 0xFFu);
    }
}

// ------------------------------------------------------------ tensor range
// Range record of a whole tensor (per-tensor scaling, the NVFP4 per-tensor
// scale). The 16-byte aligned body is cut into units of RANGE_UNIT bytes (one
// 16-byte vector per thread); CTA b takes the contiguous units
// [b*U/grid, (b+1)*U/grid), so no CTA streams more than one unit above the
// mean, and streams them through a ring of RANGE_STAGES bulk copies of up to
// RANGE_CHUNK bytes; each thread folds its vectors into
// a packed running range (two 16-bit lanes per instruction). The few
// elements before the first 16-byte boundary and after the last one go
// through scalar loads in block 0. One atomicMax per CTA and record slot, made
// after pdl_wait(): the kernel before this one on the stream clears the
// record, and this kernel is launched to overlap it.
constexpr int RANGE_CHUNK = 16384;
constexpr int RANGE_STAGES = 4;
constexpr int RANGE_UNIT = 4096;

struct RangeArgs {
    const void* x;        // first element
    int64_t head;         // elements before the 16-byte aligned body
    int64_t body_bytes;   // multiple of 16
    int64_t n;            // all elements
    unsigned long long* rec;
    float* amax;          // tensor amax: written by the last CTA (ABS only; rec[1] counts CTAs)
};

template <class T, bool ABS>
__global__ void __launch_bounds__(256) k_range_pipe(RangeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    float* red = reinterpret_cast<float*>(smem);                  // [2][8]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);      // [RANGE_STAGES]
    uint8_t* ring = smem + 128;                                   // [RANGE_STAGES][RANGE_CHUNK]
    constexpr int S = RANGE_STAGES;
    const int tid = threadIdx.x;
    const int64_t grid = gridDim.x;
    const T* x = (const T*)a.x;
    const uint8_t* body = (const uint8_t*)(x + a.head);
    const int64_t n_units = (a.body_bytes + RANGE_UNIT - 1) / RANGE_UNIT;
    const int64_t b0 = (int64_t)blockIdx.x * n_units / grid * RANGE_UNIT;
    const int64_t b1 = min(((int64_t)blockIdx.x + 1) * n_units / grid * RANGE_UNIT, a.body_bytes);
    const int64_t my_bytes = max(b1 - b0, (int64_t)0);
    const uint8_t* mine = body + b0;
    const int64_t n_chunks = (my_bytes + RANGE_CHUNK - 1) / RANGE_CHUNK;
    auto chunk_bytes = [&](int64_t c) -> uint32_t {
        return (uint32_t)min((int64_t)RANGE_CHUNK, my_bytes - c * RANGE_CHUNK);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
        for (int i = 0; i < S && i < n_chunks; ++i)
            bulk_load(smem_addr(ring + (size_t)i * RANGE_CHUNK), mine + (int64_t)i * RANGE_CHUNK,
                      chunk_bytes(i), smem_addr(&bars[i]));
    }
    __syncthreads();
    uint32_t ph = 0u, pl = 0u;
    float hi = 0.0f, nlo = 0.0f;
    int slot = 0;
    uint32_t parity = 0;
    for (int64_t c = 0; c < n_chunks; ++c) {
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s2 = slot;
                uint32_t p2 = parity;
                for (int i = 0; i < S; ++i) {
                    if (c + i >= n_chunks) break;
                    mbar_wait(smem_addr(&bars[s2]), p2);
                    if (++s2 == S) { s2 = 0; p2 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        const uint32_t base = smem_addr(ring + (size_t)slot * RANGE_CHUNK);
        const int nv = (int)(chunk_bytes(c) / 16);
        if (nv == RANGE_CHUNK / 16) {
            constexpr int NVC = RANGE_CHUNK / 16 / 256;
            U4 rv[NVC];
#pragma unroll
            for (int v = 0; v < NVC; ++v) rv[v] = ld_shared16(base + (uint32_t)((v * 256 + tid) * 16));
            range_tree<T, ABS, false, NVC>(rv, ph, pl, hi, nlo);
        } else {
            for (int v = tid; v < nv; v += 256)
                range_acc<T, ABS, false>(ld_shared16(base + (uint32_t)(v * 16)), ph, pl, hi, nlo);
        }
        __syncthreads();
        if (tid == 0) {
            const int64_t next = c + S;
            if (next < n_chunks) {
                fence_proxy_async();
                bulk_load(smem_addr(ring + (size_t)slot * RANGE_CHUNK), mine + next * RANGE_CHUNK,
                          chunk_bytes(next), smem_addr(&bars[slot]));
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
    }
    pdl_trigger();
    range_finish<T, ABS>(ph, pl, hi, nlo);
    // Unaligned head and tail: fewer than 16 bytes each.
    if (blockIdx.x == 0) {
        const int64_t tail0 = a.head + a.body_bytes / (int64_t)sizeof(T);
        int64_t e = -1;
        if (tid < a.head) e = tid;
        else if (tid >= 16 && tid - 16 < a.n - tail0) e = tail0 + (tid - 16);
        if (e >= 0) {
            const float v = ld1<T>(x + e);
            if (ABS) {
                hi = fmaxf(hi, fabsf(v));
            } else {
                hi = fmaxf(hi, v);
                nlo = fmaxf(nlo, -v);
            }
        }
    }
    hi = warp_max(hi);
    if (!ABS) nlo = warp_max(nlo);
    if ((tid & 31) == 0) { red[tid >> 5] = hi; red[8 + (tid >> 5)] = nlo; }
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < 8; ++w) { hi = fmaxf(hi, red[w]); nlo = fmaxf(nlo, red[8 + w]); }
        pdl_wait();
        atomicMax(a.rec, range_bits(hi));
        if (!ABS) atomicMax(a.rec + 1, range_bits(nlo));
        if (ABS && a.amax) {
            // The last CTA to finish turns the record into the amax: rec[1]
            // (unused by an absolute range, zeroed by the clearing kernel)
            // counts finished CTAs; each CTA's maximum is visible before its
            // count (fence), so the last one reads the final record.
            __threadfence();
            const unsigned long long done = atomicAdd(a.rec + 1, 1ull);
            if (done == (unsigned long long)gridDim.x - 1ull) {
                __threadfence();
                float h;
                range_from_bits(atomicAdd(a.rec, 0ull), h);
                *a.amax = h;
            }
        }
    }
}

// ------------------------------------------------------------ element-wise
// Tiles of 256 * ITEMS vectors; both inputs of a backward land in one slot
// (first the x part, then the dy part). Thread t handles the vectors
// t, t + 256, ... of its tile: conflict-free shared loads, coalesced stores.
// Items (16-byte vectors) per thread per tile and ring depth: enough work per
// tile to amortise the per-tile wait and barrier, within 96 KB of ring.
template <int OP> struct MapShape {
    static constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    static constexpr int ITEMS = TWO ? 4 : 8;
    static constexpr int S = 3;
};

struct MapPipeArgs {
    MapArgs m;
    int64_t n_tiles;
    int tile_elems;     // 256 * kMapItems * W
    int in_esz;         // bytes per element of input a (1 for codes)
    int slot_bytes;
    int stages;
};

template <class T, int OP, int PSRC, bool RHAZ>
__global__ void __launch_bounds__(256) k_map_pipe(MapPipeArgs p) {
    using Acc = typename Traits<T>::Acc;
    constexpr int W = Traits<T>::VEC;
    constexpr int ITEMS = MapShape<OP>::ITEMS;
    constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    constexpr int ESZ = sizeof(T);
    const MapArgs& a = p.m;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);
    uint8_t* ring = smem + 128;
    const int tid = threadIdx.x;
    constexpr int S = MapShape<OP>::S;
    const int64_t grid = gridDim.x;
    const int E = p.tile_elems;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(smem_addr(&bars[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Tile `tile` into slot `slot`: input a, then (backwards) input b.
    auto issue = [&](int64_t tile, int slot) {
        const int64_t e0 = tile * E;
        const int64_t n = min((int64_t)E, a.numel - e0);
        const uint32_t ba = (uint32_t)(n * p.in_esz);
        const uint32_t bb = TWO ? (uint32_t)(n * ESZ) : 0u;
        const uint32_t bar = smem_addr(&bars[slot]);
        uint8_t* dst = ring + (size_t)slot * p.slot_bytes;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(ba + bb) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     :: "r"(smem_addr(dst)), "l"((const uint8_t*)a.a + e0 * p.in_esz), "r"(ba), "r"(bar) : "memory");
        if (TWO)
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         :: "r"(smem_addr(dst + (size_t)E * p.in_esz)), "l"((const uint8_t*)a.b + e0 * ESZ),
                            "r"(bb), "r"(bar) : "memory");
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            const int64_t tile = blockIdx.x + (int64_t)i * grid;
            if (tile >= p.n_tiles) break;
            issue(tile, i);
        }
    }
    GState st;
    st.seg = -1;
    int slot = 0;
    uint32_t parity = 0;
    for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += grid) {
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s2 = slot;
                uint32_t p2 = parity;
                for (int i = 0; i < S; ++i) {
                    const int64_t t2 = tile + (int64_t)i * grid;
                    if (t2 >= p.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s2]), p2);
                    if (++s2 == S) { s2 = 0; p2 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        const uint8_t* sa = ring + (size_t)slot * p.slot_bytes;
        const uint8_t* sb = sa + (size_t)E * p.in_esz;
        const int64_t te0 = tile * E;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int le = (i * 256 + tid) * W;               // element offset in the tile
            const int64_t e0 = te0 + le;
            if (e0 >= a.numel) continue;
            const int64_t seg = a.use_fd ? (int64_t)fdiv((uint32_t)e0, a.fd) : e0 / a.G;
            if (seg != st.seg) load_group<T, PSRC, (OP == OP_QBWD || OP == OP_FBWD), RHAZ>(a, seg, e0 == seg * a.G, st);
            if constexpr (OP == OP_DEQ) {
                Acc o[W];
                if constexpr (W == 8) {
                    uint32_t w0, w1;
                    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(smem_addr(sa + le)));
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = deq_code_f(w0, k, st, a.cfg.q_signed);
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[4 + k] = deq_code_f(w1, k, st, a.cfg.q_signed);
                } else {
                    uint32_t w0;
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(smem_addr(sa + le)));
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = deq_code_f(w0, k, st, a.cfg.q_signed);
                }
                st16((T*)a.out + e0, pack_vec<T>(o));
            } else {
                Acc xa[W], xb[W];
                load_vec<T>(ld_shared16(smem_addr(sa + (size_t)le * ESZ)), xa);
                if constexpr (TWO) load_vec<T>(ld_shared16(smem_addr(sb + (size_t)le * ESZ)), xb);
                Acc o[W];
                uint32_t cw[W];
#pragma unroll
                for (int k = 0; k < W; ++k) o[k] = elem_f<OP, RHAZ>(xa[k], TWO ? xb[k] : 0.0f, st, &cw[k]);
                if constexpr (OP == OP_QUANT) {
                    uint8_t* q = (uint8_t*)a.out + e0;
                    if constexpr (W == 8) st8(q, pack4_lowbytes(cw[0], cw[1], cw[2], cw[3]), pack4_lowbytes(cw[4], cw[5], cw[6], cw[7]));
                    else st4(q, pack4_lowbytes(cw[0], cw[1], cw[2], cw[3]));
                } else {
                    st16((T*)a.out + e0, pack_vec<T>(o));
                }
            }
        }
        __syncthreads();
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < p.n_tiles) {
                fence_proxy_async();
                issue(next, slot);
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
    }
}

// ------------------------------------------------------------ element-wise, by group
// The element-wise ops on tiles of P whole groups, one team of 256/P threads
// per group (the layout of k_seg_pipe): each thread loads its group's
// parameters once and applies them to NV vectors. Backwards stage x and dy of
// the same groups in one slot.
struct SegMapArgs {
    MapArgs m;
    int P;
    int64_t n_tiles;
    int in_esz;         // bytes per element of input a (1 for codes)
    int code_shift;     // 1: 4-bit codes two per byte (byte counts of a halved)
    int part_bytes;     // P * G * in_esz: where the dy part of a slot starts
    int slot_bytes;
};

template <int OP> struct SegMapStages { static constexpr int S = BQ_MAP_STAGES; };

template <class T, int OP, int PSRC, int TEAM, int NV, bool RHAZ>
__global__ void __launch_bounds__(256) k_seg_map(SegMapArgs p) {
    using Acc = typename Traits<T>::Acc;
    constexpr int W = Traits<T>::VEC;
    constexpr int ESZ = sizeof(T);
    constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    constexpr int SPAN = TEAM * NV * W;
    constexpr int S = SegMapStages<OP>::S;
    const MapArgs& a = p.m;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64);
    uint8_t* ring = smem + 128;
    const int tid = threadIdx.x;
    const int team = tid / TEAM, lane = tid % TEAM;
    const int64_t grid = gridDim.x;
    const int G = (int)a.G;
    const bool full_groups = (G == SPAN);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(smem_addr(&bars[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int64_t tile, int slot) {
        const int64_t segs = min((int64_t)p.P, a.n_seg - tile * p.P);
        const int64_t e0 = tile * p.P * G;
        const uint32_t ba = (uint32_t)((segs * G * p.in_esz) >> p.code_shift);
        const uint32_t bb = TWO ? (uint32_t)(segs * G * ESZ) : 0u;
        const uint32_t bar = smem_addr(&bars[slot]);
        uint8_t* dst = ring + (size_t)slot * p.slot_bytes;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(ba + bb) : "memory");
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                     :: "r"(smem_addr(dst)), "l"((const uint8_t*)a.a + ((e0 * p.in_esz) >> p.code_shift)), "r"(ba), "r"(bar) : "memory");
        if (TWO)
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         :: "r"(smem_addr(dst + p.part_bytes)), "l"((const uint8_t*)a.b + e0 * ESZ),
                            "r"(bb), "r"(bar) : "memory");
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            const int64_t tile = blockIdx.x + (int64_t)i * grid;
            if (tile >= p.n_tiles) break;
            issue(tile, i);
        }
    }
    GState st;
    st.seg = -1;
    int slot = 0;
    uint32_t parity = 0;
    // Static group parameters, loaded one tile ahead so their latency hides
    // behind the current tile's work.
    auto fetch = [&](int64_t sg, float& s, int& z) {
        if (sg < a.n_seg) {
            s = __ldg(a.scale_in + sg);
            z = a.cfg.symmetric ? 0 : load_zp(a.zp_in, sg, a.cfg.q_signed);
        }
    };
    float pf_s = 1.0f;
    int pf_z = 0;
    fetch((int64_t)blockIdx.x * p.P + team, pf_s, pf_z);
    for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += grid) {
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        const int64_t seg = tile * p.P + team;
        const bool seg_ok = seg < a.n_seg;
        // This thread's vectors (codes: 8 / 4 bytes per vector; otherwise x and,
        // for the backwards, dy) copied to registers. (After a failed wait the
        // slot holds stale bytes; they are read but never used.)
        const uint8_t* sa = ring + (size_t)slot * p.slot_bytes + (((size_t)team * G * p.in_esz) >> p.code_shift);
        const uint8_t* sb = ring + (size_t)slot * p.slot_bytes + p.part_bytes + (size_t)team * G * ESZ;
        U4 va[NV], vb[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = (j * TEAM + lane) * W;              // element offset in the group
            const bool v_ok = seg_ok && (full_groups || e < G);
            va[j] = U4{0u, 0u, 0u, 0u};
            vb[j] = U4{0u, 0u, 0u, 0u};
            if (v_ok) {
                if constexpr (OP == OP_DEQ) {
                    if (p.code_shift) {
                        // two 4-bit codes per byte, widened to one per byte
                        if constexpr (W == 8) {
                            uint32_t v;
                            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(sa + (e >> 1))));
                            va[j].x = nib_spread(v & 0xFFFFu, a.cfg.q_signed);
                            va[j].y = nib_spread(v >> 16, a.cfg.q_signed);
                        } else {
                            unsigned short v;
                            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_addr(sa + (e >> 1))));
                            va[j].x = nib_spread(v, a.cfg.q_signed);
                        }
                    } else if constexpr (W == 8) {
                        asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(va[j].x), "=r"(va[j].y) : "r"(smem_addr(sa + e)));
                    } else {
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(va[j].x) : "r"(smem_addr(sa + e)));
                    }
                } else {
                    va[j] = ld_shared16(smem_addr(sa + (size_t)e * ESZ));
                    if constexpr (TWO) vb[j] = ld_shared16(smem_addr(sb + (size_t)e * ESZ));
                }
            }
        }
        // One barrier: the bounded wait's verdict, and the slot is free to be
        // refilled with tile + S while this tile is computed.
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s2 = slot;
                uint32_t p2 = parity;
                for (int i = 0; i < S; ++i) {
                    const int64_t t2 = tile + (int64_t)i * grid;
                    if (t2 >= p.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s2]), p2);
                    if (++s2 == S) { s2 = 0; p2 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < p.n_tiles) {
                fence_proxy_async();
                issue(next, slot);
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
        const float cur_s = pf_s;
        const int cur_z = pf_z;
        fetch((tile + grid) * p.P + team, pf_s, pf_z);
        if (seg_ok) {
            if constexpr (TWO && TEAM >= 32) {
                group_set<T, false, RHAZ>(a, seg, cur_s, cur_z, st);
                st.mfast = mask_thresholds_warp<RHAZ>(st.R, st.ip, &st.x_lo, &st.x_hi);
                st.fast = st.mfast && st.R.fast;
            } else {
                group_set<T, TWO, RHAZ>(a, seg, cur_s, cur_z, st);
            }
            const int64_t gbase = seg * G;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int e = (j * TEAM + lane) * W;              // element offset in the group
                if (!full_groups && e >= G) continue;
                Acc o[W];
                if constexpr (OP == OP_DEQ) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = deq_code_f(va[j].x, k, st, a.cfg.q_signed);
                    if constexpr (W == 8) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) o[4 + k] = deq_code_f(va[j].y, k, st, a.cfg.q_signed);
                    }
                    st16((T*)a.out + gbase + e, pack_vec<T>(o));
                } else {
                    Acc xa[W], xb[W];
                    load_vec<T>(va[j], xa);
                    if constexpr (TWO) load_vec<T>(vb[j], xb);
                    uint32_t cw[W];
                    if constexpr (TWO) {
                        if (st.fast) {
#pragma unroll
                            for (int k = 0; k < W; ++k) o[k] = elem_bwd_fast<OP>(xa[k], xb[k], st);
                        } else {
#pragma unroll
                            for (int k = 0; k < W; ++k) o[k] = elem_f<OP, RHAZ>(xa[k], xb[k], st, &cw[k]);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < W; ++k) o[k] = elem_f<OP, RHAZ>(xa[k], 0.0f, st, &cw[k]);
                    }
                    if constexpr (OP == OP_QUANT) {
                        uint8_t* q = (uint8_t*)a.out + gbase + e;
                        if constexpr (W == 8) st8(q, pack4_lowbytes(cw[0], cw[1], cw[2], cw[3]), pack4_lowbytes(cw[4], cw[5], cw[6], cw[7]));
                        else st4(q, pack4_lowbytes(cw[0], cw[1], cw[2], cw[3]));
                    } else {
                        st16((T*)a.out + gbase + e, pack_vec<T>(o));
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------------ launchers
// Resident 256-thread blocks per SM of kernel k with `smem` bytes of dynamic
// shared memory. Each caller passes its own `cache` (a static array in the
// launcher of one kernel instantiation), which remembers the answer for up to
// eight distinct ring sizes, so the query runs once per process and size.
static int occupancy_for(const void* k, size_t smem, unsigned long long (&cache)[8], int threads = 256) {
    for (int i = 0; i < 8; ++i) {
        const unsigned long long e = __atomic_load_n(&cache[i], __ATOMIC_RELAXED);
        if (e == 0) break;
        if ((e >> 8) == smem) return (int)(e & 0xFFu) - 1;
    }
    int v = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k, threads, smem) != cudaSuccess) {
        (void)cudaGetLastError();
        v = 0;
    }
    const unsigned long long ent = ((unsigned long long)smem << 8) | (unsigned long long)(v + 1);
    for (int i = 0; i < 8; ++i) {
        unsigned long long expected = 0;
        if (__atomic_compare_exchange_n(&cache[i], &expected, ent, false, __ATOMIC_RELAXED,
                                        __ATOMIC_RELAXED) || (expected >> 8) == smem)
            break;
    }
    return v;
}

template <class T, int PK, int TEAM, int NV, bool SYM, int NT = 256>
static cudaError_t launch_pipe_t(PipeArgs a, cudaStream_t st) {
    constexpr int P = NT / TEAM;
    constexpr int S = PipeStages<NV>::S;
    a.P = P;
    a.slot_bytes = P * a.G * (int)sizeof(T);
    a.n_tiles = (a.n_seg + P - 1) / P;
    a.stages = S;
    const size_t smem = 128 + (size_t)S * a.slot_bytes;
    auto k = k_seg_pipe<T, PK, TEAM, NV, SYM, NT>;
    // Largest ring this instantiation can need: P groups of TEAM*NV vectors.
    static const cudaError_t attr = cudaFuncSetAttribute(
        k, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 + S * P * TEAM * NV * 16);
    if (attr != cudaSuccess) return attr;
    static unsigned long long occ[8];
    const int bps = occupancy_for((const void*)k, smem, occ, NT);
    if (bps < 1) return cudaErrorNotSupported;
    int64_t grid = (int64_t)sm_count() * bps;
    if (grid > a.n_tiles) grid = a.n_tiles;
    // NVFP4 with a per-tensor scale from the range record: overlap the range
    // kernel's tail (the kernel waits for it before reading the record).
    if (PK == PK_NV && a.static_global == 0) return launch_pdl(k, (unsigned)grid, (unsigned)NT, smem, st, a);
    k<<<(unsigned)grid, NT, smem, st>>>(a);
    return cudaGetLastError();
}

// NVFP4 of 16-bit inputs (k_nv_quant).
template <class T>
static cudaError_t launch_nv_t(PipeArgs a, cudaStream_t st) {
    constexpr int P = 256 * NV_BPT;
    constexpr int S = BQ_NV_STAGES;
    a.P = P;
    a.n_tiles = (a.n_seg + P - 1) / P;
    const size_t smem = 128 + 256 * sizeof(NvEntry) + (size_t)S * P * 32;
    auto k = k_nv_quant<T>;
    static const cudaError_t attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    static unsigned long long occ[8];
    const int bps = occupancy_for((const void*)k, smem, occ);
    if (bps < 1) return cudaErrorNotSupported;
    int64_t grid = (int64_t)sm_count() * bps;
    if (grid > a.n_tiles) grid = a.n_tiles;
    if (a.static_global == 0) return launch_pdl(k, (unsigned)grid, 256u, smem, st, a);
    k<<<(unsigned)grid, 256, smem, st>>>(a);
    return cudaGetLastError();
}

// Configuration by vectors per group U (TEAM lanes x NV vectors >= U).
template <class T, int PK, bool SYM>
static cudaError_t launch_pipe_u(const PipeArgs& a, cudaStream_t st) {
    constexpr int VEC = Traits<T>::VEC;
    const int U = a.G / VEC;
    if (U <= 1) return launch_pipe_t<T, PK, 1, 1, SYM>(a, st);
    if (U <= 2) return launch_pipe_t<T, PK, 1, 2, SYM>(a, st);
    if (U <= 4) return launch_pipe_t<T, PK, 1, 4, SYM>(a, st);
    if (U <= 8) return launch_pipe_t<T, PK, 2, 4, SYM>(a, st);
    if (U <= 16) {
        if constexpr (BQ_SEG_TEAM_16 == 1) return launch_pipe_t<T, PK, 1, 16, SYM, 128>(a, st);
        else return launch_pipe_t<T, PK, BQ_SEG_TEAM_16, 16 / BQ_SEG_TEAM_16, SYM>(a, st);
    }
    if (U <= 32) return launch_pipe_t<T, PK, 8, 4, SYM>(a, st);
    if constexpr (PK == PK_INT_Q || PK == PK_INT_FAKE) {
        if (U <= 64) return launch_pipe_t<T, PK, 16, 4, SYM>(a, st);
        if (U <= 128) return launch_pipe_t<T, PK, 32, 4, SYM>(a, st);
        if (U <= 256) return launch_pipe_t<T, PK, 64, 4, SYM>(a, st);
        // Rows of up to 512 vectors: one warp per group, 16 vectors per lane,
        // 128-thread CTAs (the reduction stays inside the warp).
        if (U <= 512) return launch_pipe_t<T, PK, 32, 16, SYM, 128>(a, st);
        if (U <= 1024) return launch_pipe_t<T, PK, 128, 8, SYM>(a, st);
        if (U <= 2048) return launch_pipe_t<T, PK, 256, 8, SYM>(a, st);
    }
    return cudaErrorNotSupported;
}

template <class T>
static cudaError_t pipe_dt(int pk, bool sym, const PipeArgs& a, cudaStream_t st) {
    switch (pk) {
        case PK_INT_Q: return sym ? launch_pipe_u<T, PK_INT_Q, true>(a, st) : launch_pipe_u<T, PK_INT_Q, false>(a, st);
        case PK_INT_FAKE: return sym ? launch_pipe_u<T, PK_INT_FAKE, true>(a, st) : launch_pipe_u<T, PK_INT_FAKE, false>(a, st);
        case PK_FP8: return launch_pipe_u<T, PK_FP8, true>(a, st);
        case PK_MX: return launch_pipe_u<T, PK_MX, true>(a, st);
        case PK_MX4: return launch_pipe_u<T, PK_MX4, true>(a, st);
        case PK_NV:
            if constexpr (sizeof(T) == 2) {
                if (((uintptr_t)a.q & 7u) == 0) return launch_nv_t<T>(a, st);
            }
            return launch_pipe_u<T, PK_NV, true>(a, st);
    }
    return cudaErrorInvalidValue;
}

template <class T, int OP, int PSRC, bool RHAZ>
static cudaError_t launch_map_pipe_t(const MapArgs& m, cudaStream_t st) {
    constexpr int W = Traits<T>::VEC;
    constexpr int S = MapShape<OP>::S;
    MapPipeArgs p;
    p.m = m;
    p.tile_elems = 256 * MapShape<OP>::ITEMS * W;
    p.in_esz = (OP == OP_DEQ) ? 1 : (int)sizeof(T);
    const int two = (OP == OP_QBWD || OP == OP_FBWD) ? (int)sizeof(T) : 0;
    p.slot_bytes = p.tile_elems * (p.in_esz + two);
    p.stages = S;
    p.n_tiles = (m.numel + p.tile_elems - 1) / p.tile_elems;
    const size_t smem = 128 + (size_t)S * p.slot_bytes;
    auto k = k_map_pipe<T, OP, PSRC, RHAZ>;
    static const cudaError_t attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    static unsigned long long occ[8];
    const int bps = occupancy_for((const void*)k, smem, occ);
    if (bps < 1) return cudaErrorNotSupported;
    int64_t grid = (int64_t)sm_count() * bps;
    if (grid > p.n_tiles) grid = p.n_tiles;
    k<<<(unsigned)grid, 256, smem, st>>>(p);
    return cudaGetLastError();
}

template <class T, int OP, int PSRC>
static cudaError_t map_pipe_r(const MapArgs& m, cudaStream_t st) {
    return m.cfg.rhaz ? launch_map_pipe_t<T, OP, PSRC, true>(m, st) : launch_map_pipe_t<T, OP, PSRC, false>(m, st);
}

template <class T>
static cudaError_t map_pipe_dt(int op, int psrc, const MapArgs& m, cudaStream_t st) {
    switch (op) {
        case OP_QUANT: return psrc == PS_RANGE ? map_pipe_r<T, OP_QUANT, PS_RANGE>(m, st) : map_pipe_r<T, OP_QUANT, PS_STATIC>(m, st);
        case OP_FAKE: return psrc == PS_RANGE ? map_pipe_r<T, OP_FAKE, PS_RANGE>(m, st) : map_pipe_r<T, OP_FAKE, PS_STATIC>(m, st);
        case OP_QBWD: return map_pipe_r<T, OP_QBWD, PS_STATIC>(m, st);
        case OP_FBWD: return map_pipe_r<T, OP_FBWD, PS_STATIC>(m, st);
        case OP_DEQ: return map_pipe_r<T, OP_DEQ, PS_STATIC>(m, st);
        case OP_DBWD: return map_pipe_r<T, OP_DBWD, PS_STATIC>(m, st);
    }
    return cudaErrorInvalidValue;
}

template <class T, int OP, int PSRC, int TEAM, int NV, bool RHAZ>
static cudaError_t launch_seg_map_t(const MapArgs& m, cudaStream_t st) {
    constexpr int P = 256 / TEAM;
    constexpr int S = SegMapStages<OP>::S;
    constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    SegMapArgs p;
    p.m = m;
    p.P = P;
    p.n_tiles = (m.n_seg + P - 1) / P;
    p.in_esz = (OP == OP_DEQ) ? 1 : (int)sizeof(T);
    p.code_shift = (OP == OP_DEQ && m.cfg.packed) ? 1 : 0;
    p.part_bytes = (P * (int)m.G * p.in_esz) >> p.code_shift;
    p.slot_bytes = p.part_bytes + (TWO ? P * (int)m.G * (int)sizeof(T) : 0);
    const size_t smem = 128 + (size_t)S * p.slot_bytes;
    constexpr int in_max = (OP == OP_DEQ) ? 1 : (int)sizeof(T);
    constexpr int max_slot = P * TEAM * NV * Traits<T>::VEC * (in_max + (TWO ? (int)sizeof(T) : 0));
    auto k = k_seg_map<T, OP, PSRC, TEAM, NV, RHAZ>;
    static const cudaError_t attr = cudaFuncSetAttribute(
        k, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 + S * max_slot);
    if (attr != cudaSuccess) return attr;
    static unsigned long long occ[8];
    const int bps = occupancy_for((const void*)k, smem, occ);
    if (bps < 1) return cudaErrorNotSupported;
    int64_t grid = (int64_t)sm_count() * bps;
    if (grid > p.n_tiles) grid = p.n_tiles;
    k<<<(unsigned)grid, 256, smem, st>>>(p);
    return cudaGetLastError();
}

// (TEAM, NV) by vectors per group U in [5, 1024]; ring slots stay within 32 KB.
template <class T, int OP, int PSRC, bool RHAZ>
static cudaError_t seg_map_u(const MapArgs& m, cudaStream_t st) {
    const int64_t U = m.G / Traits<T>::VEC;
    if (U <= 4) return cudaErrorNotSupported;
    if (U <= 8) return launch_seg_map_t<T, OP, PSRC, 2, 4, RHAZ>(m, st);
    if (U <= 16) return launch_seg_map_t<T, OP, PSRC, 4, 4, RHAZ>(m, st);
    if (U <= 32) return launch_seg_map_t<T, OP, PSRC, 8, 4, RHAZ>(m, st);
    if (U <= 64) return launch_seg_map_t<T, OP, PSRC, 16, 4, RHAZ>(m, st);
    if (U <= 128) return launch_seg_map_t<T, OP, PSRC, 32, 4, RHAZ>(m, st);
    if (U <= 256) return launch_seg_map_t<T, OP, PSRC, 64, 4, RHAZ>(m, st);
    if (U <= 512) return launch_seg_map_t<T, OP, PSRC, 128, 4, RHAZ>(m, st);
    if (U <= 1024) return launch_seg_map_t<T, OP, PSRC, 256, 4, RHAZ>(m, st);
    return cudaErrorNotSupported;
}

// Group-tiled element kernels: dequantize and the backwards with nearest-even
// rounding (other element ops take the flat pipelined kernel).
template <class T>
static cudaError_t seg_map_dt(int op, const MapArgs& m, cudaStream_t st) {
    if (m.cfg.rhaz && (op == OP_QBWD || op == OP_FBWD)) return cudaErrorNotSupported;
    switch (op) {
        case OP_QBWD: return seg_map_u<T, OP_QBWD, PS_STATIC, false>(m, st);
        case OP_FBWD: return seg_map_u<T, OP_FBWD, PS_STATIC, false>(m, st);
        case OP_DEQ: return seg_map_u<T, OP_DEQ, PS_STATIC, false>(m, st);
        case OP_DBWD: return seg_map_u<T, OP_DBWD, PS_STATIC, false>(m, st);
    }
    return cudaErrorNotSupported;
}

// Range of a whole tensor into rec (cleared by the kernel before this one on
// the stream); launched to overlap that kernel (launch_pdl).
template <class T>
static cudaError_t range_entry(const void* x, int64_t n, bool sym, unsigned long long* rec,
                               cudaStream_t st, float* amax = nullptr) {
    RangeArgs a;
    a.amax = sym ? amax : nullptr;
    a.x = x;
    a.n = n;
    a.head = 0;
    const uintptr_t p = (uintptr_t)x;
    if (p % 16 != 0) a.head = min((int64_t)((16 - p % 16) / sizeof(T)), n);
    a.body_bytes = (n - a.head) * (int64_t)sizeof(T) / 16 * 16;
    a.rec = rec;
    const int64_t n_units = (a.body_bytes + RANGE_UNIT - 1) / RANGE_UNIT;
    const size_t smem = 128 + (size_t)RANGE_STAGES * RANGE_CHUNK;
    auto k = sym ? k_range_pipe<T, true> : k_range_pipe<T, false>;
    static const cudaError_t attr_s = cudaFuncSetAttribute(
        k_range_pipe<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    static const cudaError_t attr_a = cudaFuncSetAttribute(
        k_range_pipe<T, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr_s != cudaSuccess) return attr_s;
    if (attr_a != cudaSuccess) return attr_a;
    static unsigned long long occ[8];
    const int bps = occupancy_for((const void*)k_range_pipe<T, true>, smem, occ);
    if (bps < 1) return cudaErrorNotSupported;
    int64_t grid = (int64_t)sm_count() * bps;
    if (grid > n_units) grid = n_units;
    if (grid < 1) grid = 1;
    return launch_pdl(k, (unsigned)grid, 256u, smem, st, a);
}

// Tensor map of a row-major [rows, cols] 16-bit tensor in 128x128 boxes, from
// the driver's encoder (looked up once through the runtime).
static cudaError_t encode_tile_map(CUtensorMap* tm, const void* x, int64_t rows, int64_t cols) {
    static const PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            p = nullptr;
        }
        return (PFN_cuTensorMapEncodeTiled_v12000)p;
    }();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {128, 128};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), gdim, gstride,
                              box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorNotSupported;
}

// FP8 128x128 tiles of 16-bit inputs (k_fp8_tile_tma). Needs cols % 8 == 0
// (16-byte row stride), x 16-byte and e4m3 8-byte aligned, and dimensions
// the tensor map can describe.
template <class T>
static cudaError_t tile_entry(const void* x, int64_t rows, int64_t cols, uint8_t* e4m3,
                              float* scale, cudaStream_t st) {
    if constexpr (sizeof(T) != 2) {
        return cudaErrorNotSupported;
    } else {
        if (cols % 8 != 0 || ((uintptr_t)x & 15u) || ((uintptr_t)e4m3 & 7u)) return cudaErrorNotSupported;
        if (rows <= 0 || cols <= 0 || rows > 0x7FFFFF80ll || cols > 0x7FFFFF80ll) return cudaErrorNotSupported;
        TileArgs a;
        a.rows = rows; a.cols = cols;
        a.nbc = (cols + 127) / 128;
        a.n_tiles = ((rows + 127) / 128) * a.nbc;
        a.e4m3 = e4m3; a.scale = scale;
        CUtensorMap tm;
        const cudaError_t me = encode_tile_map(&tm, x, rows, cols);
        if (me != cudaSuccess) return me;
        const size_t smem = 128 + (size_t)BQ_TILE_STAGES * 128 * 256;
        auto k = k_fp8_tile_tma<T>;
        static const cudaError_t attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (attr != cudaSuccess) return attr;
        static unsigned long long occ[8];
        const int bps = occupancy_for((const void*)k, smem, occ);
        if (bps < 1) return cudaErrorNotSupported;
        int64_t grid = (int64_t)sm_count() * bps;
        if (grid > a.n_tiles) grid = a.n_tiles;
        k<<<(unsigned)grid, 256, smem, st>>>(tm, a);
        return cudaGetLastError();
    }
}

// FP8 per-tensor store (k_fp8t_pipe); the consumer of the range kernel when
// the scale is dynamic (launch_pdl).
template <class T>
static cudaError_t fp8t_entry(const void* x, int64_t n, uint8_t* e4m3, float* scale,
                              const unsigned long long* rec, int from_rec, cudaStream_t st) {
    constexpr int VEC = Traits<T>::VEC;
    Fp8TArgs a{x, n, e4m3, scale, rec, from_rec};
    const bool vec = (((uintptr_t)x & 15u) == 0) && (((uintptr_t)e4m3 % VEC) == 0);
    if (vec) {
        const size_t smem = 128 + (size_t)FP8T_STAGES * FP8T_CHUNK;
        auto k = k_fp8t_pipe<T>;
        static const cudaError_t attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (attr != cudaSuccess) return attr;
        static unsigned long long occ[8];
        const int bps = occupancy_for((const void*)k, smem, occ);
        if (bps < 1) return cudaErrorNotSupported;
        const int64_t n_chunks = (n / VEC * 16 + FP8T_CHUNK - 1) / FP8T_CHUNK;
        int64_t grid = (int64_t)sm_count() * bps;
        if (grid > n_chunks) grid = n_chunks;
        if (grid < 1) grid = 1;
        if (from_rec) return launch_pdl(k, (unsigned)grid, 256u, smem, st, a);
        k<<<(unsigned)grid, 256, smem, st>>>(a);
        return cudaGetLastError();
    }
    int64_t grid = (n + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    auto k = k_fp8_tensor_scalar<T>;
    if (from_rec) return launch_pdl(k, (unsigned)grid, 256u, 0, st, a);
    k<<<(unsigned)grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

// Entry points of one dtype's translation unit.
template <class T>
cudaError_t pipe_dyn_entry(int pk, bool sym, const PipeArgs& a, cudaStream_t st) {
    return pipe_dt<T>(pk, sym, a, st);
}

template <class T>
cudaError_t pipe_map_entry(int op, const MapArgs& m, cudaStream_t st) {
    const int in_esz = (op == OP_DEQ) ? 1 : (int)sizeof(T);
    // Packed 4-bit codes: only the group-tiled dequantize reads them (whole
    // 16-byte runs of codes per group); packed quantize stays element-wise.
    const bool packed = m.cfg.packed && (op == OP_DEQ || op == OP_QUANT);
    if (packed && op != OP_DEQ) return cudaErrorNotSupported;
    const int64_t a_bytes = (m.G * in_esz) >> (packed ? 1 : 0);
    if (m.n_seg > 0 && a_bytes % 16 == 0) {
        const cudaError_t e = seg_map_dt<T>(op, m, st);
        if (e != cudaErrorNotSupported || packed) return e;
    }
    if (packed) return cudaErrorNotSupported;
    return map_pipe_dt<T>(op, m.ranges ? PS_RANGE : PS_STATIC, m, st);
}

// ------------------------------------------------------------ column groups
// Column groups (groups of GS consecutive rows at one column of a row-major
// [rows, inner] tensor: the [K, N]-stored weight grouped along K) with
// dynamic scales. Tiles of GS rows x CW columns (NT * 64 bytes: 8 KB with
// 128-thread CTAs, so that a block barrier holds four warps) reach shared memory
// through 2D TMA into a ring of BQ_COL_STAGES slots; columns past `inner`
// read as zero. A thread holds COL_RPT rows of one 16-byte column vector
// (RS = GS / 4 lanes down the rows, CVN = NT / RS vectors across), so a
// tile's values sit in registers once and its slot is refilled before the
// tile is reduced. The range runs down each column: packed 16-bit max / min
// per thread, shuffles between the lanes of a column within a warp, then the
// warps' partials through shared memory; one thread per column (pair)
// derives the scale and zero-point, and the codes are encoded on f32 pairs.
#ifndef BQ_COL_STAGES
#define BQ_COL_STAGES 3
#endif
#ifndef BQ_COL_MINB
#define BQ_COL_MINB 1
#endif
constexpr int COLT_RPT = 4;

struct ColTileArgs {
    int64_t inner, n_ct, n_tiles;
    IntCfg cfg;
    float* scale;
    uint8_t* zp;
    void* out;
};

#ifndef BQ_COLT_NT
#define BQ_COLT_NT 128
#endif
template <class T, int GS> struct ColTileGeom {
    static constexpr int NT = BQ_COLT_NT;               // threads per CTA
    static constexpr int W = Traits<T>::VEC;
    static constexpr int RS = GS / COLT_RPT;            // lanes down the rows
    static constexpr int CVN = NT / RS;                 // vectors across a tile row
    static constexpr int CW = CVN * W;                  // columns per tile
    static constexpr bool H = sizeof(T) == 2;
    static constexpr int NP = H ? W / 2 : W;            // range words per thread
    static constexpr int NWORDS = CVN * NP;             // range words per tile row
    static constexpr uint32_t SLOT = (uint32_t)GS * CW * sizeof(T);
    static constexpr int RED_OFF = 64;
    static constexpr int PAR_OFF = RED_OFF + 2 * 8 * NWORDS * 4;
    static constexpr int NPAR = 6;                      // per-column parameter arrays
    static constexpr int RING_OFF = ((PAR_OFF + NPAR * CW * 4) + 1023) / 1024 * 1024;
    static_assert(CW <= 256 && (CW * sizeof(T)) % 16 == 0, "TMA box");
    static_assert(SLOT == (uint32_t)NT * 64, "slot size");
};

template <class T>
__device__ __forceinline__ uint32_t col_pk_max(uint32_t a, uint32_t b) {
    if constexpr (sizeof(T) == 2) return pk_hi<T, false, false>(a, b);
    else return __float_as_uint(fmaxf(__uint_as_float(a), __uint_as_float(b)));
}
template <class T>
__device__ __forceinline__ uint32_t col_pk_min(uint32_t a, uint32_t b) {
    if constexpr (sizeof(T) == 2) return pk_lo<T, false>(a, b);
    else return __float_as_uint(fminf(__uint_as_float(a), __uint_as_float(b)));
}
// The two (16-bit) or one (f32) values of a range word.
template <class T>
__device__ __forceinline__ void col_word_vals(uint32_t w, float& v0, float& v1) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) unpack_bf16x2(w, v0, v1);
    else if constexpr (std::is_same<T, __half>::value) unpack_f16x2(w, v0, v1);
    else { v0 = __uint_as_float(w); v1 = 0.0f; }
}

template <class T, int OP, int GS>
__global__ void __launch_bounds__(BQ_COLT_NT, BQ_COL_MINB) k_col_tma(const __grid_constant__ CUtensorMap tm, ColTileArgs a) {
    using G = ColTileGeom<T, GS>;
    constexpr int W = G::W, RS = G::RS, CVN = G::CVN, CW = G::CW, NP = G::NP, NWORDS = G::NWORDS;
    constexpr int S = BQ_COL_STAGES;
    constexpr uint32_t SLOT = G::SLOT;
    constexpr int NW = G::NT / 32;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint32_t* red_hi = reinterpret_cast<uint32_t*>(smem + G::RED_OFF);      // [NW][NWORDS]
    uint32_t* red_lo = red_hi + NW * NWORDS;
    // Per-column parameters, each array [CW]: scale, -scale, RN(1/scale),
    // qmin - zp, qmax - zp, zp (floats; a column pair reads as one 8-byte load).
    float* cs = reinterpret_cast<float*>(smem + G::PAR_OFF);
    float* cns = cs + CW;
    float* cy = cns + CW;
    float* clo = cy + CW;
    float* chi = clo + CW;
    float* czf = chi + CW;
    uint8_t* ring = smem + G::RING_OFF;
    const int tid = threadIdx.x;
    const int cv = tid % CVN, rl = tid / CVN;
    const int wid = tid >> 5, lane = tid & 31;
    const int64_t grid = gridDim.x;
    const float qlo = (float)a.cfg.qmin, qhi = (float)a.cfg.qmax;
    const bool sym = a.cfg.symmetric != 0;
    // Divisor of the scale: qmax (symmetric) or qmax - qmin.
    const Recip Rq = make_recip(sym ? qhi : (float)(a.cfg.qmax - a.cfg.qmin));

    if (tid == 0) {
        for (int i = 0; i < S; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int slot_i, int64_t tile) {
        const uint32_t bar = smem_addr(&bars[slot_i]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(SLOT) : "memory");
        tma_load_2d(smem_addr(ring + (size_t)slot_i * SLOT), &tm, (int)((tile % a.n_ct) * CW),
                    (int)((tile / a.n_ct) * GS), bar);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            const int64_t t = blockIdx.x + (int64_t)i * grid;
            if (t >= a.n_tiles) break;
            issue(i, t);
        }
    }

    int slot = 0;
    uint32_t parity = 0;
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += grid) {
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        const uint32_t sbase = smem_addr(ring + (size_t)slot * SLOT) + (uint32_t)(cv * 16);
        U4 raw[COLT_RPT];
#pragma unroll
        for (int j = 0; j < COLT_RPT; ++j)
            raw[j] = ld_shared16(sbase + (uint32_t)((rl + j * RS) * CW * (int)sizeof(T)));
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s2 = slot;
                uint32_t p2 = parity;
                for (int i = 0; i < S; ++i) {
                    const int64_t t2 = tile + (int64_t)i * grid;
                    if (t2 >= a.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s2]), p2);
                    if (++s2 == S) { s2 = 0; p2 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        // Every thread holds its vectors: refill the slot with tile + S now.
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < a.n_tiles) {
                fence_proxy_async();
                issue(slot, next);
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }

        const int64_t ct = tile % a.n_ct, ob = tile / a.n_ct;
        const int64_t col0 = ct * CW;
        // ---- range of this thread's columns over its rows (NaN skipped)
        uint32_t hw[NP], lw[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            uint32_t h = 0u, l = 0u;
#pragma unroll
            for (int j = 0; j < COLT_RPT; ++j) {
                const uint32_t wj[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
                h = col_pk_max<T>(h, wj[p]);
                l = col_pk_min<T>(l, wj[p]);
            }
            hw[p] = h;
            lw[p] = l;
        }
#pragma unroll
        for (int o = CVN; o < 32; o <<= 1) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                hw[p] = col_pk_max<T>(hw[p], __shfl_xor_sync(0xffffffffu, hw[p], o));
                lw[p] = col_pk_min<T>(lw[p], __shfl_xor_sync(0xffffffffu, lw[p], o));
            }
        }
        if (lane < CVN) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                red_hi[wid * NWORDS + cv * NP + p] = hw[p];
                red_lo[wid * NWORDS + cv * NP + p] = lw[p];
            }
        }
        __syncthreads();
        // ---- one thread per column: the tile's column parameters (the two
        // threads of a 16-bit column pair reduce the same range words)
        bool slow_col = false;
        constexpr int CPW = G::H ? 2 : 1;     // columns per range word
        static_assert(NWORDS * CPW <= G::NT, "one thread per column");
        if (tid < NWORDS * CPW) {
            const int wd = tid / CPW;
            uint32_t h = red_hi[wd], l = red_lo[wd];
#pragma unroll
            for (int w = 1; w < NW; ++w) {
                h = col_pk_max<T>(h, red_hi[w * NWORDS + wd]);
                l = col_pk_min<T>(l, red_lo[w * NWORDS + wd]);
            }
            float h0, h1, l0, l1;
            col_word_vals<T>(h, h0, h1);
            col_word_vals<T>(l, l0, l1);
            {
                const int u = tid % CPW;
                const int c = tid;
                // Scale fl(amax/qmax) or fl(fl(max'-min')/(qmax-qmin)) and
                // zero-point, each quotient through a reciprocal chain
                // (exact for a normal dividend; IEEE division outside).
                const float hi = u ? h1 : h0, nlo = -(u ? l1 : l0);
                const float num = sym ? fmaxf(hi, nlo) : __fadd_rn(hi, nlo);
                float sc = (num >= 0x1p-100f && num <= 0x1p100f) ? div_chain(num, Rq) : div_slow(num, Rq.s);
                if (sc == 0.0f) sc = 1.0f;
                const Recip R = make_recip(sc);
                int zp = 0;
                if (!sym) {
                    const float m = R.fast ? div_chain(-nlo, R) : __fdiv_rn(-nlo, sc);
                    const float zf = fminf(fmaxf(__fsub_rn(qlo, rintf(m)), qlo), qhi);   // NaN -> qmin
                    zp = (int)zf;
                }
                cs[c] = sc;
                cns[c] = -sc;
                cy[c] = R.y;
                clo[c] = qlo - (float)zp;
                chi[c] = qhi - (float)zp;
                czf[c] = (float)zp;
                slow_col = slow_col || !R.fast;
                if (col0 + c < a.inner) {
                    a.scale[ob * a.inner + col0 + c] = sc;
                    if (a.zp) a.zp[ob * a.inner + col0 + c] = (uint8_t)zp;
                }
            }
        }
        // The barrier also tells every thread whether a scale of this tile
        // lies outside the reciprocal chain's range.
        const bool tile_slow = __syncthreads_or(slow_col) != 0;
        if (col0 + cv * W >= a.inner) continue;

        // ---- codes: each column pair on f32 pairs
        const int64_t obase = (ob * GS + rl) * a.inner + col0 + cv * W;
        if (!tile_slow) {
            uint32_t cwd[COLT_RPT][(W + 3) / 4];
            uint32_t ow[COLT_RPT][4];
            const F2 magic2 = f2_bcast(kMagic);
#pragma unroll
            for (int p = 0; p < W / 2; ++p) {
                const int c = cv * W + 2 * p;
                const float2 lo = *reinterpret_cast<const float2*>(clo + c);
                const float2 hi = *reinterpret_cast<const float2*>(chi + c);
                Recip2 R2;
                R2.y = *reinterpret_cast<const F2*>(cy + c);
                R2.ns = *reinterpret_cast<const F2*>(cns + c);
                const F2 zf2 = *reinterpret_cast<const F2*>(czf + c);
                const F2 s2 = *reinterpret_cast<const F2*>(cs + c);
#pragma unroll
                for (int j = 0; j < COLT_RPT; ++j) {
                    F2 xp[W / 2];
                    widen_pairs<T>(raw[j], xp);
                    float q0, q1;
                    f2_split(div_chain2(xp[p], R2), q0, q1);
                    q0 = fminf(fmaxf(q0, lo.x), hi.x);        // NaN -> qmin
                    q1 = fminf(fmaxf(q1, lo.y), hi.y);
                    const F2 t = f2_add(f2_pack(q0, q1), magic2);   // round(q) + 1.5 * 2^23
                    if constexpr (OP == OP_QUANT) {
                        uint32_t b0, b1;
                        f2_split_bits(f2_add(t, zf2), b0, b1);      // + zp, exact; low byte = code
                        const uint32_t pair = __byte_perm(b0, b1, 0x0040);  // codes in bytes 0, 1
                        uint32_t& wd = cwd[j][(2 * p) / 4];
                        wd = ((2 * p) % 4 == 0) ? pair : __byte_perm(wd, pair, 0x5410);
                    } else {
                        float o0, o1;
                        f2_split(f2_mul(f2_sub(t, magic2), s2), o0, o1);
                        if constexpr (sizeof(T) == 2) {
                            ow[j][p] = std::is_same<T, __nv_bfloat16>::value ? pack_bf16x2(o0, o1) : pack_f16x2(o0, o1);
                        } else {
                            ow[j][2 * p] = __float_as_uint(o0);
                            ow[j][2 * p + 1] = __float_as_uint(o1);
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < COLT_RPT; ++j) {
                const int64_t e = obase + (int64_t)j * RS * a.inner;
                if constexpr (OP == OP_QUANT) {
                    uint8_t* q = code_ptr((uint8_t*)a.out, e, a.cfg.packed);
                    if (a.cfg.packed) {
                        if constexpr (W == 8) st4(q, nib_pack4(cwd[j][0]) | (nib_pack4(cwd[j][1]) << 16));
                        else *reinterpret_cast<unsigned short*>(q) = (unsigned short)nib_pack4(cwd[j][0]);
                    } else {
                        if constexpr (W == 8) st8(q, cwd[j][0], cwd[j][1]);
                        else st4(q, cwd[j][0]);
                    }
                } else {
                    st16((T*)a.out + e, U4{ow[j][0], ow[j][1], ow[j][2], ow[j][3]});
                }
            }
        } else {
            // A scale outside the reciprocal chain's range (tiny or infinite):
            // IEEE division per element.
#pragma unroll
            for (int j = 0; j < COLT_RPT; ++j) {
                float v[W], o[W];
                uint32_t code[W];
                load_vec<T>(raw[j], v);
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const int c = cv * W + k;
                    IntParams ip = make_int_params(a.cfg.qmin, a.cfg.qmax, (int)czf[c]);
                    Recip R;
                    R.s = cs[c];
                    R.y = cy[c];
                    const float m = fabsf(R.s);
                    R.fast = (m >= 0x1p-64f) && (m <= 0x1p64f);
                    const float t = rounded_rne(div_any(v[k], R), ip);
                    code[k] = code_from_rounded(t, ip.zp);
                    o[k] = dequant_from_rounded(t, R.s);
                }
                const int64_t e = obase + (int64_t)j * RS * a.inner;
                if constexpr (OP == OP_QUANT) {
                    st_codes<W>(code_ptr((uint8_t*)a.out, e, a.cfg.packed), code, a.cfg.packed);
                } else {
                    st16((T*)a.out + e, pack_vec<T>(o));
                }
            }
        }
    }
}

// Tensor map of a row-major [rows, cols] tensor of 1-, 2- or 4-byte elements
// in boxes of box_rows x box_cols, zero fill outside (no multicast).
static cudaError_t encode_map_2d(CUtensorMap* tm, const void* x, int64_t rows, int64_t cols, int esz,
                                 uint32_t box_cols, uint32_t box_rows) {
    static const PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            p = nullptr;
        }
        return (PFN_cuTensorMapEncodeTiled_v12000)p;
    }();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * (cuuint64_t)esz};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = encode(tm, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                  : (esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32),
                              2, const_cast<void*>(x), gdim, gstride, box, estride,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorNotSupported;
}

template <class T, int OP, int GS>
static cudaError_t col_tma_launch(const ColPipeArgs& p, cudaStream_t st) {
    using G = ColTileGeom<T, GS>;
    ColTileArgs a;
    a.inner = p.inner;
    a.n_ct = (p.inner + G::CW - 1) / G::CW;
    a.n_tiles = (p.rows / GS) * a.n_ct;
    a.cfg = p.cfg;
    a.scale = p.scale;
    a.zp = p.zp;
    a.out = p.out;
    CUtensorMap tm;
    const cudaError_t me = encode_map_2d(&tm, p.x, p.rows, p.inner, (int)sizeof(T), G::CW, GS);
    if (me != cudaSuccess) return me;
    const size_t smem = (size_t)G::RING_OFF + (size_t)BQ_COL_STAGES * G::SLOT;
    auto k = k_col_tma<T, OP, GS>;
    static const cudaError_t attr = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    static unsigned long long occ[8];
    const int bps = occupancy_for((const void*)k, smem, occ, G::NT);
    if (bps < 1) return cudaErrorNotSupported;
    int64_t grid = (int64_t)sm_count() * bps;
    if (grid > a.n_tiles) grid = a.n_tiles;
    if (grid < 1) grid = 1;
    k<<<(unsigned)grid, G::NT, smem, st>>>(tm, a);
    return cudaGetLastError();
}

// Column groups with dynamic scales through k_col_tma: 16-bit or f32 x, gs
// in {32, 64, 128, 256}, round-to-nearest-even, whole vectors per row,
// aligned operands; cudaErrorNotSupported otherwise.
template <class T>
static cudaError_t col_tma_entry(int op, const ColPipeArgs& p, cudaStream_t st) {
    constexpr int W = Traits<T>::VEC;
    if (sizeof(T) == 8 || p.cfg.rhaz || (op != OP_QUANT && op != OP_FAKE)) return cudaErrorNotSupported;
    if (p.inner % W != 0 || ((uintptr_t)p.x & 15u)) return cudaErrorNotSupported;
    if (op == OP_QUANT ? ((uintptr_t)p.out % W) != 0 : ((uintptr_t)p.out & 15u) != 0) return cudaErrorNotSupported;
    if (p.rows <= 0 || p.inner <= 0 || p.rows > 0x7FFFFF00ll || p.inner > 0x7FFFFF00ll) return cudaErrorNotSupported;
    if (p.rows % p.gs != 0) return cudaErrorNotSupported;
    switch (p.gs) {
        case 32: return op == OP_QUANT ? col_tma_launch<T, OP_QUANT, 32>(p, st) : col_tma_launch<T, OP_FAKE, 32>(p, st);
        case 64: return op == OP_QUANT ? col_tma_launch<T, OP_QUANT, 64>(p, st) : col_tma_launch<T, OP_FAKE, 64>(p, st);
        case 128: return op == OP_QUANT ? col_tma_launch<T, OP_QUANT, 128>(p, st) : col_tma_launch<T, OP_FAKE, 128>(p, st);
        case 256: return op == OP_QUANT ? col_tma_launch<T, OP_QUANT, 256>(p, st) : col_tma_launch<T, OP_FAKE, 256>(p, st);
    }
    return cudaErrorNotSupported;
}

// ------------------------------------------------------------ column groups, static parameters
// Every column-group op whose parameters are given (static quantize and
// fake-quantize, dequantize, the STE backwards, dequantize backward): tiles of
// gs rows x CW columns of the input (and of dy for the backwards) through 2D
// TMA into a ring of BQ_COLM_STAGES slots. The geometry is set per launch:
// RS = min(32, gs) lanes down the rows (a power of two), CVN = 256 / RS
// 16-byte column vectors across (CW = CVN * VEC columns <= 256, the widest
// box). The tile's CW scales (and zero-points) come into the same slot by
// TMA; a thread reads its W columns' parameters from there once per tile,
// walks its rows of the slot (shared memory), and writes its outputs; the
// slot is refilled once every thread is done with it. The STE backwards with
// normal scales take the mask from the exact quotient on f32 pairs. The ring holds as
// many slots (2..6) as fit in about BQ_COLM_RING_BYTES, so that three CTAs
// share an SM whatever the slot size.
#ifndef BQ_COLM_RING_BYTES
#define BQ_COLM_RING_BYTES 65536
#endif

struct ColMapArgs {
    int64_t inner, n_ct, n_tiles;
    int gs, rs_log2, cvn, cw;       // rows per group, log2(RS), vectors across, columns per tile
    uint32_t slot_a, slot_b;        // bytes of input a / dy in one slot (as copied)
    uint32_t off_b, slot_bytes;     // dy's offset in a slot and the slot stride (128-byte multiples)
    uint32_t off_s, off_z;          // the tile's scales (CW f32) and zero-points (CW bytes) in a slot
    int has_zp;                     // zero-points are copied (asymmetric codes)
    int stages;                     // ring slots
    IntCfg cfg;
    void* out;
};

template <class T, int OP>
__global__ void __launch_bounds__(256) k_col_tma_map(const __grid_constant__ CUtensorMap tma,
                                                     const __grid_constant__ CUtensorMap tmb,
                                                     const __grid_constant__ CUtensorMap tms,
                                                     const __grid_constant__ CUtensorMap tmz,
                                                     ColMapArgs a) {
    constexpr int W = Traits<T>::VEC;
    constexpr bool TWO = (OP == OP_QBWD || OP == OP_FBWD);
    constexpr bool NEEDR = (OP != OP_DEQ && OP != OP_DBWD);
    const int S = a.stages;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint8_t* ring = smem + 1024;
    const uint32_t slot_bytes = a.slot_bytes;
    const uint32_t tx_bytes = a.slot_a + a.slot_b + (uint32_t)a.cw * 4u + (a.has_zp ? (uint32_t)a.cw : 0u);
    const int tid = threadIdx.x;
    const int RS = 1 << a.rs_log2;
    const int cv = tid & (a.cvn - 1), rl = tid / a.cvn;
    const int64_t grid = gridDim.x;
    const int pk = a.cfg.packed;
    // bytes per element of input a in shared memory, as a right shift of
    // (elements * sizeof(T)): codes 1 byte (or half a byte when packed)
    const int a_row_bytes = (OP == OP_DEQ) ? (a.cw >> pk) : a.cw * (int)sizeof(T);
    const int b_row_bytes = a.cw * (int)sizeof(T);

    if (tid == 0) {
        for (int i = 0; i < S; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int slot_i, int64_t tile) {
        const uint32_t bar = smem_addr(&bars[slot_i]);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(tx_bytes) : "memory");
        const int c0 = (int)((tile % a.n_ct) * a.cw);
        const int r0 = (int)((tile / a.n_ct) * a.gs);
        uint8_t* dst = ring + (size_t)slot_i * slot_bytes;
        tma_load_2d(smem_addr(dst), &tma, (OP == OP_DEQ) ? (c0 >> pk) : c0, r0, bar);
        if (TWO) tma_load_2d(smem_addr(dst + a.off_b), &tmb, c0, r0, bar);
        // the block's row of scales (and zero-points) for these columns
        tma_load_2d(smem_addr(dst + a.off_s), &tms, c0, (int)(tile / a.n_ct), bar);
        if (a.has_zp) tma_load_2d(smem_addr(dst + a.off_z), &tmz, c0, (int)(tile / a.n_ct), bar);
    };
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            const int64_t t = blockIdx.x + (int64_t)i * grid;
            if (t >= a.n_tiles) break;
            issue(i, t);
        }
    }

    int slot = 0;
    uint32_t parity = 0;
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += grid) {
        const int64_t ct = tile % a.n_ct, ob = tile / a.n_ct;
        const int64_t col = ct * a.cw + (int64_t)cv * W;         // this thread's first column
        const bool col_ok = col < a.inner;
        const bool ok = mbar_wait(smem_addr(&bars[slot]), parity);
        if (ok && col_ok) {
            // This thread's columns' parameters, copied in with the tile.
            const uint8_t* sp = ring + (size_t)slot * slot_bytes;
            float sk[W], yk[W];
            int zk[W];
#pragma unroll
            for (int k = 0; k < W; ++k) {
                sk[k] = reinterpret_cast<const float*>(sp + a.off_s)[cv * W + k];
                const uint8_t zb = a.has_zp ? sp[a.off_z + cv * W + k] : (uint8_t)0;
                zk[k] = (OP == OP_DBWD) ? 0 : (a.cfg.q_signed ? (int)(int8_t)zb : (int)zb);
            }
            GState st[W];
#pragma unroll
            for (int k = 0; k < W; ++k) {
                if constexpr (NEEDR) yk[k] = __frcp_rn(sk[k]);
                else yk[k] = 0.0f;
                st[k].seg = 0;
                st[k].s = sk[k];
                st[k].zp = zk[k];
                st[k].R.s = sk[k];
                st[k].R.y = yk[k];
                const float m = fabsf(sk[k]);
                st[k].R.fast = (m >= 0x1p-64f) && (m <= 0x1p64f);
                st[k].ip = make_int_params(a.cfg.qmin, a.cfg.qmax, zk[k]);
                st[k].x_lo = st[k].x_hi = 0.0f;
                st[k].mfast = false;
                st[k].fast = false;
            }
            const uint8_t* sa = ring + (size_t)slot * slot_bytes;
            const uint8_t* sb = sa + a.off_b;
            bool all_fast = true;
#pragma unroll
            for (int k = 0; k < W; ++k) all_fast = all_fast && st[k].R.fast;
            bool lean = false;
            if constexpr (TWO) {
                if (all_fast && !a.cfg.rhaz) {
                    // STE backwards on f32 pairs: the mask from the exact quotient
                    // (the reciprocal chain; a NaN or overflowing quotient clamps
                    // below the code range: masked, as the exact quotient would be).
                    Recip2 R2[W / 2];
                    float lo[W];
#pragma unroll
                    for (int p = 0; p < W / 2; ++p) {
                        R2[p].y = f2_pack(yk[2 * p], yk[2 * p + 1]);
                        R2[p].ns = f2_pack(-sk[2 * p], -sk[2 * p + 1]);
                    }
#pragma unroll
                    for (int k = 0; k < W; ++k) lo[k] = st[k].ip.lo;
                    const float span = (float)(a.cfg.qmax - a.cfg.qmin);
                    const F2 magic2 = f2_bcast(kMagic);
                    for (int r = rl; r < a.gs; r += RS) {
                        const int64_t e = (ob * a.gs + r) * a.inner + col;
                        F2 xp[W / 2], dp[W / 2];
                        widen_pairs<T>(ld_shared16(smem_addr(sa + r * a_row_bytes + cv * 16)), xp);
                        widen_pairs<T>(ld_shared16(smem_addr(sb + r * b_row_bytes + cv * 16)), dp);
                        float o[W];
#pragma unroll
                        for (int p = 0; p < W / 2; ++p) {
                            float q0, q1;
                            f2_split(div_chain2(xp[p], R2[p]), q0, q1);
                            const float l0 = lo[2 * p], l1 = lo[2 * p + 1];
                            q0 = fminf(fmaxf(q0, l0 - 1.0f), l0 + span + 1.0f);      // NaN -> below the range
                            q1 = fminf(fmaxf(q1, l1 - 1.0f), l1 + span + 1.0f);
                            float k0, k1;
                            f2_split(f2_sub(f2_add(f2_pack(q0, q1), magic2), magic2), k0, k1);   // round half even
                            const float m0 = (k0 > l0 && k0 < l0 + span) ? 1.0f : 0.0f;
                            const float m1 = (k1 > l1 && k1 < l1 + span) ? 1.0f : 0.0f;
                            F2 g = dp[p];
                            if constexpr (OP == OP_QBWD) g = f2_mul(g, R2[p].y);
                            f2_split(f2_mul(g, f2_pack(m0, m1)), o[2 * p], o[2 * p + 1]);
                        }
                        st16((T*)a.out + e, pack_vec<T>(o));
                    }
                    lean = true;
                }
            }
            for (int r = lean ? a.gs : rl; r < a.gs; r += RS) {
                const int64_t e = (ob * a.gs + r) * a.inner + col;
                float o[W];
                uint32_t cw[W];
                if constexpr (OP == OP_DEQ) {
                    uint32_t w[2];
                    const uint32_t ad = smem_addr(sa + r * a_row_bytes + ((cv * W) >> pk));
                    if (pk) {
                        if constexpr (W == 8) {
                            uint32_t v;
                            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(ad));
                            w[0] = nib_spread(v & 0xFFFFu, a.cfg.q_signed);
                            w[1] = nib_spread(v >> 16, a.cfg.q_signed);
                        } else {
                            unsigned short v;
                            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(ad));
                            w[0] = nib_spread(v, a.cfg.q_signed);
                            w[1] = 0u;
                        }
                    } else if constexpr (W == 8) {
                        asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(ad));
                    } else {
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(ad));
                        w[1] = 0u;
                    }
#pragma unroll
                    for (int k = 0; k < W; ++k) o[k] = deq_code_f(w[k / 4], k % 4, st[k], a.cfg.q_signed);
                } else {
                    float xa[W], xb[W];
                    load_vec<T>(ld_shared16(smem_addr(sa + r * a_row_bytes + cv * 16)), xa);
                    if constexpr (TWO) load_vec<T>(ld_shared16(smem_addr(sb + r * b_row_bytes + cv * 16)), xb);
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        if (a.cfg.rhaz) o[k] = elem_f<OP, true>(xa[k], TWO ? xb[k] : 0.0f, st[k], &cw[k]);
                        else o[k] = elem_f<OP, false>(xa[k], TWO ? xb[k] : 0.0f, st[k], &cw[k]);
                    }
                }
                if constexpr (OP == OP_QUANT) st_codes<W>(code_ptr((uint8_t*)a.out, e, pk), cw, pk);
                else st16((T*)a.out + e, pack_vec<T>(o));
            }
        }
        // Every thread is done with the slot: refill it with tile + S (and a
        // wait that gave up ends the kernel).
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_pipe_error, 1u);
                int s2 = slot;
                uint32_t p2 = parity;
                for (int i = 0; i < S; ++i) {
                    const int64_t t2 = tile + (int64_t)i * grid;
                    if (t2 >= a.n_tiles) break;
                    mbar_wait(smem_addr(&bars[s2]), p2);
                    if (++s2 == S) { s2 = 0; p2 ^= 1u; }
                }
            }
            __syncthreads();
            return;
        }
        if (tid == 0) {
            const int64_t next = tile + (int64_t)S * grid;
            if (next < a.n_tiles) {
                fence_proxy_async();
                issue(slot, next);
            }
        }
        if (++slot == S) { slot = 0; parity ^= 1u; }
    }
}

// Column groups with static parameters through k_col_tma_map: f32 / f16 /
// bf16 float tensors, 8 <= gs <= 256, whole vectors per row, 16-byte aligned
// operands; cudaErrorNotSupported otherwise. a: x, codes (OP_DEQ) or dy
// (OP_DBWD); b: dy (OP_QBWD, OP_FBWD); out: codes (OP_QUANT) or a tensor of T.
template <class T>
static cudaError_t col_map_entry(int op, const void* ap, const void* bp, int64_t rows, int64_t inner,
                                 int64_t gs, IntCfg cfg, const float* scale, const uint8_t* zp,
                                 void* out, cudaStream_t st) {
    constexpr int W = Traits<T>::VEC;
    if constexpr (sizeof(T) == 8) {
        return cudaErrorNotSupported;
    } else {
        const bool two = (op == OP_QBWD || op == OP_FBWD);
        if (gs < 8 || gs > 256 || rows % gs != 0 || inner % W != 0) return cudaErrorNotSupported;
        if (rows <= 0 || inner <= 0 || rows > 0x7FFFFF00ll || inner > 0x7FFFFF00ll) return cudaErrorNotSupported;
        if (((uintptr_t)ap & 15u) || (two && ((uintptr_t)bp & 15u)) || ((uintptr_t)out & 15u))
            return cudaErrorNotSupported;
        int rs_log2 = 0;
        while ((2 << rs_log2) <= gs && (1 << (rs_log2 + 1)) <= 32) ++rs_log2;   // RS = largest power of two <= min(gs, 32)
        const int RS = 1 << rs_log2;
        const int cvn = 256 / RS;
        const int cw = cvn * W;
        if (cw > 256) return cudaErrorNotSupported;
        const int pk = cfg.packed;
        const int a_esz = (op == OP_DEQ) ? 1 : (int)sizeof(T);
        const int a_box_cols = (op == OP_DEQ) ? (cw >> pk) : cw;
        if ((a_box_cols * a_esz) % 16 != 0) return cudaErrorNotSupported;
        if (op == OP_DEQ && pk && (inner % 2 != 0)) return cudaErrorNotSupported;
        // Scales [rows / gs, inner] f32 and zero-points [rows / gs, inner]
        // bytes come in by TMA as well: 16-byte aligned, rows of whole 16 bytes.
        const bool has_zp = zp != nullptr && !cfg.symmetric && op != OP_DBWD;
        if (((uintptr_t)scale & 15u) || (has_zp && (((uintptr_t)zp & 15u) || inner % 16 != 0)))
            return cudaErrorNotSupported;
        ColMapArgs a;
        a.inner = inner;
        a.n_ct = (inner + cw - 1) / cw;
        a.n_tiles = (rows / gs) * a.n_ct;
        a.gs = (int)gs;
        a.rs_log2 = rs_log2;
        a.cvn = cvn;
        a.cw = cw;
        a.slot_a = (uint32_t)((int64_t)gs * a_box_cols * a_esz);
        a.slot_b = two ? (uint32_t)((int64_t)gs * cw * sizeof(T)) : 0u;
        a.off_b = (a.slot_a + 127u) & ~127u;                 // TMA destinations on 128-byte boundaries
        a.off_s = (a.off_b + a.slot_b + 127u) & ~127u;
        a.off_z = (a.off_s + (uint32_t)cw * 4u + 127u) & ~127u;
        a.has_zp = has_zp ? 1 : 0;
        a.slot_bytes = (a.off_z + (uint32_t)cw + 127u) & ~127u;
        a.stages = (int)(BQ_COLM_RING_BYTES / a.slot_bytes);
        if (a.stages > 6) a.stages = 6;
        if (a.stages < 2) a.stages = 2;
        a.cfg = cfg;
        a.out = out;
        CUtensorMap ta, tb, ts, tz;
        const int64_t a_cols = (op == OP_DEQ) ? (inner >> pk) : inner;
        cudaError_t e = encode_map_2d(&ta, ap, rows, a_cols, a_esz, (uint32_t)a_box_cols, (uint32_t)gs);
        if (e != cudaSuccess) return e;
        if (two) {
            e = encode_map_2d(&tb, bp, rows, inner, (int)sizeof(T), (uint32_t)cw, (uint32_t)gs);
            if (e != cudaSuccess) return e;
        } else {
            tb = ta;
        }
        e = encode_map_2d(&ts, scale, rows / gs, inner, 4, (uint32_t)cw, 1u);
        if (e != cudaSuccess) return e;
        if (has_zp) {
            e = encode_map_2d(&tz, zp, rows / gs, inner, 1, (uint32_t)cw, 1u);
            if (e != cudaSuccess) return e;
        } else {
            tz = ts;
        }
        const size_t smem = 1024 + (size_t)a.stages * a.slot_bytes;
        if (smem > 200 * 1024) return cudaErrorNotSupported;
        void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, ColMapArgs) = nullptr;
        switch (op) {
            case OP_QUANT: k = k_col_tma_map<T, OP_QUANT>; break;
            case OP_FAKE: k = k_col_tma_map<T, OP_FAKE>; break;
            case OP_QBWD: k = k_col_tma_map<T, OP_QBWD>; break;
            case OP_FBWD: k = k_col_tma_map<T, OP_FBWD>; break;
            case OP_DEQ: k = k_col_tma_map<T, OP_DEQ>; break;
            case OP_DBWD: k = k_col_tma_map<T, OP_DBWD>; break;
            default: return cudaErrorNotSupported;
        }
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return cudaErrorNotSupported;
        int bps = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k, 256, smem) != cudaSuccess || bps < 1) {
            (void)cudaGetLastError();
            return cudaErrorNotSupported;
        }
        int64_t grid = (int64_t)sm_count() * bps;
        if (grid > a.n_tiles) grid = a.n_tiles;
        if (grid < 1) grid = 1;
        k<<<(unsigned)grid, 256, smem, st>>>(ta, tb, ts, tz, a);
        return cudaGetLastError();
    }
}

// ------------------------------------------------------------ bounded-wait diagnostic
// One CTA waits on an mbarrier that nothing will ever complete, `tries` times
// (each try suspends for at most about a microsecond), then records the
// give-up in g_pipe_error exactly as the pipelined kernels do and returns: the
// host-visible path of a bounded wait that runs out, with no fault and no hang.
__global__ void k_wait_diag(uint32_t tries) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    bool done = false;
    for (uint32_t i = 0; i < tries && !done; ++i) done = mbar_try_wait(smem_addr(&bar), 0u);
    if (!done) atomicOr(&g_pipe_error, 1u);
}

template <class T>
cudaError_t pipe_error_entry(unsigned int* flag) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_pipe_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_pipe_error, &zero, sizeof(unsigned int));
}

}  // namespace

#define BQ_PIPE_ENTRIES(T, NAME)                                                        \
    cudaError_t pipe_dyn_##NAME(int pk, bool sym, const PipeArgs& a, cudaStream_t st) { \
        return pipe_dyn_entry<T>(pk, sym, a, st);                                        \
    }                                                                                    \
    cudaError_t pipe_map_##NAME(int op, const MapArgs& m, cudaStream_t st) {            \
        return pipe_map_entry<T>(op, m, st);                                             \
    }                                                                                    \
    cudaError_t pipe_err_##NAME(unsigned int* flag) { return pipe_error_entry<T>(flag); }       \
    cudaError_t pipe_wait_diag_##NAME(uint32_t tries, cudaStream_t st) {                         \
        k_wait_diag<<<1, 32, 0, st>>>(tries);                                                    \
        return cudaGetLastError();                                                               \
    }                                                                                            \
    cudaError_t pipe_range_##NAME(const void* x, int64_t n, bool sym, unsigned long long* rec,   \
                                  cudaStream_t st) {                                              \
        return range_entry<T>(x, n, sym, rec, st);                                               \
    }                                                                                            \
    cudaError_t pipe_amax_##NAME(const void* x, int64_t n, unsigned long long* rec, float* amax,  \
                                 cudaStream_t st) {                                               \
        return range_entry<T>(x, n, true, rec, st, amax);                                        \
    }                                                                                            \
    cudaError_t pipe_tile_##NAME(const void* x, int64_t rows, int64_t cols, uint8_t* e4m3,       \
                                 float* scale, cudaStream_t st) {                                 \
        return tile_entry<T>(x, rows, cols, e4m3, scale, st);                                    \
    }                                                                                            \
    cudaError_t pipe_fp8t_##NAME(const void* x, int64_t n, uint8_t* e4m3, float* scale,           \
                                 const unsigned long long* rec, int from_rec, cudaStream_t st) {  \
        return fp8t_entry<T>(x, n, e4m3, scale, rec, from_rec, st);                              \
    }                                                                                            \
    cudaError_t pipe_col_##NAME(int op, const ColPipeArgs& p, cudaStream_t st) {                 \
        return col_tma_entry<T>(op, p, st);                                                      \
    }                                                                                            \
    cudaError_t pipe_colmap_##NAME(int op, const void* a, const void* b, int64_t rows,           \
                                   int64_t inner, int64_t gs, IntCfg cfg, const float* scale,    \
                                   const uint8_t* zp, void* out, cudaStream_t st) {              \
        return col_map_entry<T>(op, a, b, rows, inner, gs, cfg, scale, zp, out, st);             \
    }

}  // namespace bq
