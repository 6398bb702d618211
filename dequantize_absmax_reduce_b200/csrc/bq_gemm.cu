// W8A8 block-FP8 matrix multiply with the activation quantization fused into
// its prologue ([smile.llm.quant] Fp8BlockGemm: activations quantized on the
// fly to E4M3 with one f32 scale per 1x128 group, weights E4M3 with one f32
// scale per 128x128 tile):
//   C[i, j] = sum over k-blocks b of sa[i, b] * sw[j / 128, b] * S(i, j, b),
//   S(i, j, b) = sum over the 128 k of block b of dec(ea[i, k]) * dec(ew[j, k]).
//
// One persistent CTA per SM (512 threads, 16 warps) walks 128 x 256 tiles of
// C; per tile it streams the k-blocks of 128:
//   warp 12      TMA: bf16 / f16 activation tiles [128 rows x 2 x 64 cols]
//                (128-byte swizzle) into a 2-slot ring;
//   warp 14      TMA: E4M3 weight tiles [256 rows x 128 bytes] (128-byte
//                swizzle) into a 3-slot ring;
//   warps 0-3    prologue: thread r quantizes row r of the activation tile
//                exactly as bq_fp8_block_quantize does for a 1 x 128 block
//                (amax, s = fl(amax / 448), E4M3(fl(x / s)), the same device
//                functions) and writes the codes into the K-major,
//                128-byte-swizzled operand layout the tensor core reads, and
//                the scale into a 4-slot ring;
//   warp 13      TMEM allocation (512 columns) and, from one thread, the
//                tcgen05.mma.kind::f8f6f4 instructions (M 128, N 256, K 32;
//                four per k-block) into one of two TMEM partial buffers;
//   warps 4-11   promotion: each thread owns one row and 128 columns of the
//                tile; per k-block it reads the block's partial sums from
//                TMEM (tcgen05.ld) and adds partial * fl(sa * sw) into f32
//                registers (one FMA per element), then frees the buffer; at
//                the end of the tile it writes its row of C.
// The two TMEM buffers let the tensor core run the next k-block while the
// promotion warps drain the previous one. No multicast of any kind.
//
// Every mbarrier wait is bounded (about two seconds); a role that gives up
// sets a shared abort flag that the other roles see within microseconds,
// records the error in g_gemm_error, waits (bounded) for the copies and MMAs
// it has in flight, and the CTA frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "bq.h"
#include "bq_device.cuh"
#include "bq_internal.h"
#include "bq_quant_ops.cuh"
#include "bq_range.cuh"

namespace bq {
namespace {

__device__ unsigned int g_gemm_error;

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int SA = 2;   // activation (16-bit) slots
constexpr int SQ = 2;   // activation operand (E4M3) slots
constexpr int SW = 3;   // weight slots
constexpr int SS = 4;   // activation scale slots
constexpr int NT = 512;
constexpr uint32_t A16_BYTES = BM * BK * 2;   // two boxes of 128 rows x 64 columns
constexpr uint32_t A16_BOX = A16_BYTES / 2;
constexpr uint32_t AQ_BYTES = BM * BK;
constexpr uint32_t W_BYTES = BN * BK;
constexpr uint32_t OFF_A16 = 0;
constexpr uint32_t OFF_AQ = OFF_A16 + SA * A16_BYTES;
constexpr uint32_t OFF_W = OFF_AQ + SQ * AQ_BYTES;
constexpr uint32_t OFF_SA = OFF_W + SW * W_BYTES;
constexpr uint32_t OFF_BAR = OFF_SA + SS * BM * 4;
// Barrier indices.
constexpr int B_FULL_A = 0, B_EMPTY_A = B_FULL_A + SA, B_FULL_Q = B_EMPTY_A + SA,
              B_EMPTY_Q = B_FULL_Q + SQ, B_FULL_W = B_EMPTY_Q + SQ, B_EMPTY_W = B_FULL_W + SW,
              B_FULL_S = B_EMPTY_W + SW, B_EMPTY_S = B_FULL_S + SS, B_TFULL = B_EMPTY_S + SS,
              B_TEMPTY = B_TFULL + 2, B_MMA_DONE = B_TEMPTY + 2, N_BAR = B_MMA_DONE + 1;
constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;     // [0] TMEM base, [1] abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;     // room to align the base to 1024
constexpr uint32_t TMEM_COLS = 512;                   // two partial buffers of BN columns
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(2 * BN <= (int)TMEM_COLS, "TMEM");

// Register split (setmaxnreg): the block launches with NT x 128 registers.
// Prologue warps 0-3 keep 120, promotion warps 4-11 take 176, warps 12-15
// keep 40: 128*120 + 256*176 + 128*40 = 65536 = 512 * 128.
constexpr int REG_LAUNCH = 128, REG_PRO = 120, REG_ACC = 176, REG_CTL = 40;
static_assert(128 * REG_PRO + 256 * REG_ACC + 128 * REG_CTL == NT * REG_LAUNCH, "register split");

struct GemmArgs {
    int64_t m, n, k;
    int nkb;            // k / 128
    int mtiles, ntiles;
    int band;           // raster band height in M tiles
    int64_t n_tiles;
    const float* sw;    // [ceil(n / 128), nkb]
    void* c;
    int c_bf16;
    uint8_t* dump_q;    // optional [m, k]: operand bytes read back from shared memory
    float* dump_s;      // optional [m, nkb]
};

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t sm_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(1000u) : "memory");
    return ok != 0;
}
// Bounded wait (each try suspends for at most about a microsecond); gives up
// early once another role has set the abort flag. On giving up by itself it
// sets the flag and the device error.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag) {
    for (uint32_t i = 0; i < (1u << 21); ++i) {
        if (bar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 15u && *abort_flag) return false;
    }
    *abort_flag = 1u;
    atomicOr(&g_gemm_error, 1u);
    return false;
}
// Wait used while draining after an abort: bounded, ignores the flag.
__device__ __forceinline__ void bar_drain(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < (1u << 21); ++i)
        if (bar_try_wait(bar, parity)) return;
    atomicOr(&g_gemm_error, 1u);
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"((uint64_t)tm), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap* tm) {
    asm volatile("prefetch.tensormap [%0];" :: "l"((uint64_t)tm) : "memory");
}
__device__ __forceinline__ void st_shared16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ U4 ld_shared16(uint32_t addr) {
    U4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr) : "memory");
    return r;
}
__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void set_max_regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(N));
}
template <int N>
__device__ __forceinline__ void set_max_regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(N));
}

// tcgen05 (5th-generation tensor core, accumulators in TMEM).
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(dst_smem), "r"(cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, both K-major E4M3, f32 D.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// The mbarrier completes (one arrival) when every tcgen05 operation this
// thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}
// 16 consecutive f32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand with 128-byte rows in
// the 128-byte swizzle (8-row atoms of 1024 bytes): start address, leading
// byte offset 16 (unused by this layout), stride byte offset 1024 between
// 8-row groups, descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor: f32 accumulator, E4M3 x E4M3, both K-major,
// N = BN, M = BM, dense, no negation.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// Tile t -> (M tile, N tile): bands of `band` M tiles, walked down M first,
// so the CTAs working at one time share a few weight panels and a band of
// activation rows in L2.
__device__ __forceinline__ void tile_coords(const GemmArgs& g, int64_t t, int& mt, int& nt) {
    const int64_t per_band = (int64_t)g.band * g.ntiles;
    const int b = (int)(t / per_band);
    const int r = (int)(t - (int64_t)b * per_band);
    const int rows = min(g.band, g.mtiles - b * g.band);
    mt = b * g.band + r % rows;
    nt = r / rows;
}

template <class T>
__global__ void __launch_bounds__(NT, 1) k_fp8_gemm(const __grid_constant__ CUtensorMap tm_a,
                                                     const __grid_constant__ CUtensorMap tm_w,
                                                     const GemmArgs g) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = sm_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw_base);
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(sb + OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;
    const float* sa_ring = reinterpret_cast<const float*>(sb + OFF_SA);
    auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SA; ++i) { bar_init(bar(B_FULL_A + i), 1); bar_init(bar(B_EMPTY_A + i), 128); }
        for (int i = 0; i < SQ; ++i) { bar_init(bar(B_FULL_Q + i), 128); bar_init(bar(B_EMPTY_Q + i), 1); }
        for (int i = 0; i < SW; ++i) { bar_init(bar(B_FULL_W + i), 1); bar_init(bar(B_EMPTY_W + i), 1); }
        for (int i = 0; i < SS; ++i) { bar_init(bar(B_FULL_S + i), 128); bar_init(bar(B_EMPTY_S + i), 256); }
        for (int i = 0; i < 2; ++i) { bar_init(bar(B_TFULL + i), 1); bar_init(bar(B_TEMPTY + i), 256); }
        bar_init(bar(B_MMA_DONE), 1);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 12 && lane == 0) prefetch_map(&tm_a);
    if (warp == 14 && lane == 0) prefetch_map(&tm_w);
    if (warp == 13) tmem_alloc(base + OFF_MISC, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int nkb = g.nkb;

    if (warp < 4) {
        // ---------------------------------------------------- prologue
        set_max_regs_dec<REG_PRO>();
        const int r = threadIdx.x;                     // row of the tile
        const uint32_t swz = (uint32_t)(r & 7);
        const Recip Rq = make_recip(448.0f);
        int ia = 0, iq = 0, is = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; ok && t < g.n_tiles; t += gridDim.x) {
            int mt, nt;
            tile_coords(g, t, mt, nt);
            const int64_t row = (int64_t)mt * BM + r;
            const bool dump = g.dump_q != nullptr && nt == 0 && row < g.m;
            for (int kb = 0; kb < nkb; ++kb) {
                const int sa = ia % SA;
                if (!(ok = bar_wait(bar(B_FULL_A + sa), (uint32_t)(ia / SA) & 1u, abort_flag))) break;
                const uint32_t a16 = base + OFF_A16 + (uint32_t)sa * A16_BYTES + (uint32_t)r * 128u;
                // Range of the row's 128 values (NaN propagated to detect one).
                uint32_t ph = 0u, pl = 0u;
                float hi = 0.0f, nlo = 0.0f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    U4 v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] = ld_shared16(a16 + h * A16_BOX + (((uint32_t)j ^ swz) << 4));
                    range_tree<T, true, true, 8>(v, ph, pl, hi, nlo);
                }
                const bool nan = range_finish_nan<T, true>(ph, pl, hi, nlo);
                if (nan) {
                    ph = pl = 0u;
                    hi = nlo = 0.0f;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        U4 v[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) v[j] = ld_shared16(a16 + h * A16_BOX + (((uint32_t)j ^ swz) << 4));
                        range_tree<T, true, false, 8>(v, ph, pl, hi, nlo);
                    }
                    range_finish<T, true>(ph, pl, hi, nlo);
                }
                float s = (hi >= 0x1p-100f && hi <= 0x1p100f) ? div_chain(hi, Rq) : div_slow(hi, 448.0f);
                if (s == 0.0f) s = 1.0f;
                const Recip R = make_recip(s);
                const int sq = iq % SQ;
                if (!(ok = bar_wait(bar(B_EMPTY_Q + sq), ((uint32_t)(iq / SQ) & 1u) ^ 1u, abort_flag))) break;
                const uint32_t aq = base + OFF_AQ + (uint32_t)sq * AQ_BYTES + (uint32_t)r * 128u;
                const bool fast = R.fast && !nan;
                const Recip2 R2 = make_recip2(R);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // Codes 16j .. 16j+15 from 16-bit chunks 2j and 2j+1.
                    const int c0 = 2 * j, c1 = 2 * j + 1;
                    const U4 x0 = ld_shared16(a16 + (c0 >> 3) * A16_BOX + ((((uint32_t)c0 & 7u) ^ swz) << 4));
                    const U4 x1 = ld_shared16(a16 + (c1 >> 3) * A16_BOX + ((((uint32_t)c1 & 7u) ^ swz) << 4));
                    uint2 w0, w1;
                    if (fast) {
                        w0 = fp8_words_fast<T>(x0, R2);
                        w1 = fp8_words_fast<T>(x1, R2);
                    } else {
                        float v0[8], v1[8];
                        load_vec<T>(x0, v0);
                        load_vec<T>(x1, v1);
                        if (R.fast) {
                            w0 = fp8_words_general8<true>(v0, R);
                            w1 = fp8_words_general8<true>(v1, R);
                        } else {
                            w0 = fp8_words_general8<false>(v0, R);
                            w1 = fp8_words_general8<false>(v1, R);
                        }
                    }
                    st_shared16(aq + (((uint32_t)j ^ swz) << 4), w0.x, w0.y, w1.x, w1.y);
                }
                bar_arrive(bar(B_EMPTY_A + sa));       // done with the 16-bit tile
                ++ia;
                if (dump) {
                    // The operand bytes as the tensor core will read them.
                    uint8_t* dst = g.dump_q + row * g.k + (int64_t)kb * BK;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const U4 w = ld_shared16(aq + (((uint32_t)j ^ swz) << 4));
                        *reinterpret_cast<U4*>(dst + 16 * j) = w;
                    }
                    g.dump_s[row * nkb + kb] = s;
                }
                fence_async_shared();                  // codes visible to the tensor core
                bar_arrive(bar(B_FULL_Q + sq));
                ++iq;
                const int ss = is % SS;
                if (!(ok = bar_wait(bar(B_EMPTY_S + ss), ((uint32_t)(is / SS) & 1u) ^ 1u, abort_flag))) break;
                reinterpret_cast<volatile float*>(sb + OFF_SA)[ss * BM + r] = s;
                bar_arrive(bar(B_FULL_S + ss));
                ++is;
            }
        }
    } else if (warp < 12) {
        // ---------------------------------------------------- promotion
        set_max_regs_inc<REG_ACC>();
        const int q = warp & 3, h = (warp - 4) >> 2;
        const int rloc = 32 * q + lane;
        int is = 0, it = 0;
        bool ok = true;
        float acc[128];
        for (int64_t t = blockIdx.x; ok && t < g.n_tiles; t += gridDim.x) {
            int mt, nt;
            tile_coords(g, t, mt, nt);
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            const int64_t col0 = (int64_t)nt * BN + 128 * h;        // first column of this half
            const bool half_in = col0 < g.n;
            const float* swp = g.sw + (col0 / 128) * nkb;
            for (int kb = 0; kb < nkb; ++kb) {
                const int ss = is % SS;
                if (!(ok = bar_wait(bar(B_FULL_S + ss), (uint32_t)(is / SS) & 1u, abort_flag))) break;
                const float sa_v = sa_ring[ss * BM + rloc];
                bar_arrive(bar(B_EMPTY_S + ss));
                ++is;
                const float sw_v = half_in ? __ldg(swp + kb) : 0.0f;
                const float cf = __fmul_rn(sa_v, sw_v);
                const int buf = it & 1;
                if (!(ok = bar_wait(bar(B_TFULL + buf), (uint32_t)(it >> 1) & 1u, abort_flag))) break;
                tc_fence_after();
                const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 128 * h);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float p[16];
                    tmem_ld16(ta + 16 * ch, p);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[16 * ch + i] = __fmaf_rn(p[i], cf, acc[16 * ch + i]);
                }
                tc_fence_before();
                bar_arrive(bar(B_TEMPTY + buf));
                ++it;
            }
            if (!ok) break;
            const int64_t row = (int64_t)mt * BM + rloc;
            if (row < g.m && half_in) {
                const int64_t ncols = min((int64_t)128, g.n - col0);
                if (g.c_bf16) {
                    __nv_bfloat16* cr = reinterpret_cast<__nv_bfloat16*>(g.c) + row * g.n + col0;
                    if (ncols == 128 && (g.n & 7) == 0) {
#pragma unroll
                        for (int i = 0; i < 128; i += 8) {
                            U4 u;
                            u.x = pack_bf16x2(acc[i], acc[i + 1]); u.y = pack_bf16x2(acc[i + 2], acc[i + 3]);
                            u.z = pack_bf16x2(acc[i + 4], acc[i + 5]); u.w = pack_bf16x2(acc[i + 6], acc[i + 7]);
                            *reinterpret_cast<U4*>(cr + i) = u;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 128; ++i)
                            if (i < ncols) cr[i] = __float2bfloat16_rn(acc[i]);
                    }
                } else {
                    float* cr = reinterpret_cast<float*>(g.c) + row * g.n + col0;
                    if (ncols == 128 && (g.n & 3) == 0) {
#pragma unroll
                        for (int i = 0; i < 128; i += 4)
                            *reinterpret_cast<float4*>(cr + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 128; ++i)
                            if (i < ncols) cr[i] = acc[i];
                    }
                }
            }
        }
    } else {
        // ---------------------------------------------------- control warps
        set_max_regs_dec<REG_CTL>();
        if (warp == 12 && lane == 0) {
            // Activation tiles.
            int ia = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < g.n_tiles; t += gridDim.x) {
                int mt, nt;
                tile_coords(g, t, mt, nt);
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sa = ia % SA;
                    if (!(ok = bar_wait(bar(B_EMPTY_A + sa), ((uint32_t)(ia / SA) & 1u) ^ 1u, abort_flag))) break;
                    const uint32_t fb = bar(B_FULL_A + sa);
                    bar_expect_tx(fb, A16_BYTES);
                    const uint32_t dst = base + OFF_A16 + (uint32_t)sa * A16_BYTES;
                    tma_2d(dst, &tm_a, kb * BK, mt * BM, fb);
                    tma_2d(dst + A16_BOX, &tm_a, kb * BK + 64, mt * BM, fb);
                    ++ia;
                }
            }
            // Copies still in flight land before the CTA can exit.
            for (int i = max(0, ia - SA); i < ia; ++i) bar_drain(bar(B_FULL_A + i % SA), (uint32_t)(i / SA) & 1u);
        } else if (warp == 14 && lane == 0) {
            // Weight tiles.
            int iw = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < g.n_tiles; t += gridDim.x) {
                int mt, nt;
                tile_coords(g, t, mt, nt);
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sw = iw % SW;
                    if (!(ok = bar_wait(bar(B_EMPTY_W + sw), ((uint32_t)(iw / SW) & 1u) ^ 1u, abort_flag))) break;
                    const uint32_t fb = bar(B_FULL_W + sw);
                    bar_expect_tx(fb, W_BYTES);
                    tma_2d(base + OFF_W + (uint32_t)sw * W_BYTES, &tm_w, kb * BK, nt * BN, fb);
                    ++iw;
                }
            }
            for (int i = max(0, iw - SW); i < iw; ++i) bar_drain(bar(B_FULL_W + i % SW), (uint32_t)(i / SW) & 1u);
        } else if (warp == 13 && lane == 0) {
            // MMA issue.
            int iq = 0, iw = 0, it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < g.n_tiles; t += gridDim.x) {
                for (int kb = 0; kb < nkb; ++kb) {
                    const int buf = it & 1;
                    if (!(ok = bar_wait(bar(B_TEMPTY + buf), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag))) break;
                    const int sq = iq % SQ, sw = iw % SW;
                    if (!(ok = bar_wait(bar(B_FULL_Q + sq), (uint32_t)(iq / SQ) & 1u, abort_flag))) break;
                    if (!(ok = bar_wait(bar(B_FULL_W + sw), (uint32_t)(iw / SW) & 1u, abort_flag))) break;
                    tc_fence_after();
                    const uint64_t da = desc_k_sw128(base + OFF_AQ + (uint32_t)sq * AQ_BYTES);
                    const uint64_t dw = desc_k_sw128(base + OFF_W + (uint32_t)sw * W_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                    for (int k4 = 0; k4 < BK / 32; ++k4)      // K = 32 bytes per instruction
                        mma_f8(d, da + (uint64_t)(2 * k4), dw + (uint64_t)(2 * k4), kIdesc, k4 > 0 ? 1u : 0u);
                    mma_commit(bar(B_EMPTY_Q + sq));
                    mma_commit(bar(B_EMPTY_W + sw));
                    mma_commit(bar(B_TFULL + buf));
                    ++iq; ++iw; ++it;
                }
            }
            // Every MMA issued has completed before the TMEM is freed.
            mma_commit(bar(B_MMA_DONE));
            bar_drain(bar(B_MMA_DONE), 0u);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t encode_map(CUtensorMap* tm, CUtensorMapDataType dt, const void* p, uint64_t inner,
                       uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    static const PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            f = nullptr;
        }
        return (PFN_cuTensorMapEncodeTiled_v12000)f;
    }();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {inner, outer};
    const cuuint64_t gstride[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = encode(tm, dt, 2, const_cast<void*>(p), gdim, gstride, box, estride,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Per device: the kernel's shared-memory limit is raised once, and its
// launch register count is checked once (the setmaxnreg split above assumes
// REG_LAUNCH registers per thread at launch; any other count is refused).
template <class T>
cudaError_t prepare_kernel() {
    static int ready[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorUnknown;
    if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
    if (__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) return cudaSuccess;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, k_fp8_gemm<T>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != REG_LAUNCH) return cudaErrorNotSupported;
    e = cudaFuncSetAttribute(k_fp8_gemm<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    return cudaSuccess;
}

template <class T>
cudaError_t launch_gemm(const void* a, int64_t m, int64_t k, const uint8_t* w, const float* sw, int64_t n,
                        void* c, int c_bf16, uint8_t* dq, float* ds, cudaStream_t st) {
    cudaError_t e = prepare_kernel<T>();
    if (e != cudaSuccess) return e;
    CUtensorMap ta, tw;
    if ((e = encode_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT16, a, (uint64_t)k, (uint64_t)m, (uint64_t)k * 2, 64,
                        BM)) != cudaSuccess)
        return e;
    if ((e = encode_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)k, (uint64_t)n, (uint64_t)k, BK,
                        BN)) != cudaSuccess)
        return e;
    GemmArgs g;
    g.m = m; g.n = n; g.k = k;
    g.nkb = (int)(k / BK);
    g.mtiles = (int)((m + BM - 1) / BM);
    g.ntiles = (int)((n + BN - 1) / BN);
    g.band = min(16, g.mtiles);
    g.n_tiles = (int64_t)g.mtiles * g.ntiles;
    g.sw = sw; g.c = c; g.c_bf16 = c_bf16; g.dump_q = dq; g.dump_s = ds;
    int64_t grid = sm_count();
    if (grid > g.n_tiles) grid = g.n_tiles;
    k_fp8_gemm<T><<<(unsigned)grid, NT, SMEM_BYTES, st>>>(ta, tw, g);
    return cudaGetLastError();
}

}  // namespace

cudaError_t gemm_error_take(unsigned int* flag) {
    unsigned int v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v));
    if (e != cudaSuccess) return e;
    if (v) e = cudaMemcpyToSymbol(g_gemm_error, &z, sizeof(z));
    *flag = v;
    return e;
}

}  // namespace bq

extern "C" bq_status bq_fp8_block_gemm(const void* a, bq_dtype a_dtype, int64_t m, int64_t k,
                                       const uint8_t* w_e4m3, const float* w_scale, int64_t n, void* c,
                                       bq_dtype c_dtype, uint8_t* a_e4m3, float* a_scale, void* stream) {
    if (a_dtype != BQ_BF16 && a_dtype != BQ_F16) return BQ_ERR_UNSUPPORTED;
    if (c_dtype != BQ_F32 && c_dtype != BQ_BF16) return BQ_ERR_UNSUPPORTED;
    if (m < 0 || n < 0 || k <= 0 || k % 128 != 0) return BQ_ERR_INVALID_ARG;
    if (m >= (1ll << 31) || n >= (1ll << 31) || k >= (1ll << 31)) return BQ_ERR_INVALID_ARG;
    if ((a_e4m3 == nullptr) != (a_scale == nullptr)) return BQ_ERR_INVALID_ARG;
    if (m == 0 || n == 0) return BQ_OK;
    if (!a || !w_e4m3 || !w_scale || !c) return BQ_ERR_INVALID_ARG;
    const int64_t esz = c_dtype == BQ_F32 ? 4 : 2;
    if (((uintptr_t)a & 15u) || ((uintptr_t)w_e4m3 & 15u) || ((uintptr_t)w_scale & 3u) ||
        ((uintptr_t)c & 15u) || ((uintptr_t)a_e4m3 & 15u) || ((uintptr_t)a_scale & 3u))
        return BQ_ERR_MISALIGNED;
    (void)esz;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e = (a_dtype == BQ_BF16)
        ? bq::launch_gemm<__nv_bfloat16>(a, m, k, w_e4m3, w_scale, n, c, c_dtype == BQ_BF16, a_e4m3, a_scale, st)
        : bq::launch_gemm<__half>(a, m, k, w_e4m3, w_scale, n, c, c_dtype == BQ_BF16, a_e4m3, a_scale, st);
    if (e == cudaErrorNotSupported) return BQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
