// W8A8 block-FP8 matrix multiply with the activation quantization fused into
// its prologue ([smile.llm.quant] Fp8BlockGemm: activations quantized on the
// fly to E4M3 with one f32 scale per 1x128 group, weights E4M3 with one f32
// scale per 128x128 tile):
//   C[i, j] = sum over k-blocks b of sa[i, b] * sw[j / 128, b] * S(i, j, b),
//   S(i, j, b) = sum over the 128 k of block b of dec(ea[i, k]) * dec(ew[j, k]).
//
// A cluster of CL CTAs (one per SM, 512 threads each) works on CL adjacent
// 128 x 256 tiles of C that share their 128 activation rows. The activation
// tile of a k-block (128 rows x 128 k) is quantized once per cluster: each
// CTA loads RB = 128 / CL of its rows and writes their E4M3 codes and scales
// into the shared memory of every CTA of the cluster (distributed shared
// memory), so the per-SM prologue work and activation traffic drop by CL.
// Per CTA and k-block of 128:
//   warp 12      TMA: its RB activation rows (bf16 / f16, two 64-column boxes,
//                128-byte swizzle) into a ring;
//   warp 14      TMA: E4M3 weight tile [256 rows x 128 bytes] into a ring;
//   warps 0-3    prologue: CL threads per row quantize the RB rows exactly as
//                bq_fp8_block_quantize does for a 1 x 128 block (amax,
//                s = fl(amax / 448), E4M3(fl(x / s)), the same device
//                functions) and store the codes, in the K-major 128-byte
//                swizzled layout the tensor core reads, and the scales into
//                every CTA of the cluster;
//   warp 13      TMEM allocation (512 columns) and, from one thread, the
//                tcgen05.mma.kind::f8f6f4 instructions (M 128, N 256, K 32;
//                four per k-block) into one of two TMEM partial buffers;
//   warps 4-11   promotion: each thread owns one row and 128 columns of the
//                tile; per k-block it reads the block's partial sums from
//                TMEM (tcgen05.ld) and adds partial * fl(sa * sw) into f32
//                registers, then frees the buffer; at the end of the tile it
//                writes its row of C.
// A code stage is free again when the MMAs of every CTA of the cluster have
// read it (tcgen05.commit multicast to the cluster's barriers); a scale slot
// when every CTA's promotion warps have read it (remote mbarrier arrivals).
// No TMA multicast of any kind.
//
// Every mbarrier wait is bounded (about two seconds); a role that gives up
// sets the abort flag of every CTA of its cluster (the other roles see it
// within microseconds), records the error in g_gemm_error, waits (bounded)
// for the copies and MMAs it has in flight, and the CTAs free their TMEM and
// return after one cluster-wide barrier.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>

#include "bq.h"
#include "bq_device.cuh"
#include "bq_internal.h"
#include "bq_quant_ops.cuh"
#include "bq_range.cuh"

namespace bq {
namespace {

__device__ unsigned int g_gemm_error;

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int NT = 512;
constexpr uint32_t AQ_BYTES = BM * BK;
constexpr uint32_t W_BYTES = BN * BK;
constexpr uint32_t TMEM_COLS = 512;                   // two partial buffers of BN columns
static_assert(2 * BN <= (int)TMEM_COLS, "TMEM");

// Shared-memory plan for a cluster of CL CTAs.
template <int CL>
struct Plan {
    static constexpr int RB = BM / CL;                 // activation rows this CTA quantizes
    static constexpr int SA = CL == 1 ? 2 : (CL == 2 ? 3 : 4);   // activation (16-bit) slots
    static constexpr int SQ = CL == 1 ? 3 : (CL == 2 ? 4 : 5);   // operand (E4M3) slots
    static constexpr int SW = 3;                                 // weight slots
    static constexpr int SS = 4;                       // scale slots
    static constexpr uint32_t A16_BOX = RB * 128;      // RB rows x 64 columns x 2 bytes
    static constexpr uint32_t A16_BYTES = 2 * A16_BOX;
    static constexpr uint32_t OFF_A16 = 0;
    static constexpr uint32_t OFF_AQ = OFF_A16 + SA * A16_BYTES;
    static constexpr uint32_t OFF_W = OFF_AQ + SQ * AQ_BYTES;
    static constexpr uint32_t OFF_SA = OFF_W + SW * W_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_SA + SS * BM * 4;
    static constexpr int B_FULL_A = 0, B_EMPTY_A = B_FULL_A + SA, B_FULL_Q = B_EMPTY_A + SA,
                         B_EMPTY_Q = B_FULL_Q + SQ, B_FULL_W = B_EMPTY_Q + SQ, B_EMPTY_W = B_FULL_W + SW,
                         B_FULL_S = B_EMPTY_W + SW, B_EMPTY_S = B_FULL_S + SS, B_TFULL = B_EMPTY_S + SS,
                         B_TEMPTY = B_TFULL + 2, B_MMA_DONE = B_TEMPTY + 2, B_PDONE = B_MMA_DONE + 1,
                         B_QREAD = B_PDONE + SQ, N_BAR = B_QREAD + SQ;
    static constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;   // [0] TMEM base, [1] abort flag
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024; // room to align the base to 1024
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(A16_BOX % 1024 == 0 && A16_BYTES % 1024 == 0 && OFF_AQ % 1024 == 0 && OFF_W % 1024 == 0,
                  "swizzled tiles start on 1024-byte boundaries");
};

// Register split (setmaxnreg): the block launches with NT x 128 registers.
// Prologue warps 0-3 keep 120, promotion warps 4-11 take 176, warps 12-15
// keep 40: 128*120 + 256*176 + 128*40 = 65536 = 512 * 128.
constexpr int REG_LAUNCH = 128, REG_PRO = 120, REG_ACC = 176, REG_CTL = 40;
static_assert(128 * REG_PRO + 256 * REG_ACC + 128 * REG_CTL == NT * REG_LAUNCH, "register split");

struct GemmArgs {
    int64_t m, n, k;
    int nkb;            // k / 128
    int mtiles, ntiles;
    int nct;            // cluster tiles along N: ceil(ntiles / CL)
    int band;           // raster band height in M tiles
    int64_t n_ctiles;   // mtiles * nct
    const float* sw;    // [ceil(n / 128), nkb]
    void* c;
    int c_bf16;
    uint8_t* dump_q;    // optional [m, k]: operand bytes read back from shared memory
    float* dump_s;      // optional [m, nkb]
    const float* sa;    // activation scales [m, nkb] (pre-quantized activations only)
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
// The same wait with cluster-scope acquire, for barriers other CTAs of the
// cluster arrive on (their stores to this CTA become visible).
__device__ __forceinline__ bool bar_try_wait_cl(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(1000u) : "memory");
    return ok != 0;
}
// Shared-memory address of the same location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void bar_arrive_remote(uint32_t cl_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(cl_addr) : "memory");
}
__device__ __forceinline__ void bar_arrive_remote_relaxed(uint32_t cl_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" :: "r"(cl_addr) : "memory");
}
// One arrival on the barrier at `bar` in every CTA of the cluster, lane d of
// the (converged) warp arriving on CTA d, so the arrivals travel in
// parallel. RELEASE: the warp's earlier stores (ordered before by the
// __syncwarp the caller ran) are visible in the cluster before the arrival
// counts; otherwise the arrival only orders what the barrier guards against
// overwriting (reads that have completed).
template <int CL, bool RELEASE>
__device__ __forceinline__ void arrive_all_ranks(uint32_t bar, int lane) {
    if (lane < CL) {
        const uint32_t a = map_rank(bar, (uint32_t)lane);
        if (RELEASE) bar_arrive_remote(a);
        else bar_arrive_remote_relaxed(a);
    }
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cl_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(cl_addr), "r"(v) : "memory");
}
// Bulk copy of `bytes` from this CTA's shared memory to a cluster address
// (another CTA's shared memory); completes transaction bytes on the mbarrier
// at the cluster address `cl_bar` (in the destination CTA).
__device__ __forceinline__ void bulk_to_rank(uint32_t cl_dst, uint32_t src, uint32_t bytes, uint32_t cl_bar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(cl_dst), "r"(src), "r"(bytes), "r"(cl_bar) : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Bounded wait (each try suspends for at most about a microsecond); gives up
// early once another role (of any CTA of the cluster) has set the abort
// flag. On giving up by itself it sets the flag in every CTA of the cluster
// and the device error.
// Non-blocking probe of a phase (no suspension): the common case of a
// barrier that has already completed costs one instruction.
template <bool CLUSTER_SCOPE>
__device__ __forceinline__ bool bar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    if (CLUSTER_SCOPE)
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    else
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
template <int CL, bool CLUSTER_SCOPE>
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                         uint32_t abort_addr) {
    if (bar_test<CLUSTER_SCOPE>(bar, parity)) return true;
    for (uint32_t i = 0; i < (1u << 21); ++i) {
        if (CLUSTER_SCOPE ? bar_try_wait_cl(bar, parity) : bar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 15u && *abort_flag) return false;
    }
    if (CL == 1) *abort_flag = 1u;
    else
        for (uint32_t d = 0; d < (uint32_t)CL; ++d) st_cluster_u32(map_rank(abort_addr, d), 1u);
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
// 32 consecutive f32 columns of this thread's TMEM lane (raw bits). The
// registers hold the values only after tmem_ld_wait and tmem_regs_ready.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}
// Placed after tcgen05.wait::ld: no use of the loaded registers is moved
// above it (the compiler sees them written here).
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
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

// One k-block of promotion for one thread (a TMEM lane = a row of the tile,
// 128 columns from `ta`): acc[i] += partial[i] * cf, one fused multiply-add
// per column, on column pairs. Four loads of 32 columns, each waited for.
__device__ __forceinline__ void promote_block(F2 (&acc)[64], uint32_t ta, F2 cf) {
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld32(ta + 32 * ch, r);
        tmem_ld_wait();
        tmem_regs_ready(r);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            acc[16 * ch + i] = f2_fma(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), cf,
                                      acc[16 * ch + i]);
    }
}
// The same with two loads in flight per wait (64 more registers): half the
// TMEM round trips per k-block.
__device__ __forceinline__ void promote_block_2x(F2 (&acc)[64], uint32_t ta, F2 cf) {
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
        uint32_t r0[32], r1[32];
        tmem_ld32(ta + 64 * hb, r0);
        tmem_ld32(ta + 64 * hb + 32, r1);
        tmem_ld_wait();
        tmem_regs_ready(r0);
        tmem_regs_ready(r1);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            acc[32 * hb + i] = f2_fma(f2_pack(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1])), cf,
                                      acc[32 * hb + i]);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            acc[32 * hb + 16 + i] = f2_fma(f2_pack(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1])),
                                           cf, acc[32 * hb + 16 + i]);
    }
}
// The thread's 128 columns of C (row `row`, from column col0), in C's dtype;
// columns past n are skipped.
__device__ __forceinline__ void store_c_half(const GemmArgs& g, int64_t row, int64_t col0, const F2 (&acc)[64]) {
    const int64_t ncols = min((int64_t)128, g.n - col0);
    float v[128];
#pragma unroll
    for (int i = 0; i < 64; ++i) f2_split(acc[i], v[2 * i], v[2 * i + 1]);
    if (g.c_bf16) {
        __nv_bfloat16* cr = reinterpret_cast<__nv_bfloat16*>(g.c) + row * g.n + col0;
        if (ncols == 128 && (g.n & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 128; i += 8) {
                U4 o;
                o.x = pack_bf16x2(v[i], v[i + 1]); o.y = pack_bf16x2(v[i + 2], v[i + 3]);
                o.z = pack_bf16x2(v[i + 4], v[i + 5]); o.w = pack_bf16x2(v[i + 6], v[i + 7]);
                *reinterpret_cast<U4*>(cr + i) = o;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 128; ++i)
                if (i < ncols) cr[i] = __float2bfloat16_rn(v[i]);
        }
    } else {
        float* cr = reinterpret_cast<float*>(g.c) + row * g.n + col0;
        if (ncols == 128 && (g.n & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 128; i += 4)
                *reinterpret_cast<float4*>(cr + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 128; ++i)
                if (i < ncols) cr[i] = v[i];
        }
    }
}

// Cluster tile u -> (M tile, cluster tile along N): bands of `band` M tiles,
// walked down M first, so the clusters working at one time share a few
// weight panels and a band of activation rows in L2.
__device__ __forceinline__ void ctile_coords(const GemmArgs& g, int64_t u, int& mt, int& ntc) {
    const int64_t per_band = (int64_t)g.band * g.nct;
    const int b = (int)(u / per_band);
    const int r = (int)(u - (int64_t)b * per_band);
    const int rows = min(g.band, g.mtiles - b * g.band);
    mt = b * g.band + r % rows;
    ntc = r / rows;
}

template <class T, int CL>
__global__ void __launch_bounds__(NT, 1) k_fp8_gemm(const __grid_constant__ CUtensorMap tm_a,
                                                     const __grid_constant__ CUtensorMap tm_w,
                                                     const GemmArgs g) {
    using P = Plan<CL>;
    constexpr int RB = P::RB, SA = P::SA, SQ = P::SQ, SW = P::SW, SS = P::SS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = sm_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw_base);
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(sb + P::OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;
    const uint32_t abort_addr = base + P::OFF_MISC + 4;
    const float* sa_ring = reinterpret_cast<const float*>(sb + P::OFF_SA);
    auto bar = [&](int i) -> uint32_t { return base + P::OFF_BAR + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CL == 1 ? 0u : cluster_rank();
    const int64_t cid = blockIdx.x / CL, ncl = gridDim.x / CL;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SA; ++i) { bar_init(bar(P::B_FULL_A + i), 1); bar_init(bar(P::B_EMPTY_A + i), 128); }
        for (int i = 0; i < SQ; ++i) { bar_init(bar(P::B_FULL_Q + i), 1); bar_init(bar(P::B_EMPTY_Q + i), CL); }
        for (int i = 0; i < SW; ++i) { bar_init(bar(P::B_FULL_W + i), 1); bar_init(bar(P::B_EMPTY_W + i), 1); }
        for (int i = 0; i < SS; ++i) { bar_init(bar(P::B_FULL_S + i), 1); bar_init(bar(P::B_EMPTY_S + i), 8 * CL); }
        for (int i = 0; i < 2; ++i) { bar_init(bar(P::B_TFULL + i), 1); bar_init(bar(P::B_TEMPTY + i), 256); }
        bar_init(bar(P::B_MMA_DONE), 1);
        for (int i = 0; i < SQ; ++i) bar_init(bar(P::B_PDONE + i), 128);
        for (int i = 0; i < SQ; ++i) bar_init(bar(P::B_QREAD + i), 1);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 12 && lane == 0) prefetch_map(&tm_a);
    if (warp == 14 && lane == 0) prefetch_map(&tm_w);
    if (warp == 13) tmem_alloc(base + P::OFF_MISC, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    if (CL > 1) cluster_sync();                       // every barrier of the cluster initialised
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int nkb = g.nkb;

    if (warp < 4) {
        // ---------------------------------------------------- prologue
        set_max_regs_dec<REG_PRO>();
        const int t = threadIdx.x;
        const int rl = t / CL;                         // row among this CTA's RB rows
        const int part = t % CL;                       // which 128/CL columns of the row
        const int R = (int)rank * RB + rl;             // row of the 128-row tile
        const int swz = rl & 7;                        // == R & 7 (RB is a multiple of 8)
        constexpr int CPT = 16 / CL;                   // 16-byte input chunks per thread
        // Chunk order rotated per part, so that the lanes of one shared-memory
        // phase read distinct bank groups.
        const int rot = CL == 2 ? 4 * part : (CL == 4 ? 2 * (part >> 1) : 0);
        const Recip Rq = make_recip(448.0f);
        int ia = 0, iq = 0, is = 0;
        bool ok = true;
        for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
            int mt, ntc;
            ctile_coords(g, u, mt, ntc);
            const int64_t row = (int64_t)mt * BM + R;
            const bool dump = g.dump_q != nullptr && ntc == 0 && row < g.m;
            for (int kb = 0; kb < nkb; ++kb) {
                const int sa = ia % SA;
                if (!(ok = bar_wait<CL, false>(bar(P::B_FULL_A + sa), (uint32_t)(ia / SA) & 1u, abort_flag, abort_addr))) break;
                // Row rl of the two 64-column boxes (128-byte swizzle: 16-byte
                // chunk j of the row sits at chunk j ^ (rl & 7)).
                const U4* a16 = reinterpret_cast<const U4*>(sb + P::OFF_A16 + (uint32_t)sa * P::A16_BYTES +
                                                            (uint32_t)rl * 128u);
                constexpr int BOX = P::A16_BOX / 16;
                auto chunk = [&](int j) -> U4 {            // the thread's j-th chunk (rotated order)
                    const int c = part * CPT + ((j + rot) & (CPT - 1));
                    return a16[(c >> 3) * BOX + ((c & 7) ^ swz)];
                };
                // Range of the row's 128 values (NaN propagated to detect one),
                // CL threads per row combined by shuffles.
                uint32_t ph = 0u, pl = 0u;
                float hi = 0.0f, nlo = 0.0f;
                {
                    U4 v[CPT];
#pragma unroll
                    for (int j = 0; j < CPT; ++j) v[j] = chunk(j);
                    range_tree<T, true, true, CPT>(v, ph, pl, hi, nlo);
                }
#pragma unroll
                for (int o = 1; o < CL; o <<= 1)
                    ph = pk_hi<T, true, true>(ph, __shfl_xor_sync(0xffffffffu, ph, o));
                bool nan = range_finish_nan<T, true>(ph, pl, hi, nlo);
                if (__any_sync(0xffffffffu, nan)) {
                    uint32_t qh = 0u, ql = 0u;
                    float h2 = 0.0f, n2 = 0.0f;
                    U4 v[CPT];
#pragma unroll
                    for (int j = 0; j < CPT; ++j) v[j] = chunk(j);
                    range_tree<T, true, false, CPT>(v, qh, ql, h2, n2);
#pragma unroll
                    for (int o = 1; o < CL; o <<= 1)
                        qh = pk_hi<T, true, false>(qh, __shfl_xor_sync(0xffffffffu, qh, o));
                    range_finish<T, true>(qh, ql, h2, n2);
                    if (nan) hi = h2;
                }
                float s = (hi >= 0x1p-100f && hi <= 0x1p100f) ? div_chain(hi, Rq) : div_slow(hi, 448.0f);
                if (s == 0.0f) s = 1.0f;
                const Recip R1 = make_recip(s);
                const int sq = iq % SQ;
                if (!(ok = bar_wait<CL, true>(bar(P::B_EMPTY_Q + sq), ((uint32_t)(iq / SQ) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                const uint32_t aq_row = base + P::OFF_AQ + (uint32_t)sq * AQ_BYTES + (uint32_t)R * 128u;
                const bool fast = R1.fast && !nan;
                const Recip2T R2 = make_recip2(R1);
#pragma unroll
                for (int jj = 0; jj < CPT / 2; ++jj) {
                    // Codes of input chunks c0, c0 + 1 (16 values) -> code chunk c0 / 2.
                    const int c0 = part * CPT + ((2 * jj + rot) & (CPT - 1));
                    const U4 x0 = a16[(c0 >> 3) * BOX + ((c0 & 7) ^ swz)];
                    const U4 x1 = a16[((c0 + 1) >> 3) * BOX + (((c0 + 1) & 7) ^ swz)];
                    uint2 w0, w1;
                    if (fast) {
                        w0 = fp8_words_fast<T>(x0, R2);
                        w1 = fp8_words_fast<T>(x1, R2);
                    } else {
                        float v0[8], v1[8];
                        load_vec<T>(x0, v0);
                        load_vec<T>(x1, v1);
                        if (R1.fast) {
                            w0 = fp8_words_general8<true>(v0, R1);
                            w1 = fp8_words_general8<true>(v1, R1);
                        } else {
                            w0 = fp8_words_general8<false>(v0, R1);
                            w1 = fp8_words_general8<false>(v1, R1);
                        }
                    }
                    U4 o;
                    o.x = w0.x; o.y = w0.y; o.z = w1.x; o.w = w1.y;
                    reinterpret_cast<U4*>(sb + (aq_row - base))[(c0 >> 1) ^ swz] = o;
                }
                bar_arrive(bar(P::B_EMPTY_A + sa));    // done with the 16-bit tile
                ++ia;
                if (dump) {
                    // The operand bytes as the tensor core will read them.
                    const U4* aq = reinterpret_cast<const U4*>(sb + (aq_row - base));
                    U4* dst = reinterpret_cast<U4*>(g.dump_q + row * g.k + (int64_t)kb * BK);
#pragma unroll
                    for (int jj = 0; jj < CPT / 2; ++jj) {
                        const int cc = (part * CPT) / 2 + jj;
                        dst[cc] = aq[cc ^ swz];
                    }
                    if (part == 0) g.dump_s[row * nkb + kb] = s;
                }
                // The scale of each row, in this CTA's slot.
                const int ss = is % SS;
                if (!(ok = bar_wait<CL, true>(bar(P::B_EMPTY_S + ss), ((uint32_t)(is / SS) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                if (part == 0) reinterpret_cast<volatile float*>(sb + P::OFF_SA)[ss * BM + R] = s;
                // Codes and scales visible to the async proxy (tensor core,
                // bulk copies), then one thread publishes them: its own
                // barriers get one arrival plus the bytes the other CTAs'
                // copies will bring; the other CTAs get this CTA's rows by
                // bulk copy, completing on their barriers.
                fence_async_shared();
                bar_arrive(bar(P::B_PDONE + sq));
                ++iq;
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
        F2 acc[64];                                      // columns 2i, 2i+1 of this half
        for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
            int mt, ntc;
            ctile_coords(g, u, mt, ntc);
            const int nt = ntc * CL + (int)rank;
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0ull;
            const int64_t col0 = (int64_t)nt * BN + 128 * h;        // first column of this half
            const bool half_in = col0 < g.n;
            const float* swp = g.sw + (half_in ? (col0 / 128) * nkb : 0);
            // Weight-tile scales two blocks ahead (their loads overlap the
            // TMEM work of the blocks before).
            float sw0 = half_in ? __ldg(swp) : 0.0f;
            float sw1 = (half_in && nkb > 1) ? __ldg(swp + 1) : 0.0f;
            for (int kb = 0; kb < nkb; ++kb) {
                const float sw2 = (half_in && kb + 2 < nkb) ? __ldg(swp + kb + 2) : 0.0f;
                const int ss = is % SS;
                if (!(ok = bar_wait<CL, true>(bar(P::B_FULL_S + ss), (uint32_t)(is / SS) & 1u, abort_flag, abort_addr))) break;
                const float sa_v = sa_ring[ss * BM + rloc];
                const F2 cf = f2_bcast(__fmul_rn(sa_v, sw0));
                __syncwarp();
                if (CL == 1) {
                    if (lane == 0) bar_arrive(bar(P::B_EMPTY_S + ss));
                } else {
                    arrive_all_ranks<CL, false>(bar(P::B_EMPTY_S + ss), lane);
                }
                ++is;
                const int buf = it & 1;
                if (!(ok = bar_wait<CL, false>(bar(P::B_TFULL + buf), (uint32_t)(it >> 1) & 1u, abort_flag, abort_addr))) break;
                tc_fence_after();
                const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 128 * h);
                promote_block(acc, ta, cf);
                tc_fence_before();
                bar_arrive(bar(P::B_TEMPTY + buf));
                ++it;
                sw0 = sw1;
                sw1 = sw2;
            }
            if (!ok) break;
            const int64_t row = (int64_t)mt * BM + rloc;
            if (row < g.m && half_in) store_c_half(g, row, col0, acc);
        }
    } else {
        // ---------------------------------------------------- control warps
        set_max_regs_dec<REG_CTL>();
        if (warp == 12 && lane == 0) {
            // This CTA's activation rows.
            int ia = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                int mt, ntc;
                ctile_coords(g, u, mt, ntc);
                const int y = mt * BM + (int)rank * RB;
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sa = ia % SA;
                    if (!(ok = bar_wait<CL, false>(bar(P::B_EMPTY_A + sa), ((uint32_t)(ia / SA) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const uint32_t fb = bar(P::B_FULL_A + sa);
                    bar_expect_tx(fb, P::A16_BYTES);
                    const uint32_t dst = base + P::OFF_A16 + (uint32_t)sa * P::A16_BYTES;
                    tma_2d(dst, &tm_a, kb * BK, y, fb);
                    tma_2d(dst + P::A16_BOX, &tm_a, kb * BK + 64, y, fb);
                    ++ia;
                }
            }
            // Copies still in flight land before the CTA can exit.
            for (int i = max(0, ia - SA); i < ia; ++i) bar_drain(bar(P::B_FULL_A + i % SA), (uint32_t)(i / SA) & 1u);
        } else if (warp == 14 && lane == 0) {
            // Weight tiles.
            int iw = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                int mt, ntc;
                ctile_coords(g, u, mt, ntc);
                const int nt = ntc * CL + (int)rank;
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sw = iw % SW;
                    if (!(ok = bar_wait<CL, false>(bar(P::B_EMPTY_W + sw), ((uint32_t)(iw / SW) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const uint32_t fb = bar(P::B_FULL_W + sw);
                    bar_expect_tx(fb, W_BYTES);
                    tma_2d(base + P::OFF_W + (uint32_t)sw * W_BYTES, &tm_w, kb * BK, nt * BN, fb);
                    ++iw;
                }
            }
            for (int i = max(0, iw - SW); i < iw; ++i) bar_drain(bar(P::B_FULL_W + i % SW), (uint32_t)(i / SW) & 1u);
        } else if (warp == 15 && lane == 0) {
            // Publisher: once the 128 prologue threads have written a k-block's
            // codes and scales (PDONE), this CTA's barriers get one arrival plus
            // the bytes the other CTAs' copies will bring, and the other CTAs
            // get this CTA's rows by bulk copy, completing on their barriers.
            constexpr uint32_t QB = RB * 128u, SB4 = RB * 4u;
            int iq = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sq = iq % SQ, ss = iq % SS;
                    if (!(ok = bar_wait<CL, false>(bar(P::B_PDONE + sq), (uint32_t)(iq / SQ) & 1u, abort_flag, abort_addr))) break;
                    bar_expect_tx(bar(P::B_FULL_Q + sq), (CL - 1) * QB);
                    bar_expect_tx(bar(P::B_FULL_S + ss), (CL - 1) * SB4);
                    if (CL > 1) {
                        const uint32_t qsrc = base + P::OFF_AQ + (uint32_t)sq * AQ_BYTES + rank * QB;
                        const uint32_t ssrc = base + P::OFF_SA + (uint32_t)(ss * BM) * 4u + rank * SB4;
                        for (uint32_t d = 1; d < (uint32_t)CL; ++d) {
                            const uint32_t dr = (rank + d) % (uint32_t)CL;
                            bulk_to_rank(map_rank(qsrc, dr), qsrc, QB, map_rank(bar(P::B_FULL_Q + sq), dr));
                            bulk_to_rank(map_rank(ssrc, dr), ssrc, SB4, map_rank(bar(P::B_FULL_S + ss), dr));
                        }
                    }
                    ++iq;
                }
            }
        } else if (CL > 1 && warp == 13 && lane >= 1 && lane <= CL) {
            // Relay (lane l for CTA l - 1): when this CTA's MMAs have read a
            // code stage (QREAD), release it in every CTA of the cluster: its
            // rows there came from this CTA and will be overwritten next.
            int iq = 0;
            bool ok = true;
            const uint32_t dr = (uint32_t)(lane - 1);
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sq = iq % SQ;
                    if (!(ok = bar_wait<CL, false>(bar(P::B_QREAD + sq), (uint32_t)(iq / SQ) & 1u, abort_flag, abort_addr))) break;
                    bar_arrive_remote_relaxed(map_rank(bar(P::B_EMPTY_Q + sq), dr));
                    ++iq;
                }
            }
        } else if (warp == 13 && lane == 0) {
            // MMA issue.
            int iq = 0, iw = 0, it = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                for (int kb = 0; kb < nkb; ++kb) {
                    const int buf = it & 1;
                    if (!(ok = bar_wait<CL, false>(bar(P::B_TEMPTY + buf), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const int sq = iq % SQ, sw = iw % SW;
                    if (!(ok = bar_wait<CL, true>(bar(P::B_FULL_Q + sq), (uint32_t)(iq / SQ) & 1u, abort_flag, abort_addr))) break;
                    if (!(ok = bar_wait<CL, false>(bar(P::B_FULL_W + sw), (uint32_t)(iw / SW) & 1u, abort_flag, abort_addr))) break;
                    tc_fence_after();
                    const uint64_t da = desc_k_sw128(base + P::OFF_AQ + (uint32_t)sq * AQ_BYTES);
                    const uint64_t dw = desc_k_sw128(base + P::OFF_W + (uint32_t)sw * W_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                    for (int k4 = 0; k4 < BK / 32; ++k4)      // K = 32 bytes per instruction
                        mma_f8(d, da + (uint64_t)(2 * k4), dw + (uint64_t)(2 * k4), kIdesc, k4 > 0 ? 1u : 0u);
                    mma_commit(bar(P::B_TFULL + buf));
                    mma_commit(bar(P::B_EMPTY_W + sw));
                    // In a cluster the code stage is released in every CTA by
                    // warp 15 once these MMAs have read it (QREAD).
                    mma_commit(bar(CL == 1 ? P::B_EMPTY_Q + sq : P::B_QREAD + sq));
                    ++iq; ++iw; ++it;
                }
            }
            // Every MMA issued has completed before the TMEM is freed.
            mma_commit(bar(P::B_MMA_DONE));
            bar_drain(bar(P::B_MMA_DONE), 0u);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    // No CTA leaves while another of its cluster may still write into it.
    if (CL > 1) cluster_sync();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------ activations
// already quantized
// The same matrix multiply for activations given as 1x128 E4M3 codes and
// scales (as bq_fp8_block_quantize writes them): no prologue, so every CTA
// works alone. 384 threads: warp 0 loads activation code tiles
// [128 rows x 128 bytes] and warp 1 weight tiles [256 rows x 128 bytes] by TMA
// (128-byte swizzle: the operand layout the MMA reads), warp 2 allocates TMEM
// and issues the MMAs, warps 4-11 promote as in k_fp8_gemm with the
// activation scales read from global memory two blocks ahead. Register
// split: warps 0-3 keep 56, warps 4-11 take 224 (128*56 + 256*224 =
// 384 * 168, the launch count).
struct PlanQ {
    static constexpr int SQ = 4, SW = 4;
    static constexpr uint32_t OFF_AQ = 0;
    static constexpr uint32_t OFF_W = OFF_AQ + SQ * AQ_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_W + SW * W_BYTES;
    static constexpr int B_FULL_Q = 0, B_EMPTY_Q = B_FULL_Q + SQ, B_FULL_W = B_EMPTY_Q + SQ,
                         B_EMPTY_W = B_FULL_W + SW, B_TFULL = B_EMPTY_W + SW, B_TEMPTY = B_TFULL + 2,
                         B_MMA_DONE = B_TEMPTY + 2, N_BAR = B_MMA_DONE + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};
constexpr int NT_Q = 384;
constexpr int REGQ_LAUNCH = 168, REGQ_CTL = 56, REGQ_ACC = 224;
static_assert(128 * REGQ_CTL + 256 * REGQ_ACC <= NT_Q * REGQ_LAUNCH, "register split");

__global__ void __launch_bounds__(NT_Q, 1) k_fp8_gemm_q(const __grid_constant__ CUtensorMap tm_a,
                                                         const __grid_constant__ CUtensorMap tm_w,
                                                         const GemmArgs g) {
    using P = PlanQ;
    constexpr int SQ = P::SQ, SW = P::SW;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = sm_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw_base);
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(sb + P::OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;
    const uint32_t abort_addr = base + P::OFF_MISC + 4;
    auto bar = [&](int i) -> uint32_t { return base + P::OFF_BAR + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SQ; ++i) { bar_init(bar(P::B_FULL_Q + i), 1); bar_init(bar(P::B_EMPTY_Q + i), 1); }
        for (int i = 0; i < SW; ++i) { bar_init(bar(P::B_FULL_W + i), 1); bar_init(bar(P::B_EMPTY_W + i), 1); }
        for (int i = 0; i < 2; ++i) { bar_init(bar(P::B_TFULL + i), 1); bar_init(bar(P::B_TEMPTY + i), 256); }
        bar_init(bar(P::B_MMA_DONE), 1);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) prefetch_map(&tm_a);
    if (warp == 1 && lane == 0) prefetch_map(&tm_w);
    if (warp == 2) tmem_alloc(base + P::OFF_MISC, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int nkb = g.nkb;
    const int64_t cid = blockIdx.x, ncl = gridDim.x;

    if (warp < 4) {
        set_max_regs_dec<REGQ_CTL>();
        if (warp == 0 && lane == 0) {
            // Activation code tiles.
            int iq = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                int mt, nt;
                ctile_coords(g, u, mt, nt);
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sq = iq % SQ;
                    if (!(ok = bar_wait<1, false>(bar(P::B_EMPTY_Q + sq), ((uint32_t)(iq / SQ) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const uint32_t fb = bar(P::B_FULL_Q + sq);
                    bar_expect_tx(fb, AQ_BYTES);
                    tma_2d(base + P::OFF_AQ + (uint32_t)sq * AQ_BYTES, &tm_a, kb * BK, mt * BM, fb);
                    ++iq;
                }
            }
            for (int i = max(0, iq - SQ); i < iq; ++i) bar_drain(bar(P::B_FULL_Q + i % SQ), (uint32_t)(i / SQ) & 1u);
        } else if (warp == 1 && lane == 0) {
            // Weight tiles.
            int iw = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                int mt, nt;
                ctile_coords(g, u, mt, nt);
                for (int kb = 0; kb < nkb; ++kb) {
                    const int sw = iw % SW;
                    if (!(ok = bar_wait<1, false>(bar(P::B_EMPTY_W + sw), ((uint32_t)(iw / SW) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const uint32_t fb = bar(P::B_FULL_W + sw);
                    bar_expect_tx(fb, W_BYTES);
                    tma_2d(base + P::OFF_W + (uint32_t)sw * W_BYTES, &tm_w, kb * BK, nt * BN, fb);
                    ++iw;
                }
            }
            for (int i = max(0, iw - SW); i < iw; ++i) bar_drain(bar(P::B_FULL_W + i % SW), (uint32_t)(i / SW) & 1u);
        } else if (warp == 2 && lane == 0) {
            // MMA issue.
            int iq = 0, iw = 0, it = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                for (int kb = 0; kb < nkb; ++kb) {
                    const int buf = it & 1;
                    if (!(ok = bar_wait<1, false>(bar(P::B_TEMPTY + buf), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const int sq = iq % SQ, sw = iw % SW;
                    if (!(ok = bar_wait<1, false>(bar(P::B_FULL_Q + sq), (uint32_t)(iq / SQ) & 1u, abort_flag, abort_addr))) break;
                    if (!(ok = bar_wait<1, false>(bar(P::B_FULL_W + sw), (uint32_t)(iw / SW) & 1u, abort_flag, abort_addr))) break;
                    tc_fence_after();
                    const uint64_t da = desc_k_sw128(base + P::OFF_AQ + (uint32_t)sq * AQ_BYTES);
                    const uint64_t dw = desc_k_sw128(base + P::OFF_W + (uint32_t)sw * W_BYTES);
                    const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                    for (int k4 = 0; k4 < BK / 32; ++k4)
                        mma_f8(d, da + (uint64_t)(2 * k4), dw + (uint64_t)(2 * k4), kIdesc, k4 > 0 ? 1u : 0u);
                    mma_commit(bar(P::B_TFULL + buf));
                    mma_commit(bar(P::B_EMPTY_W + sw));
                    mma_commit(bar(P::B_EMPTY_Q + sq));
                    ++iq; ++iw; ++it;
                }
            }
            mma_commit(bar(P::B_MMA_DONE));
            bar_drain(bar(P::B_MMA_DONE), 0u);
        }
    } else {
        // ---------------------------------------------------- promotion
        set_max_regs_inc<REGQ_ACC>();
        const int q = warp & 3, h = (warp - 4) >> 2;
        const int rloc = 32 * q + lane;
        int it = 0;
        bool ok = true;
        F2 acc[64];
        for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
            int mt, nt;
            ctile_coords(g, u, mt, nt);
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0ull;
            const int64_t col0 = (int64_t)nt * BN + 128 * h;
            const bool half_in = col0 < g.n;
            const int64_t row = (int64_t)mt * BM + rloc;
            const bool row_in = row < g.m;
            const float* swp = g.sw + (half_in ? (col0 / 128) * nkb : 0);
            const float* sap = g.sa + (row_in ? row * nkb : 0);
            // Both scales two blocks ahead.
            float sw0 = half_in ? __ldg(swp) : 0.0f, sa0 = row_in ? __ldg(sap) : 0.0f;
            float sw1 = (half_in && nkb > 1) ? __ldg(swp + 1) : 0.0f;
            float sa1 = (row_in && nkb > 1) ? __ldg(sap + 1) : 0.0f;
            for (int kb = 0; kb < nkb; ++kb) {
                const bool more = kb + 2 < nkb;
                const float sw2 = (half_in && more) ? __ldg(swp + kb + 2) : 0.0f;
                const float sa2 = (row_in && more) ? __ldg(sap + kb + 2) : 0.0f;
                const F2 cf = f2_bcast(__fmul_rn(sa0, sw0));
                const int buf = it & 1;
                if (!(ok = bar_wait<1, false>(bar(P::B_TFULL + buf), (uint32_t)(it >> 1) & 1u, abort_flag, abort_addr))) break;
                tc_fence_after();
                promote_block_2x(acc, tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 128 * h), cf);
                tc_fence_before();
                bar_arrive(bar(P::B_TEMPTY + buf));
                ++it;
                sw0 = sw1; sw1 = sw2;
                sa0 = sa1; sa1 = sa2;
            }
            if (!ok) break;
            if (row_in && half_in) store_c_half(g, row, col0, acc);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// The same product for activations already quantized, on CTA pairs: a
// cluster of two CTAs (one per SM) computes a 256 x 256 tile of C with
// tcgen05.mma.cta_group::2 (M 256, N 256, K 32). CTA r of the pair loads
// activation rows [128 r, 128 r + 128) and weight rows [128 r, 128 r + 128)
// of the tile into its own shared memory; the MMA, issued by CTA 0, reads A
// split by rows and B split by columns across the pair and writes each
// CTA's 128 rows x 256 columns of the k-block's partial into that CTA's
// TMEM. Per k-block and SM, shared memory then takes 32 KB of TMA writes and
// serves 32 KB of operand reads (the one-CTA form: 48 KB and 48 KB), L2
// serves a third less, and one MMA instruction carries twice the work, so
// the issuing thread's per-block overhead is spread over twice the FLOPs.
// (Issuing each block as two N = 128 halves into four TMEM quarters, to give
// the promotion more slack, measured 23 % slower: twice the instructions and
// activation reads.)
// Roles (384 threads in each CTA):
//   warp 0       TMA: both operand tiles of the k-block into one ring stage;
//                the copies of both CTAs complete on the stage's barrier in
//                CTA 0, whose producer expects the pair's 64 KB;
//   warp 2       TMEM allocation for the pair (512 columns in each CTA); in
//                CTA 0 one thread issues the MMAs and commits each k-block to
//                the barriers of both CTAs (ring stage free, partial ready);
//   warps 4-11   promotion as in k_fp8_gemm_q, for this CTA's 128 rows;
//                each warp frees a TMEM buffer with one arrival on CTA 0's
//                barrier (16 per k-block).
struct PlanQ2 {
    static constexpr int S = 6;
    static constexpr uint32_t HALF = 128 * BK;                   // 128 rows x 128 bytes
    static constexpr uint32_t STAGE = 2 * HALF;                  // A half, then B half
    static constexpr uint32_t PAIR_TX = 2 * STAGE;               // both CTAs' bytes
    static constexpr uint32_t OFF_RING = 0;
    static constexpr uint32_t OFF_BAR = OFF_RING + S * STAGE;
    static constexpr int B_FULL = 0, B_EMPTY = B_FULL + S, B_TFULL = B_EMPTY + S, B_TEMPTY = B_TFULL + 2,
                         B_MMA_DONE = B_TEMPTY + 2, N_BAR = B_MMA_DONE + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + N_BAR * 8;   // [0] TMEM base, [1] abort flag
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(PAIR_TX < (1u << 20), "transaction count range");
};
// f32 accumulator, E4M3 x E4M3, both K-major, N 256, M 256 (the pair).
constexpr uint32_t kIdescPair = (1u << 4) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(dst_smem), "r"(cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// One arrival on the barrier at the same offset in both CTAs of the pair
// when the pair's MMAs issued before by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 :: "r"(bar), "h"((uint16_t)3) : "memory");
}
// Tiled TMA load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`cl_bar`, a cluster address).
__device__ __forceinline__ void tma_2d_pair(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t cl_bar) {
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"((uint64_t)tm), "r"(x), "r"(y), "r"(cl_bar) : "memory");
}
// Bounded pause (about `us` microseconds).
__device__ __forceinline__ void pause_us(uint32_t us) {
    for (uint32_t i = 0; i < us; ++i) __nanosleep(1000);
}

__global__ void __launch_bounds__(NT_Q, 1) k_fp8_gemm_q2(const __grid_constant__ CUtensorMap tm_a,
                                                          const __grid_constant__ CUtensorMap tm_w,
                                                          const GemmArgs g) {
    using P = PlanQ2;
    constexpr int S = P::S;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = sm_addr(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw_base);
    volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(sb + P::OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;
    const uint32_t abort_addr = base + P::OFF_MISC + 4;
    auto bar = [&](int i) -> uint32_t { return base + P::OFF_BAR + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) { bar_init(bar(P::B_FULL + i), 1); bar_init(bar(P::B_EMPTY + i), 1); }
        for (int i = 0; i < 2; ++i) { bar_init(bar(P::B_TFULL + i), 1); bar_init(bar(P::B_TEMPTY + i), 16); }
        bar_init(bar(P::B_MMA_DONE), 1);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) { prefetch_map(&tm_a); prefetch_map(&tm_w); }
    if (warp == 2) tmem_alloc_pair(base + P::OFF_MISC, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                   // both CTAs' barriers initialised
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int nkb = g.nkb;
    const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

    if (warp < 4) {
        set_max_regs_dec<REGQ_CTL>();
        if (warp == 0 && lane == 0) {
            // Both operand halves of this CTA, completing on CTA 0's stage barrier.
            int i = 0;
            bool ok = true;
            for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                int mt, nt;
                ctile_coords(g, u, mt, nt);
                for (int kb = 0; kb < nkb; ++kb) {
                    const int s = i % S;
                    if (!(ok = bar_wait<2, true>(bar(P::B_EMPTY + s), ((uint32_t)(i / S) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                    const uint32_t fb = bar(P::B_FULL + s);
                    if (leader) bar_expect_tx(fb, P::PAIR_TX);
                    const uint32_t cl_fb = map_rank(fb, 0u);
                    const uint32_t dst = base + P::OFF_RING + (uint32_t)s * P::STAGE;
                    tma_2d_pair(dst, &tm_a, kb * BK, mt * 256 + (int)rank * 128, cl_fb);
                    tma_2d_pair(dst + P::HALF, &tm_w, kb * BK, nt * 256 + (int)rank * 128, cl_fb);
                    ++i;
                }
            }
        } else if (warp == 2 && lane == 0) {
            if (leader) {
                // MMA issue for the pair.
                int i = 0, it = 0;
                bool ok = true;
                for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
                    for (int kb = 0; kb < nkb; ++kb) {
                        const int buf = it & 1;
                        if (!(ok = bar_wait<2, true>(bar(P::B_TEMPTY + buf), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, abort_addr))) break;
                        const int s = i % S;
                        if (!(ok = bar_wait<2, true>(bar(P::B_FULL + s), (uint32_t)(i / S) & 1u, abort_flag, abort_addr))) break;
                        tc_fence_after();
                        const uint32_t st = base + P::OFF_RING + (uint32_t)s * P::STAGE;
                        const uint64_t da = desc_k_sw128(st);
                        const uint64_t dw = desc_k_sw128(st + P::HALF);
                        const uint32_t d = tmem + (uint32_t)(buf * BN);
#pragma unroll
                        for (int k4 = 0; k4 < BK / 32; ++k4)
                            mma_f8_pair(d, da + (uint64_t)(2 * k4), dw + (uint64_t)(2 * k4), kIdescPair, k4 > 0 ? 1u : 0u);
                        mma_commit_pair(bar(P::B_TFULL + buf));
                        mma_commit_pair(bar(P::B_EMPTY + s));
                        ++i; ++it;
                    }
                }
                mma_commit_pair(bar(P::B_MMA_DONE));
            }
            // Both CTAs: the pair's MMAs (which write this CTA's TMEM) are done.
            bar_drain(bar(P::B_MMA_DONE), 0u);
        }
    } else {
        // ---------------------------------------------------- promotion
        set_max_regs_inc<REGQ_ACC>();
        const int q = warp & 3, h = (warp - 4) >> 2;
        const int rloc = 32 * q + lane;
        const uint32_t tempty0 = map_rank(bar(P::B_TEMPTY), 0u);
        int it = 0;
        bool ok = true;
        F2 acc[64];
        for (int64_t u = cid; ok && u < g.n_ctiles; u += ncl) {
            int mt, nt;
            ctile_coords(g, u, mt, nt);
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0ull;
            const int64_t col0 = (int64_t)nt * BN + 128 * h;
            const bool half_in = col0 < g.n;
            const int64_t row = (int64_t)mt * 256 + (int64_t)rank * 128 + rloc;
            const bool row_in = row < g.m;
            const float* swp = g.sw + (half_in ? (col0 / 128) * nkb : 0);
            const float* sap = g.sa + (row_in ? row * nkb : 0);
            float sw0 = half_in ? __ldg(swp) : 0.0f, sa0 = row_in ? __ldg(sap) : 0.0f;
            float sw1 = (half_in && nkb > 1) ? __ldg(swp + 1) : 0.0f;
            float sa1 = (row_in && nkb > 1) ? __ldg(sap + 1) : 0.0f;
            for (int kb = 0; kb < nkb; ++kb) {
                const bool more = kb + 2 < nkb;
                const float sw2 = (half_in && more) ? __ldg(swp + kb + 2) : 0.0f;
                const float sa2 = (row_in && more) ? __ldg(sap + kb + 2) : 0.0f;
                const F2 cf = f2_bcast(__fmul_rn(sa0, sw0));
                const int buf = it & 1;
                if (!(ok = bar_wait<2, true>(bar(P::B_TFULL + buf), (uint32_t)(it >> 1) & 1u, abort_flag, abort_addr))) break;
                tc_fence_after();
                promote_block_2x(acc, tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 128 * h), cf);
                tc_fence_before();
                __syncwarp();
                // The warp's TMEM reads have completed (tcgen05.wait::ld): the
                // arrival only has to follow them, so it needs no release (a
                // release at cluster scope would also wait for the scale loads
                // issued above for later blocks: measured 2x slower).
                if (lane == 0) {
                    if (leader) bar_arrive(bar(P::B_TEMPTY + buf));
                    else bar_arrive_remote_relaxed(tempty0 + 8u * (uint32_t)buf);
                }
                ++it;
                sw0 = sw1; sw1 = sw2;
                sa0 = sa1; sa1 = sa2;
            }
            if (!ok) break;
            if (row_in && half_in) store_c_half(g, row, col0, acc);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                   // no TMEM access or remote arrival left in the pair
    tc_fence_after();
    if (warp == 2) tmem_dealloc_pair(tmem, TMEM_COLS);
    // Every stage loaded was consumed unless the pair gave up (the flag is
    // visible here after the cluster barrier); then copies may still be in
    // flight to this CTA's ring or CTA 0's barriers: keep the shared memory
    // alive until they have landed.
    if (threadIdx.x == 0 && *abort_flag) pause_us(1000);
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

// Per device and kernel: the shared-memory limit is raised once, the launch
// register count is checked once (the setmaxnreg split above assumes
// REG_LAUNCH registers per thread at launch; any other count is refused),
// and the number of clusters that fit at once is queried once.
template <class T, int CL>
cudaError_t prepare_kernel(int* max_clusters) {
    static int ready[64] = {0};
    static int clusters[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorUnknown;
    if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
    if (__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        *max_clusters = clusters[dev];
        return cudaSuccess;
    }
    auto k = k_fp8_gemm<T, CL>;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, k);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != REG_LAUNCH) return cudaErrorNotSupported;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Plan<CL>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int n = sm_count() / CL;
    if (CL > 1) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(n * CL));
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = Plan<CL>::SMEM_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        e = cudaOccupancyMaxActiveClusters(&c, k, &cfg);
        if (e != cudaSuccess) return e;
        if (c < 1) return cudaErrorNotSupported;
        n = c;
    }
    clusters[dev] = n;
    __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    *max_clusters = n;
    return cudaSuccess;
}

template <class T, int CL>
cudaError_t launch_gemm(const void* a, int64_t m, int64_t k, const uint8_t* w, const float* sw, int64_t n,
                        void* c, int c_bf16, uint8_t* dq, float* ds, cudaStream_t st) {
    int max_clusters = 0;
    cudaError_t e = prepare_kernel<T, CL>(&max_clusters);
    if (e != cudaSuccess) return e;
    CUtensorMap ta, tw;
    if ((e = encode_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT16, a, (uint64_t)k, (uint64_t)m, (uint64_t)k * 2, 64,
                        Plan<CL>::RB)) != cudaSuccess)
        return e;
    if ((e = encode_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)k, (uint64_t)n, (uint64_t)k, BK,
                        BN)) != cudaSuccess)
        return e;
    GemmArgs g;
    g.m = m; g.n = n; g.k = k;
    g.nkb = (int)(k / BK);
    g.mtiles = (int)((m + BM - 1) / BM);
    g.ntiles = (int)((n + BN - 1) / BN);
    g.nct = (g.ntiles + CL - 1) / CL;
    g.band = min(16, g.mtiles);
    g.n_ctiles = (int64_t)g.mtiles * g.nct;
    g.sw = sw; g.c = c; g.c_bf16 = c_bf16; g.dump_q = dq; g.dump_s = ds;
    int64_t clusters = max_clusters;
    if (clusters > g.n_ctiles) clusters = g.n_ctiles;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(clusters * CL));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = Plan<CL>::SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_fp8_gemm<T, CL>, ta, tw, g);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_gemm_q(const uint8_t* ea, const float* sa, int64_t m, int64_t k, const uint8_t* w,
                          const float* sw, int64_t n, void* c, int c_bf16, cudaStream_t st) {
    static int ready[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorUnknown;
    if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
    if (!__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, k_fp8_gemm_q);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != REGQ_LAUNCH) return cudaErrorNotSupported;
        e = cudaFuncSetAttribute(k_fp8_gemm_q, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PlanQ::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    }
    CUtensorMap ta, tw;
    cudaError_t e;
    if ((e = encode_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, ea, (uint64_t)k, (uint64_t)m, (uint64_t)k, BK, BM)) !=
        cudaSuccess)
        return e;
    if ((e = encode_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)k, (uint64_t)n, (uint64_t)k, BK, BN)) !=
        cudaSuccess)
        return e;
    GemmArgs g = {};
    g.m = m; g.n = n; g.k = k;
    g.nkb = (int)(k / BK);
    g.mtiles = (int)((m + BM - 1) / BM);
    g.ntiles = (int)((n + BN - 1) / BN);
    g.nct = g.ntiles;
    g.band = min(16, g.mtiles);
    g.n_ctiles = (int64_t)g.mtiles * g.nct;
    g.sw = sw; g.c = c; g.c_bf16 = c_bf16; g.sa = sa;
    int64_t grid = sm_count();
    if (grid > g.n_ctiles) grid = g.n_ctiles;
    k_fp8_gemm_q<<<(unsigned)grid, NT_Q, PlanQ::SMEM_BYTES, st>>>(ta, tw, g);
    return cudaGetLastError();
}

cudaError_t launch_gemm_q2(const uint8_t* ea, const float* sa, int64_t m, int64_t k, const uint8_t* w,
                           const float* sw, int64_t n, void* c, int c_bf16, cudaStream_t st) {
    static int ready[64] = {0};
    static int pairs[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorUnknown;
    if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(NT_Q);
    cfg.dynamicSmemBytes = PlanQ2::SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, k_fp8_gemm_q2);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != REGQ_LAUNCH) return cudaErrorNotSupported;
        e = cudaFuncSetAttribute(k_fp8_gemm_q2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)PlanQ2::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3((unsigned)(sm_count() & ~1));
        int cnum = 0;
        e = cudaOccupancyMaxActiveClusters(&cnum, k_fp8_gemm_q2, &cfg);
        if (e != cudaSuccess) return e;
        if (cnum < 1) return cudaErrorNotSupported;
        pairs[dev] = cnum;
        __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    }
    CUtensorMap ta, tw;
    cudaError_t e;
    if ((e = encode_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, ea, (uint64_t)k, (uint64_t)m, (uint64_t)k, BK, 128)) !=
        cudaSuccess)
        return e;
    if ((e = encode_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)k, (uint64_t)n, (uint64_t)k, BK, 128)) !=
        cudaSuccess)
        return e;
    GemmArgs g = {};
    g.m = m; g.n = n; g.k = k;
    g.nkb = (int)(k / BK);
    g.mtiles = (int)((m + 255) / 256);             // pair tiles of 256 rows
    g.ntiles = (int)((n + BN - 1) / BN);
    g.nct = g.ntiles;
    g.band = min(16, g.mtiles);
    g.n_ctiles = (int64_t)g.mtiles * g.nct;
    g.sw = sw; g.c = c; g.c_bf16 = c_bf16; g.sa = sa;
    int64_t np = pairs[dev];
    if (np > g.n_ctiles) np = g.n_ctiles;
    cfg.gridDim = dim3((unsigned)(2 * np));
    cfg.stream = st;
    e = cudaLaunchKernelEx(&cfg, k_fp8_gemm_q2, ta, tw, g);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Cluster size: activations are quantized once per cluster of CL CTAs that
// share them; CL = 4 when the tile row holds at least four N tiles.
template <class T>
cudaError_t launch_gemm_any(const void* a, int64_t m, int64_t k, const uint8_t* w, const float* sw, int64_t n,
                            void* c, int c_bf16, uint8_t* dq, float* ds, cudaStream_t st, int cl) {
    if (cl <= 0) cl = (n > 3 * BN) ? 4 : ((n > BN) ? 2 : 1);
    switch (cl) {
        case 1: return launch_gemm<T, 1>(a, m, k, w, sw, n, c, c_bf16, dq, ds, st);
        case 2: return launch_gemm<T, 2>(a, m, k, w, sw, n, c, c_bf16, dq, ds, st);
        case 4: return launch_gemm<T, 4>(a, m, k, w, sw, n, c, c_bf16, dq, ds, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

// Kernel for bq_fp8_block_gemm_quantized: BQ_GEMM_PAIR = 0 forces the
// one-CTA kernel, 1 the CTA-pair kernel (for measurement); otherwise the
// pair kernel takes every m above 128.
int gemm_pair_override() {
    static const int v = [] {
        const char* e = getenv("BQ_GEMM_PAIR");
        if (!e) return -1;
        const int x = atoi(e);
        return (x == 0 || x == 1) ? x : -1;
    }();
    return v;
}

// Cluster size for bq_fp8_block_gemm: BQ_GEMM_CLUSTER = 1, 2 or 4 forces one
// (for measurement); unset or anything else lets the shape decide.
int gemm_cluster_override() {
    static const int v = [] {
        const char* e = getenv("BQ_GEMM_CLUSTER");
        const int x = e ? atoi(e) : 0;
        return (x == 1 || x == 2 || x == 4) ? x : 0;
    }();
    return v;
}

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
    const int cl = bq::gemm_cluster_override();
    const cudaError_t e = (a_dtype == BQ_BF16)
        ? bq::launch_gemm_any<__nv_bfloat16>(a, m, k, w_e4m3, w_scale, n, c, c_dtype == BQ_BF16, a_e4m3, a_scale, st, cl)
        : bq::launch_gemm_any<__half>(a, m, k, w_e4m3, w_scale, n, c, c_dtype == BQ_BF16, a_e4m3, a_scale, st, cl);
    if (e == cudaErrorNotSupported) return BQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

extern "C" bq_status bq_fp8_block_gemm_quantized(const uint8_t* a_e4m3, const float* a_scale, int64_t m,
                                                 int64_t k, const uint8_t* w_e4m3, const float* w_scale,
                                                 int64_t n, void* c, bq_dtype c_dtype, void* stream) {
    if (c_dtype != BQ_F32 && c_dtype != BQ_BF16) return BQ_ERR_UNSUPPORTED;
    if (m < 0 || n < 0 || k <= 0 || k % 128 != 0) return BQ_ERR_INVALID_ARG;
    if (m >= (1ll << 31) || n >= (1ll << 31) || k >= (1ll << 31)) return BQ_ERR_INVALID_ARG;
    if (m == 0 || n == 0) return BQ_OK;
    if (!a_e4m3 || !a_scale || !w_e4m3 || !w_scale || !c) return BQ_ERR_INVALID_ARG;
    if (((uintptr_t)a_e4m3 & 15u) || ((uintptr_t)w_e4m3 & 15u) || ((uintptr_t)w_scale & 3u) ||
        ((uintptr_t)a_scale & 3u) || ((uintptr_t)c & 15u))
        return BQ_ERR_MISALIGNED;
    const int pair = bq::gemm_pair_override();
    const bool use_pair = pair < 0 ? m > 128 : pair == 1;
    const cudaError_t e = use_pair
        ? bq::launch_gemm_q2(a_e4m3, a_scale, m, k, w_e4m3, w_scale, n, c, c_dtype == BQ_BF16, (cudaStream_t)stream)
        : bq::launch_gemm_q(a_e4m3, a_scale, m, k, w_e4m3, w_scale, n, c, c_dtype == BQ_BF16, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return BQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
