// Encoder and divider diagnostics. bq_diag_encode_f32: f32 values encoded by the same
// device functions the quantize and dequantize kernels call — the E4M3 and
// E2M1 conversions of the microscaled formats and the round-to-nearest-even
// narrowing to bf16 / f16 of every float output — so that the encoders can
// be compared with a CPU definition over every f32 bit pattern.
#include "bq.h"
#include "bq_device.cuh"

namespace {

constexpr int kThreads = 256;

// Eight values per thread and step; `fmt` 0 E4M3, 1 E2M1 (packed), 2 bf16,
// 3 f16. n8 = n / 8 full groups of eight; the tail (n % 8 values) is encoded
// by thread 0 of block 0.
__global__ void __launch_bounds__(kThreads) k_diag_encode(const float* __restrict__ x, int64_t n,
                                                          int fmt, uint8_t* __restrict__ out) {
    const int64_t n8 = n / 8;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * kThreads) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * i);
        const float4 b = __ldg(reinterpret_cast<const float4*>(x) + 2 * i + 1);
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        if (fmt == 0) {
            uint2 w;
            w.x = bq::e4m3x4(v[0], v[1], v[2], v[3]);
            w.y = bq::e4m3x4(v[4], v[5], v[6], v[7]);
            reinterpret_cast<uint2*>(out)[i] = w;
        } else if (fmt == 1) {
            reinterpret_cast<uint32_t*>(out)[i] = bq::e2m1x8(v);
        } else {
            bq::U4 w;
            if (fmt == 2) {
                w.x = bq::pack_bf16x2(v[0], v[1]); w.y = bq::pack_bf16x2(v[2], v[3]);
                w.z = bq::pack_bf16x2(v[4], v[5]); w.w = bq::pack_bf16x2(v[6], v[7]);
            } else {
                w.x = bq::pack_f16x2(v[0], v[1]); w.y = bq::pack_f16x2(v[2], v[3]);
                w.z = bq::pack_f16x2(v[4], v[5]); w.w = bq::pack_f16x2(v[6], v[7]);
            }
            reinterpret_cast<bq::U4*>(out)[i] = w;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int64_t j = n8 * 8; j < n; ++j) {
            const float v = x[j];
            if (fmt == 0) {
                out[j] = (uint8_t)bq::e4m3x2(v, 0.0f);
            } else if (fmt == 1) {
                // n is even for E2M1: the tail is whole pairs.
                if ((j & 1) == 0) {
                    const float t[8] = {v, x[j + 1], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    out[j / 2] = (uint8_t)bq::e2m1x8(t);
                }
            } else if (fmt == 2) {
                reinterpret_cast<__nv_bfloat16*>(out)[j] = bq::to_out<__nv_bfloat16>(v);
            } else {
                reinterpret_cast<__half*>(out)[j] = bq::to_out<__half>(v);
            }
        }
    }
}

}  // namespace

extern "C" bq_status bq_diag_encode_f32(const float* x, int64_t n, bq_dtype fmt, void* out,
                                        void* stream) {
    int f;
    switch (fmt) {
        case BQ_E4M3: f = 0; break;
        case BQ_E2M1X2: f = 1; break;
        case BQ_BF16: f = 2; break;
        case BQ_F16: f = 3; break;
        default: return BQ_ERR_UNSUPPORTED;
    }
    if (n < 0 || (f == 1 && (n & 1))) return BQ_ERR_INVALID_ARG;
    if (n == 0) return BQ_OK;
    if (!x || !out) return BQ_ERR_INVALID_ARG;
    // Full groups of eight are read as two 16-byte vectors and written as one
    // 4-, 8- or 16-byte word: those need aligned pointers.
    const uintptr_t need_out = (f == 1) ? 4 : (f == 0 ? 8 : 16);
    if (((uintptr_t)x % 16) != 0 || ((uintptr_t)out % need_out) != 0) return BQ_ERR_MISALIGNED;
    const int64_t n8 = n / 8;
    int64_t blocks = (n8 + kThreads - 1) / kThreads;
    if (blocks < 1) blocks = 1;
    if (blocks > 148 * 8) blocks = 148 * 8;
    k_diag_encode<<<(unsigned)blocks, kThreads, 0, (cudaStream_t)stream>>>(x, n, f, (uint8_t*)out);
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

namespace {

// fl(x / s) on pairs through the kernels' reciprocal chains (CHAIN 0: five
// roundings, 1: four from a two-term reciprocal).
template <int CHAIN>
__global__ void __launch_bounds__(kThreads) k_diag_divide(const float2* __restrict__ x, int64_t n2, float s,
                                                           float2* __restrict__ out) {
    const bq::Recip r = bq::make_recip(s);
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n2; i += (int64_t)gridDim.x * kThreads) {
        const float2 v = x[i];
        const bq::F2 xv = bq::f2_pack(v.x, v.y);
        bq::F2 q;
        if (CHAIN == 0) {
            bq::Recip2 r2;
            r2.y = bq::f2_bcast(r.y);
            r2.ns = bq::f2_bcast(-r.s);
            q = bq::div_chain2(xv, r2);
        } else {
            q = bq::div_chain2(xv, bq::make_recip2(r));
        }
        float a, b;
        bq::f2_split(q, a, b);
        out[i] = make_float2(a, b);
    }
}

}  // namespace

extern "C" bq_status bq_diag_divide_f32(const float* x, int64_t n, float s, int chain, float* out,
                                        void* stream) {
    if (n < 0 || (n & 1) || (chain != 0 && chain != 1)) return BQ_ERR_INVALID_ARG;
    const float as = fabsf(s);
    if (!(as >= 0x1p-64f && as <= 0x1p64f)) return BQ_ERR_INVALID_ARG;
    if (n == 0) return BQ_OK;
    if (!x || !out) return BQ_ERR_INVALID_ARG;
    if (((uintptr_t)x % 8) != 0 || ((uintptr_t)out % 8) != 0) return BQ_ERR_MISALIGNED;
    const int64_t n2 = n / 2;
    int64_t blocks = (n2 + kThreads - 1) / kThreads;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (chain == 0)
        k_diag_divide<0><<<(unsigned)blocks, kThreads, 0, (cudaStream_t)stream>>>(
            reinterpret_cast<const float2*>(x), n2, s, reinterpret_cast<float2*>(out));
    else
        k_diag_divide<1><<<(unsigned)blocks, kThreads, 0, (cudaStream_t)stream>>>(
            reinterpret_cast<const float2*>(x), n2, s, reinterpret_cast<float2*>(out));
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
