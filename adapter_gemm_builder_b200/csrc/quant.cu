// quant.cu -- per-row FP8 (E4M3) quantisation for the 8-bit base GEMM.
//
// The pages make the base GEMM 8-bit (EpiLoRA abstract, sentence 2) without
// fixing the scaling; rows are scaled by amax/448 so the largest magnitude of
// each row lands on the largest finite E4M3 value, then rounded to nearest
// even with saturation. One CTA per output row; both divisions are IEEE
// binary32 divisions rounded to nearest (__fdiv_rn), so the result does not
// depend on compiler flags.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kThreads = 256;

// kCopy: the rows are copied as bf16 (the 16-bit GEMM's operand in segment order), sx = 1.
template <bool kCopy>
__global__ void __launch_bounds__(kThreads)
quantize_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int K,
                     uint8_t* __restrict__ xq, float* __restrict__ sx, uint32_t* __restrict__ zero,
                     size_t zero_words)
{
    __shared__ float s_red[kThreads / 32];
    // launched as a programmatic dependent of the previous kernel (which may produce x
    // or still read this call's scratch): wait for it, then let the GEMM start streaming
    // its weights
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    if (zero) {  // scratch the dependent GEMM accumulates into (block b: its slice)
        const size_t per = (zero_words + gridDim.x - 1) / gridDim.x;
        const size_t z0 = per * blockIdx.x, z1 = min(zero_words, z0 + per);
        for (size_t i = z0 + threadIdx.x; i < z1; i += kThreads) zero[i] = 0u;
    }
    const int prow = blockIdx.x;
    const int row = perm ? perm[prow] : prow;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)row * K);
    const int n16 = K >> 3;  // 8 bf16 per 16-byte chunk
    if constexpr (kCopy) {
        uint4* dst = reinterpret_cast<uint4*>(xq + (size_t)prow * K * 2);
        for (int i = threadIdx.x; i < n16; i += kThreads) dst[i] = src[i];
        if (threadIdx.x == 0) sx[prow] = 1.f;
        return;
    }

    float amax = 0.f;
    for (int i = threadIdx.x; i < n16; i += kThreads) {
        const uint4 c = src[i];
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[e] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[e] & 0xffff0000u)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = s_red[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, s_red[i]);
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
    if (threadIdx.x == 0) sx[prow] = s;

    uint2* dst = reinterpret_cast<uint2*>(xq + (size_t)prow * K);
    for (int i = threadIdx.x; i < n16; i += kThreads) {
        const uint4 c = src[i];
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        uint32_t out[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float a0 = __fdiv_rn(__uint_as_float(w[2 * e] << 16), s);
            const float a1 = __fdiv_rn(__uint_as_float(w[2 * e] & 0xffff0000u), s);
            const float a2 = __fdiv_rn(__uint_as_float(w[2 * e + 1] << 16), s);
            const float a3 = __fdiv_rn(__uint_as_float(w[2 * e + 1] & 0xffff0000u), s);
            out[e] = (uint32_t)ptx::cvt_e4m3x2(a0, a1) | ((uint32_t)ptx::cvt_e4m3x2(a2, a3) << 16);
        }
        dst[i] = make_uint2(out[0], out[1]);
    }
}

// OCP MX FP4 quantisation of weight rows: thread = (row n, block b of 32
// values). X = 2^(floor(log2(amax)) - 2) as an E8M0 exponent clamped to
// 0..254 (0 for an all-zero block); each value v / X (exact: a power of two)
// rounded to the nearest E2M1 value, ties to the even fraction bit, magnitudes
// past 6 saturated. Codes are packed two per byte, element 2i in the low
// nibble, in tiles of 128 rows x 64 values (the GEMM's k-block): tile (n / 128,
// k / 64) is 4096 contiguous bytes, row n % 128 at 32-byte pitch, so one
// k-block's weights arrive as one contiguous copy. The scales are stored per
// group of 128 rows, block-major ([n / 128][b][n % 128]), so one k-block's
// scales for 128 rows are contiguous too.
__global__ void __launch_bounds__(kThreads)
mxfp4_quantize_kernel(const uint16_t* __restrict__ W, int N, int K, uint8_t* __restrict__ Wp,
                      uint8_t* __restrict__ Wsc)
{
    const int nb = K / 32;
    const long long i = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (i >= (long long)N * nb) return;
    const int n = (int)(i / nb), b = (int)(i - (long long)n * nb);
    const uint4* src = reinterpret_cast<const uint4*>(W + (size_t)n * K + b * 32);
    uint32_t w[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 c = src[q];
        w[4 * q] = c.x;
        w[4 * q + 1] = c.y;
        w[4 * q + 2] = c.z;
        w[4 * q + 3] = c.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        amax = fmaxf(amax, fabsf(__uint_as_float(w[q] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(w[q] & 0xffff0000u)));
    }
    int e = 0;
    if (amax > 0.f) e = min(254, max(0, ilogbf(amax) - 2 + 127));
    auto code = [&](float v) -> uint32_t {
        const float a = fabsf(ldexpf(v, 127 - e));
        uint32_t c;
        if (a <= 0.25f) c = 0;
        else if (a < 0.75f) c = 1;
        else if (a <= 1.25f) c = 2;
        else if (a < 1.75f) c = 3;
        else if (a <= 2.5f) c = 4;
        else if (a < 3.5f) c = 5;
        else if (a <= 5.0f) c = 6;
        else c = 7;
        return c | (signbit(v) ? 8u : 0u);
    };
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t o = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint32_t word = w[4 * q + h];
            o |= code(__uint_as_float(word << 16)) << (8 * h);
            o |= code(__uint_as_float(word & 0xffff0000u)) << (8 * h + 4);
        }
        out[q] = o;
    }
    *reinterpret_cast<uint4*>(Wp + ((size_t)(n >> 7) * (K / 64) + (b >> 1)) * 4096 + (n & 127) * 32 + (b & 1) * 16) =
        make_uint4(out[0], out[1], out[2], out[3]);
    Wsc[((size_t)(n >> 7) * nb + b) * 128 + (n & 127)] = (uint8_t)e;
}

}  // namespace

cudaError_t launch_mxfp4_quantize(const void* W, int N, int K, uint8_t* Wp, uint8_t* Wsc, cudaStream_t stream)
{
    const long long threads = (long long)N * (K / 32);
    const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
    mxfp4_quantize_kernel<<<blocks, kThreads, 0, stream>>>(static_cast<const uint16_t*>(W), N, K, Wp, Wsc);
    return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const void* x, const int32_t* perm, int M, int K, uint8_t* xq,
                                 float* sx, void* zero, size_t zero_words, cudaStream_t stream,
                                 bool copy_bf16)
{
    if (M == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)M, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (copy_bf16)
        return cudaLaunchKernelEx(&cfg, quantize_rows_kernel<true>, static_cast<const uint16_t*>(x), perm, K, xq,
                                  sx, static_cast<uint32_t*>(zero), zero_words);
    return cudaLaunchKernelEx(&cfg, quantize_rows_kernel<false>, static_cast<const uint16_t*>(x), perm, K, xq, sx,
                              static_cast<uint32_t*>(zero), zero_words);
}

}  // namespace lora
