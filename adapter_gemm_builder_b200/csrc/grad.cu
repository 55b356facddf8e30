// grad.cu -- the adapter gradients of the LoRA layer for training on a frozen
// 8-bit base (EpiLoRA abstract, sentence 6; the chain rule of
// y = x.W^T + s_a (x.A_a).B_a from the Punica README's "How?"):
//   dA_a[k][j] = s_a sum_{m in a} x[m][k] u[m][j],   u = dY.B_a^T
//   dB_a[j][n] = s_a sum_{m in a} v[m][j] dY[m][n],  v = x.A_a
// and the transposed pool (A'_a = B_a^T, B'_a = A_a^T) with which the backward's
// dX = dY.W + s_a (dY.B_a^T).A_a^T is the forward's fused GEMM of dY.
//
// Both gradients are one kernel, a segmented sum of outer products: for every
// active adapter and every block of 256 "long" indices l (k of dA, n of dB),
// thread l keeps the r_a sums of one row of the output and walks the adapter's
// tokens, 32 at a time: the tokens' short vectors (u or v, fp32) are staged in
// shared memory and each thread reads its token rows' bf16 element of x or dY
// (coalesced across the block; eight tokens' loads are issued before their
// FMAs, so their latencies overlap). Bound by HBM: x or dY rows of the adapter's
// tokens in, the gradient rows out.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kGThreads = 256;
constexpr int kTokChunk = 32;

struct GradParams {
    const uint16_t* lng;  // bf16 [T][L]: x (dA) or dY (dB), by token index
    const float* shrt;    // fp32 [T][r_max]: u (dA) or v (dB), by token index
    float* out;           // dA [n_adapters][L][r_max] or dB [n_adapters][r_max][L]
    const int32_t* perm;
    const int32_t* indptr;
    const int32_t* active;
    const int32_t* counts;
    const int32_t* ranks;
    const float* scales;
    int L, r_max, n_adapters;
};

// kRowMajorLong: the output is [L][r_max] (dA); else [r_max][L] (dB). MAXR: the
// pool's r_max rounded up to 16 or 64 (the sums a thread keeps).
template <bool kRowMajorLong, int MAXR>
__global__ void __launch_bounds__(kGThreads)
grad_outer_kernel(const GradParams p)
{
    __shared__ float s_short[kTokChunk][MAXR];
    __shared__ int s_tok[kTokChunk];
    ptx::pdl_wait();  // the shrinks that produced u / v come first in the stream
    const int slot = blockIdx.y;
    if (slot >= p.counts[1]) return;  // fewer active adapters than slots
    const int a = p.active[slot];
    int r = p.ranks ? p.ranks[a] : p.r_max;
    r = max(1, min(r, p.r_max));
    const float s = p.scales ? p.scales[a] : 1.f;
    const int l = blockIdx.x * kGThreads + threadIdx.x;
    const int t0 = p.indptr[a], t1 = p.indptr[a + 1];
    float acc[MAXR];
#pragma unroll
    for (int j = 0; j < MAXR; ++j) acc[j] = 0.f;
    for (int c0 = t0; c0 < t1; c0 += kTokChunk) {
        const int nc = min(kTokChunk, t1 - c0);
        __syncthreads();  // the previous chunk's short vectors are consumed
        if (threadIdx.x < nc) s_tok[threadIdx.x] = p.perm[c0 + threadIdx.x];
        __syncthreads();
        for (int i = threadIdx.x; i < nc * MAXR; i += kGThreads) {
            const int t = i / MAXR, j = i % MAXR;
            s_short[t][j] = j < r ? p.shrt[(size_t)s_tok[t] * p.r_max + j] : 0.f;
        }
        __syncthreads();
        if (l < p.L) {
            // eight tokens at a time: their long elements first (independent loads, in
            // flight together), then the FMAs (columns past the rank hold zeros)
            for (int t0 = 0; t0 < nc; t0 += 8) {
                float lv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    lv[u] = t0 + u < nc ? __uint_as_float((uint32_t)p.lng[(size_t)s_tok[t0 + u] * p.L + l] << 16)
                                        : 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (t0 + u < nc)
#pragma unroll
                        for (int j = 0; j < MAXR; ++j) acc[j] = fmaf(lv[u], s_short[t0 + u][j], acc[j]);
            }
        }
    }
    ptx::pdl_launch_dependents();
    if (l >= p.L) return;
    if (kRowMajorLong) {
        float4* o = reinterpret_cast<float4*>(p.out + ((size_t)a * p.L + l) * p.r_max);
#pragma unroll
        for (int j = 0; j < MAXR; j += 4)
            if (j < p.r_max)
                o[j >> 2] = make_float4(j < r ? s * acc[j] : 0.f, j + 1 < r ? s * acc[j + 1] : 0.f,
                                        j + 2 < r ? s * acc[j + 2] : 0.f, j + 3 < r ? s * acc[j + 3] : 0.f);
    } else {
#pragma unroll
        for (int j = 0; j < MAXR; ++j)
            if (j < p.r_max) p.out[((size_t)a * p.r_max + j) * p.L + l] = j < r ? s * acc[j] : 0.f;
    }
}

// A'_a[n][j] = B_a[j][n] and B'_a[j][k] = A_a[k][j] for the active adapters.
__global__ void __launch_bounds__(kGThreads)
transpose_pool_kernel(const uint16_t* A, const uint16_t* B, uint16_t* At, uint16_t* Bt, const int32_t* active,
                      const int32_t* counts, int K, int N, int r_max)
{
    ptx::pdl_wait();
    const int slot = blockIdx.y;
    if (slot >= counts[1]) return;
    const size_t a = (size_t)active[slot];
    const int i = blockIdx.x * kGThreads + threadIdx.x;
    if (i < N) {  // row n of A'_a: the column n of B_a (r_max bf16, 16-byte pieces)
        for (int j0 = 0; j0 < r_max; j0 += 8) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h)
                w[h] = (uint32_t)B[(a * r_max + j0 + 2 * h) * N + i] |
                       ((uint32_t)B[(a * r_max + j0 + 2 * h + 1) * N + i] << 16);
            *reinterpret_cast<uint4*>(At + (a * N + i) * r_max + j0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    if (i < K) {  // column k of B'_a: the row k of A_a
        const uint16_t* src = A + (a * K + i) * r_max;
        for (int j = 0; j < r_max; ++j) Bt[(a * r_max + j) * K + i] = src[j];
    }
    ptx::pdl_launch_dependents();
}

// u[t][j] = sum_c vg[c][pos][j] for the token t = perm[pos] of every position with an
// adapter: the down-projection the backward's fused GEMM already computed (dY.B^T
// with the transposed pool, in its workspace as v_rep partial copies in segment
// order), so no second shrink of dY is needed.
__global__ void __launch_bounds__(kGThreads)
gather_u_kernel(const float* vg, int v_rep, const int32_t* perm, const int32_t* counts, int M, int r_max, float* u)
{
    ptx::pdl_wait();  // the GEMM wrote vg
    const int n_valid = counts[0];
    const int i = blockIdx.x * kGThreads + threadIdx.x;
    const int pos = i / r_max, j = i - pos * r_max;
    if (pos < n_valid && pos < M) {
        float acc = 0.f;
        for (int c = 0; c < v_rep; ++c) acc += vg[((size_t)c * M + pos) * r_max + j];
        u[(size_t)perm[pos] * r_max + j] = acc;
    }
    ptx::pdl_launch_dependents();
}

cudaError_t launch_pdl(const void* kern, dim3 grid, void** args, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kGThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, kern, args);
}

}  // namespace

cudaError_t launch_transpose_pool(const lora_pool_t& pool, const lora_segments_t& seg, void* At, void* Bt,
                                  cudaStream_t stream)
{
    const int K = pool.h_in, N = pool.h_out;
    const dim3 grid((unsigned)((max(K, N) + kGThreads - 1) / kGThreads), (unsigned)pool.n_adapters, 1);
    const uint16_t* A = static_cast<const uint16_t*>(pool.A);
    const uint16_t* B = static_cast<const uint16_t*>(pool.B);
    uint16_t* at = static_cast<uint16_t*>(At);
    uint16_t* bt = static_cast<uint16_t*>(Bt);
    const int32_t* active = seg.active;
    const int32_t* counts = seg.counts;
    int k = K, n = N, r = pool.r_max;
    void* args[] = {&A, &B, &at, &bt, &active, &counts, &k, &n, &r};
    return launch_pdl((const void*)transpose_pool_kernel, grid, args, stream);
}

cudaError_t launch_gather_u(const float* vg, int v_rep, const lora_segments_t& seg, int M, int r_max, float* u,
                            cudaStream_t stream)
{
    const dim3 grid((unsigned)(((long long)M * r_max + kGThreads - 1) / kGThreads), 1, 1);
    const int32_t* perm = seg.perm;
    const int32_t* counts = seg.counts;
    int m = M, r = r_max;
    void* args[] = {&vg, &v_rep, &perm, &counts, &m, &r, &u};
    return launch_pdl((const void*)gather_u_kernel, grid, args, stream);
}

cudaError_t launch_grad_outer(bool row_major_long, const void* lng, const float* shrt, int L,
                              const lora_pool_t& pool, const lora_segments_t& seg, float* out, cudaStream_t stream)
{
    GradParams p = {};
    p.lng = static_cast<const uint16_t*>(lng);
    p.shrt = shrt;
    p.out = out;
    p.perm = seg.perm;
    p.indptr = seg.indptr;
    p.active = seg.active;
    p.counts = seg.counts;
    p.ranks = pool.ranks;
    p.scales = pool.scales;
    p.L = L;
    p.r_max = pool.r_max;
    p.n_adapters = pool.n_adapters;
    const dim3 grid((unsigned)((L + kGThreads - 1) / kGThreads), (unsigned)pool.n_adapters, 1);
    void* args[] = {&p};
    const bool r16 = pool.r_max <= 16;
    const void* kern = row_major_long ? (r16 ? (const void*)grad_outer_kernel<true, 16> : (const void*)grad_outer_kernel<true, 64>)
                                      : (r16 ? (const void*)grad_outer_kernel<false, 16> : (const void*)grad_outer_kernel<false, 64>);
    return launch_pdl(kern, grid, args, stream);
}

}  // namespace lora
