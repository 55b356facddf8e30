// merge.cu -- token-wise merge of router-selected LoRA adapters into the
// backbone weight (LoRA-Switch abstract, shd-paper.top page: for each token a
// router switches the adapters and their weights, which are merged into the
// backbone before inference, all selected adapters in one fused kernel):
//   W_out[n][k] = bf16( W[n][k] + sum_e g_e s_a sum_{j < r_a} A_a[k][j] B_a[j][n] ).
//
// The kernel is bound by HBM (W read once, W_out written once); the adapters'
// slices are re-read from L2. One CTA per tile of 64 rows (n) x 128 columns
// (k) of W:
//   1. 16-byte cp.async copies of the W tile, of the selected adapters' A rows
//      for the tile's columns and of their B columns for the tile's rows into
//      padded shared-memory tiles (no bank conflicts for ldmatrix);
//   2. per selected adapter, bf16 mma.sync (m16n8k16, fp32 accumulate) of
//      D[n][k] = sum_j B[j][n] A[k][j] over its rank, then D += g s D_e in
//      fp32 (the gate and scale are applied to the fp32 product, so the only
//      rounding of the merged weight is the final one to bf16);
//   3. the tile updated in shared memory, a pair of consecutive k per access,
//      and stored with 16-byte stores.
// W_out may be W itself (each CTA reads its whole tile before writing it).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kTN = 64;   // W rows per tile
constexpr int kTK = 128;  // W columns per tile
constexpr int kWarps = 8;
constexpr int kThreadsM = kWarps * 32;
constexpr int kWPitch = kTK * 2 + 16;  // bytes per W row in shared memory
constexpr int kBPitch = kTN * 2 + 16;  // bytes per B row (one rank index j)

struct MergeParams {
    const uint16_t* W;
    uint16_t* Wout;
    const uint16_t* A;  // [n_adapters][K][r_max]
    const uint16_t* B;  // [n_adapters][r_max][N]
    const int32_t* ranks;
    const float* scales;
    const int32_t* sel;
    const float* gates;
    int n_sel, N, K, n_adapters, r_max;
    int a_pitch;  // bytes per A row in shared memory: (n_sel * r16_max) * 2 + 16
};

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kThreadsM, 4)
merge_kernel(const MergeParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int s_a[8], s_r[8], s_j0[8];
    __shared__ float s_c[8];
    __shared__ int s_ne;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k0 = blockIdx.x * kTK, n0 = blockIdx.y * kTN;
    const int r_cap = (p.r_max + 15) & ~15;
    uint8_t* Ws = smem;                                  // [kTN][kWPitch]
    uint8_t* As = Ws + kTN * kWPitch;                    // [kTK][a_pitch]
    uint8_t* Bs = As + kTK * p.a_pitch;                  // [n_sel * r_cap][kBPitch]

    // the router output may come from the previous kernel in the stream
    ptx::pdl_wait();
    if (tid == 0) {
        int ne = 0, j0 = 0;
        for (int e = 0; e < p.n_sel; ++e) {
            const int a = p.sel[e];
            if (a < 0 || a >= p.n_adapters) continue;
            int r = p.ranks ? p.ranks[a] : p.r_max;
            r = max(1, min(r, p.r_max));
            s_a[ne] = a;
            s_r[ne] = r;
            s_j0[ne] = j0;
            s_c[ne] = p.gates[e] * (p.scales ? p.scales[a] : 1.f);
            j0 += (r + 15) & ~15;
            ++ne;
        }
        s_ne = ne;
    }
    __syncthreads();
    ptx::pdl_launch_dependents();
    const int ne = s_ne;

    // ---- 1. copies: the W tile, A rows [k0, k0 + 128) and B columns [n0, n0 + 64) of each
    // selected adapter (columns / rows past the rank zeroed, out-of-range rows zero-filled)
    const int wchunks = kTK / 8;
    for (int i = tid; i < kTN * wchunks; i += kThreadsM) {
        const int row = i / wchunks, c = i - row * wchunks;
        const int n = n0 + row, k = k0 + c * 8;
        const bool in = n < p.N && k < p.K;
        ptx::cp_async16(ptx::smem_u32(Ws + row * kWPitch + c * 16), in ? p.W + (size_t)n * p.K + k : p.W,
                        in ? 16u : 0u);
    }
    for (int e = 0; e < ne; ++e) {
        const int a = s_a[e], r16 = (s_r[e] + 15) & ~15, j0 = s_j0[e];
        const int ach = r16 / 8;  // 16-byte chunks of an A row slice
        for (int i = tid; i < kTK * ach; i += kThreadsM) {
            const int row = i / ach, c = i - row * ach;
            const int k = k0 + row;
            const bool in = k < p.K && c * 8 < p.r_max;
            ptx::cp_async16(ptx::smem_u32(As + row * p.a_pitch + (j0 + c * 8) * 2),
                            in ? p.A + ((size_t)a * p.K + k) * p.r_max + c * 8 : p.A, in ? 16u : 0u);
        }
        const int bch = kTN / 8;
        for (int i = tid; i < r16 * bch; i += kThreadsM) {
            const int j = i / bch, c = i - j * bch;
            const int n = n0 + c * 8;
            const bool in = j < p.r_max && n < p.N;
            ptx::cp_async16(ptx::smem_u32(Bs + (j0 + j) * kBPitch + c * 16),
                            in ? p.B + ((size_t)a * p.r_max + j) * p.N + n : p.B, in ? 16u : 0u);
        }
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait<0>();
    __syncthreads();
    // the pool's padding past each rank (A columns, B rows j >= r) is never used: zero it
    for (int e = 0; e < ne; ++e) {
        const int r = s_r[e], r16 = (r + 15) & ~15, j0 = s_j0[e];
        if (r == r16) continue;
        for (int i = tid; i < kTK * (r16 - r); i += kThreadsM) {
            const int row = i / (r16 - r), j = r + (i - row * (r16 - r));
            *reinterpret_cast<uint16_t*>(As + row * p.a_pitch + (j0 + j) * 2) = 0;
        }
        for (int i = tid; i < (r16 - r) * kTN; i += kThreadsM) {
            const int j = r + i / kTN, n = i % kTN;
            *reinterpret_cast<uint16_t*>(Bs + (j0 + j) * kBPitch + n * 2) = 0;
        }
    }
    __syncthreads();

    // ---- 2. warp w: D rows n = 16 (w % 4) .. + 15, columns k = 64 (w / 4) .. + 63, in two
    // passes of 32 columns (4 MMA tiles of 8; fewer live accumulators): D[n][k] =
    // sum_j B[j][n] A[k][j], so a thread's accumulator pairs are pairs of consecutive k,
    // contiguous in W's row n
    const int mt = warp & 3, kh = warp >> 2;
    const int gq = lane >> 2, tq = lane & 3;
    // A operand (n x j, from B stored [j][n]): transposed 8x8 loads, lane -> row j, n block
    const uint32_t a_row = ptx::smem_u32(Bs + ((lane & 7) + ((lane >> 4) << 3)) * kBPitch +
                                         (mt * 16 + ((lane >> 3) & 1) * 8) * 2);
    for (int pass = 0; pass < 2; ++pass) {
        const int kq = kh * 64 + pass * 32;  // first column of this pass
        // B operand (j x k, from A stored [k][j]): two k tiles per 4-matrix load
        const uint32_t b_row = ptx::smem_u32(As + (kq + ((lane >> 4) << 3) + (lane & 7)) * p.a_pitch +
                                             ((lane >> 3) & 1) * 16);
        float acc[4][4], part[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;
        for (int e = 0; e < ne; ++e) {
            const int r16 = (s_r[e] + 15) & ~15, j0 = s_j0[e];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) part[t][i] = 0.f;
            for (int ks = 0; ks < r16 / 16; ++ks) {
                const int j = j0 + ks * 16;
                uint32_t af[4];
                ptx::ldsm_x4_t(a_row + j * kBPitch, af[0], af[1], af[2], af[3]);
#pragma unroll
                for (int t = 0; t < 4; t += 2) {
                    uint32_t b[4];
                    ptx::ldsm_x4(b_row + t * 8 * p.a_pitch + j * 2, b[0], b[1], b[2], b[3]);
                    ptx::mma_bf16_16816(part[t], af, b[0], b[1]);
                    ptx::mma_bf16_16816(part[t + 1], af, b[2], b[3]);
                }
            }
            const float c = s_c[e];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[t][i] = fmaf(c, part[t][i], acc[t][i]);
        }
        // ---- 3. W tile += D: the fragment's pairs (n = gq or gq + 8, k = 2 tq, 2 tq + 1)
        if (ne > 0) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = mt * 16 + gq + h * 8;
                    const int k = kq + t * 8 + tq * 2;
                    uint32_t* w = reinterpret_cast<uint32_t*>(Ws + n * kWPitch + k * 2);
                    const uint32_t wv = *w;
                    const float f0 = __uint_as_float(wv << 16) + acc[t][2 * h];
                    const float f1 = __uint_as_float(wv & 0xffff0000u) + acc[t][2 * h + 1];
                    *w = pack2(f0, f1);
                }
        }
    }
    __syncthreads();
    for (int i = tid; i < kTN * wchunks; i += kThreadsM) {
        const int row = i / wchunks, c = i - row * wchunks;
        const int n = n0 + row, k = k0 + c * 8;
        if (n < p.N && k < p.K)
            *reinterpret_cast<uint4*>(p.Wout + (size_t)n * p.K + k) =
                *reinterpret_cast<const uint4*>(Ws + row * kWPitch + c * 16);
    }
}

}  // namespace

cudaError_t launch_lora_switch_merge(const void* W, int N, int K, const lora_pool_t& pool, const int32_t* sel,
                                     const float* gates, int n_sel, void* W_out, cudaStream_t stream)
{
    MergeParams p = {};
    p.W = static_cast<const uint16_t*>(W);
    p.Wout = static_cast<uint16_t*>(W_out);
    p.A = static_cast<const uint16_t*>(pool.A);
    p.B = static_cast<const uint16_t*>(pool.B);
    p.ranks = pool.ranks;
    p.scales = pool.scales;
    p.sel = sel;
    p.gates = gates;
    p.n_sel = n_sel;
    p.N = N;
    p.K = K;
    p.n_adapters = pool.n_adapters;
    p.r_max = pool.r_max;
    const int r_cap = (pool.r_max + 15) & ~15;
    p.a_pitch = n_sel * r_cap * 2 + 16;
    const size_t smem = (size_t)kTN * kWPitch + (size_t)kTK * p.a_pitch + (size_t)n_sel * r_cap * kBPitch;
    cudaError_t e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((K + kTK - 1) / kTK), (unsigned)((N + kTN - 1) / kTN), 1);
    cfg.blockDim = dim3(kThreadsM, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_kernel, p);
}

}  // namespace lora
