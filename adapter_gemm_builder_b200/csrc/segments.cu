// segments.cu -- group the tokens of a batch by adapter id.
//
// The SGMV of the Punica README ("How?") works on segments: runs of tokens
// that map to the same adapter. One CTA of 1024 threads builds them with a
// stable counting sort: a shared-memory histogram, block-wide prefix sums
// for the segment starts, the list of active adapters and their tile counts,
// then a scatter that keeps token order inside every segment (tokens are
// taken 1024 at a time, warp by warp, and within a warp the lanes that share
// an id rank themselves with __match_any_sync). The result is unique, so it
// is bit-exact and independent of thread timing.
#include <cuda_runtime.h>

#include "internal.h"

namespace lora {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Exclusive block-wide scan of one 64-bit value per thread; returns the
// thread's exclusive prefix and writes the block total to *total.
__device__ long long block_exclusive_scan(long long val, long long* total)
{
    __shared__ long long warp_sums[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long incl = val;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        long long n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        long long w = warp_sums[lane];
        long long wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            long long n = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += n;
        }
        warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    long long excl = incl - val + warp_sums[warp];
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(kThreads, 1)
build_segments_kernel(const int32_t* __restrict__ ids, int T, int n_adapters,
                      int32_t* __restrict__ perm, int32_t* __restrict__ indptr,
                      int32_t* __restrict__ active, int32_t* __restrict__ tile_ptr,
                      int32_t* __restrict__ tok_adapter, int32_t* __restrict__ counts)
{
    extern __shared__ int32_t smem[];
    const int nb = n_adapters + 1;  // bins: adapters, then "no adapter"
    int32_t* hist = smem;           // [nb]
    int32_t* cursor = smem + nb;    // [nb]
    __shared__ long long s_total;
    __shared__ int s_bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
    if (tid == 0) s_bad = 0;
    __syncthreads();

    // 1. histogram + per-token served id
    int bad = 0;
    for (int t = tid; t < T; t += kThreads) {
        const int id = ids[t];
        const bool ok = id >= 0 && id < n_adapters;
        if (!ok && id != -1) ++bad;
        tok_adapter[t] = ok ? id : -1;
        atomicAdd(&hist[ok ? id : n_adapters], 1);
    }
    if (bad) atomicAdd(&s_bad, bad);
    __syncthreads();

    // 2. segment starts: exclusive scan of hist over contiguous chunks
    const int chunk = (nb + kThreads - 1) / kThreads;
    const int c0 = min(nb, tid * chunk), c1 = min(nb, c0 + chunk);
    long long local = 0;
    for (int i = c0; i < c1; ++i) local += hist[i];
    long long base = block_exclusive_scan(local, &s_total);
    for (int i = c0; i < c1; ++i) {
        cursor[i] = (int32_t)base;
        indptr[i] = (int32_t)base;
        base += hist[i];
    }

    // 3. active adapters (count > 0) and their tiles: one packed scan of
    //    (#active << 32 | #tiles) over the adapter bins
    const int ca0 = min(n_adapters, tid * chunk), ca1 = min(n_adapters, ca0 + chunk);
    long long pk = 0;
    for (int a = ca0; a < ca1; ++a)
        if (hist[a] > 0)
            pk += (1ll << 32) + (hist[a] + LORA_TILE_TOKENS - 1) / LORA_TILE_TOKENS;
    __syncthreads();
    long long pbase = block_exclusive_scan(pk, &s_total);
    {
        int pos = (int)(pbase >> 32);
        int tiles = (int)(pbase & 0xffffffffll);
        for (int a = ca0; a < ca1; ++a) {
            if (hist[a] > 0) {
                active[pos] = a;
                tile_ptr[pos] = tiles;
                ++pos;
                tiles += (hist[a] + LORA_TILE_TOKENS - 1) / LORA_TILE_TOKENS;
            }
        }
    }
    __syncthreads();
    const int n_active = (int)(s_total >> 32);
    const int n_tiles = (int)(s_total & 0xffffffffll);
    for (int s = n_active + tid; s < n_adapters; s += kThreads) active[s] = -1;
    for (int s = n_active + tid; s <= n_adapters; s += kThreads) tile_ptr[s] = n_tiles;
    if (tid == 0) {
        counts[0] = cursor[n_adapters];  // start of the no-adapter tail = #valid
        counts[1] = n_active;
        counts[2] = s_bad;
        counts[3] = n_tiles;
    }
    __syncthreads();

    // 4. stable scatter, 1024 tokens per round, one warp at a time
    for (int t0 = 0; t0 < T; t0 += kThreads) {
        const int t = t0 + tid;
        const bool in = t < T;
        int bin = -2 - lane;  // unique per lane when out of range
        if (in) {
            const int id = ids[t];
            bin = (id >= 0 && id < n_adapters) ? id : n_adapters;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        for (int w = 0; w < kWarps; ++w) {
            if (warp == w) {
                int p = 0;
                if (in && lane == leader) {
                    p = cursor[bin];
                    cursor[bin] = p + __popc(peers);
                }
                p = __shfl_sync(0xffffffffu, p, leader);
                if (in) perm[p + rank] = t;
            }
            __syncthreads();
        }
    }
}

}  // namespace

cudaError_t launch_build_segments(const int32_t* ids, int T, int n_adapters,
                                  const lora_segments_t& seg, cudaStream_t stream)
{
    const size_t smem = sizeof(int32_t) * 2 * (size_t)(n_adapters + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(build_segments_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             2 * (LORA_MAX_ADAPTERS + 1) * (int)sizeof(int32_t));
        if (e != cudaSuccess) return e;
    }
    build_segments_kernel<<<1, kThreads, smem, stream>>>(ids, T, n_adapters, seg.perm, seg.indptr,
                                                         seg.active, seg.tile_ptr, seg.tok_adapter,
                                                         seg.counts);
    return cudaGetLastError();
}

}  // namespace lora
