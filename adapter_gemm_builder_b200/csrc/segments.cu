// segments.cu -- group the tokens of a batch by adapter id.
//
// The SGMV of the Punica README ("How?") works on segments: runs of tokens
// that map to the same adapter. One CTA builds them with a stable counting
// sort and cuts every segment into work tiles of at most LORA_TILE_TOKENS
// tokens. The order is unique (ascending id, ascending token index inside an
// id, the tokens without an adapter last), so the result is bit-exact and
// independent of thread timing.
//
// Two paths:
//  * small batches (T <= 1024 and a per-warp count table that fits shared
//    memory): one thread per token. Each warp ranks its lanes that share an
//    id with __match_any_sync and records per-id counts in its own row of a
//    [warps][bins] table; a column-wise exclusive scan of that table gives
//    every warp its offset inside each segment and the histogram itself.
//  * large batches: a histogram, then 1024 tokens per round scattered warp by
//    warp (the same per-warp ranking) to keep token order.
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kMaxThreads = 1024;

// Exclusive block-wide scan of one 64-bit value per thread (any blockDim that
// is a multiple of 32); *total receives the sum. Ends with __syncthreads.
__device__ long long block_exclusive_scan(long long val, long long* total)
{
    __shared__ long long warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    long long incl = val;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        long long n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        long long w = lane < nw ? warp_sums[lane] : 0;
        long long wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            long long n = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += n;
        }
        if (lane < nw) warp_sums[lane] = wi - w;
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    const long long excl = incl - val + warp_sums[warp];
    __syncthreads();
    return excl;
}

struct SegOut {
    int32_t* perm;
    int32_t* indptr;
    int32_t* active;
    int32_t* tiles;
    int32_t* tok_adapter;
    int32_t* counts;
    int tile_t;  // tokens per tile (tile_tokens_for)
};

// Given per-bin counts hist[0..nb) in shared memory (nb = n_adapters + 1),
// write starts[] (shared) and indptr, then the active list, the tile table
// and the counts. Every thread of the block must call it.
__device__ void finish_tables(const int32_t* hist, int32_t* starts, int n_adapters, int max_tiles,
                              int n_bad, const SegOut& o)
{
    __shared__ long long s_total;
    const int nb = n_adapters + 1;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int chunk = (nb + nthr - 1) / nthr;
    const int c0 = min(nb, tid * chunk), c1 = min(nb, c0 + chunk);
    long long local = 0;
    for (int i = c0; i < c1; ++i) local += hist[i];
    long long base = block_exclusive_scan(local, &s_total);
    for (int i = c0; i < c1; ++i) {
        starts[i] = (int32_t)base;
        o.indptr[i] = (int32_t)base;
        base += hist[i];
    }
    // active adapters and their tiles: one packed scan of (#active << 32 | #tiles)
    const int ca0 = min(n_adapters, c0), ca1 = min(n_adapters, c1);
    long long pk = 0;
    for (int a = ca0; a < ca1; ++a)
        if (hist[a] > 0) pk += (1ll << 32) + (hist[a] + o.tile_t - 1) / o.tile_t;
    const long long pbase = block_exclusive_scan(pk, &s_total);
    int pos = (int)(pbase >> 32);
    int tile = (int)(pbase & 0xffffffffll);
    for (int a = ca0; a < ca1; ++a) {
        const int c = hist[a];
        if (c > 0) {
            o.active[pos] = a;
            for (int off = 0; off < c; off += o.tile_t, ++tile)
                reinterpret_cast<int4*>(o.tiles)[tile] =
                    make_int4(a, starts[a] + off, min(o.tile_t, c - off), pos);
            ++pos;
        }
    }
    const int n_active = (int)(s_total >> 32);
    const int n_tiles = (int)(s_total & 0xffffffffll);
    for (int s = n_active + tid; s < n_adapters; s += nthr) o.active[s] = -1;
    for (int g = n_tiles + tid; g < max_tiles; g += nthr)
        reinterpret_cast<int4*>(o.tiles)[g] = make_int4(-1, 0, 0, -1);
    if (tid == 0) {
        o.counts[0] = starts[n_adapters];
        o.counts[1] = n_active;
        o.counts[2] = n_bad;
        o.counts[3] = n_tiles;
        o.counts[4] = 0;  // device status word
        o.counts[5] = o.counts[6] = o.counts[7] = 0;
    }
    __syncthreads();
}

__device__ __forceinline__ int bin_of(int id, int n_adapters)
{
    return (id >= 0 && id < n_adapters) ? id : n_adapters;
}

// Tiny batches (T <= 64, n_adapters <= 64, a decode step): one warp and no block
// barriers. Lane l holds tokens l and l + 32; match_any groups equal ids, so a
// token's rank among its id is the number of equal ids before it (the slot-0
// tokens of its id come first), and a scan over the <= 65 bins (3 per lane)
// gives starts, indptr, the active list and the tile rows.
constexpr int kWarpMaxT = 64;
constexpr int kWarpMaxAdapters = 64;

__device__ __forceinline__ int warp_excl_scan(int v, int* total)
{
    const int lane = threadIdx.x & 31;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
    }
    *total = __shfl_sync(0xffffffffu, incl, 31);
    return incl - v;
}

__global__ void __launch_bounds__(32, 1)
segments_warp_kernel(const int32_t* __restrict__ ids, int T, int n_adapters, int max_tiles, SegOut o)
{
    __shared__ int32_t hist[96];    // per bin (n_adapters + 1 <= 65), 3 per lane
    __shared__ int32_t cnt0[96];    // the same over slot-0 tokens only
    __shared__ int32_t starts[96];
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    const int lane = threadIdx.x;
    const int nb = n_adapters + 1;
    for (int b = lane; b < 96; b += 32) hist[b] = 0;
    __syncwarp();

    int bin[2], rank[2];
    bool in[2];
    int nbad = 0;
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
        const int t = lane + 32 * sl;
        in[sl] = t < T;
        const int id = in[sl] ? ids[t] : -1;
        bin[sl] = in[sl] ? bin_of(id, n_adapters) : -2 - lane;  // absent tokens match nobody
        if (in[sl]) {
            o.tok_adapter[t] = bin[sl] < n_adapters ? id : -1;
            if (bin[sl] == n_adapters && id != -1) ++nbad;
        }
    }
    nbad = __reduce_add_sync(0xffffffffu, (unsigned)nbad);
    const unsigned lt = (1u << lane) - 1u;
    // slot 0: one leader per distinct bin sets its count
    const unsigned p0 = __match_any_sync(0xffffffffu, bin[0]);
    rank[0] = __popc(p0 & lt);
    if (in[0] && lane == __ffs(p0) - 1) hist[bin[0]] = __popc(p0);
    __syncwarp();
    for (int b = lane; b < 96; b += 32) cnt0[b] = hist[b];
    __syncwarp();
    // slot 1: after every slot-0 token of the same bin
    const unsigned p1 = __match_any_sync(0xffffffffu, bin[1]);
    rank[1] = in[1] ? cnt0[bin[1]] + __popc(p1 & lt) : 0;
    if (in[1] && lane == __ffs(p1) - 1) hist[bin[1]] = cnt0[bin[1]] + __popc(p1);
    __syncwarp();

    // starts / indptr over bins 3*lane .. 3*lane+2
    int h[3], sum = 0;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int b = 3 * lane + i;
        h[i] = b < nb ? hist[b] : 0;
        sum += h[i];
    }
    int n_valid_all;
    int base = warp_excl_scan(sum, &n_valid_all);
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int b = 3 * lane + i;
        if (b < nb) {
            starts[b] = base;
            o.indptr[b] = base;
        }
        base += h[i];
    }
    // active adapters and their tiles: (#active << 16) | #tiles, scanned over bins
    int pk = 0;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int b = 3 * lane + i;
        if (b < n_adapters && h[i] > 0) pk += (1 << 16) + (h[i] + o.tile_t - 1) / o.tile_t;
    }
    int pk_total;
    const int pbase = warp_excl_scan(pk, &pk_total);
    int pos = pbase >> 16, tile = pbase & 0xffff;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int b = 3 * lane + i;
        if (b < n_adapters && h[i] > 0) {
            o.active[pos] = b;
            for (int off = 0; off < h[i]; off += o.tile_t, ++tile)
                reinterpret_cast<int4*>(o.tiles)[tile] = make_int4(b, starts[b] + off, min(o.tile_t, h[i] - off), pos);
            ++pos;
        }
    }
    const int n_active = pk_total >> 16, n_tiles = pk_total & 0xffff;
    for (int a = n_active + lane; a < n_adapters; a += 32) o.active[a] = -1;
    for (int g = n_tiles + lane; g < max_tiles; g += 32)
        reinterpret_cast<int4*>(o.tiles)[g] = make_int4(-1, 0, 0, -1);
    __syncwarp();  // starts[] complete
#pragma unroll
    for (int sl = 0; sl < 2; ++sl)
        if (in[sl]) o.perm[starts[bin[sl]] + rank[sl]] = lane + 32 * sl;
    if (lane == 0) {
        o.counts[0] = starts[n_adapters];
        o.counts[1] = n_active;
        o.counts[2] = nbad;
        o.counts[3] = n_tiles;
        o.counts[4] = 0;  // device status word
        o.counts[5] = o.counts[6] = o.counts[7] = 0;
    }
}

// Small batches: blockDim >= T, shared memory = (warps + 2) * nb ints.
__global__ void __launch_bounds__(kMaxThreads, 1)
segments_small_kernel(const int32_t* __restrict__ ids, int T, int n_adapters, int max_tiles, SegOut o)
{
    extern __shared__ int32_t smem[];
    __shared__ int s_bad;
    // PDL: whatever ran before may still be writing our outputs; wait, then
    // let the consumer of the segments launch early.
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    const int nb = n_adapters + 1;
    const int nw = blockDim.x >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t* cnt = smem;             // [nw][nb] per-warp counts, then offsets
    int32_t* hist = smem + nw * nb;  // [nb]
    int32_t* starts = hist + nb;     // [nb]
    for (int i = tid; i < nw * nb; i += blockDim.x) cnt[i] = 0;
    if (tid == 0) s_bad = 0;
    __syncthreads();

    const bool in = tid < T;
    int id = -1, bin = -2 - lane;
    if (in) {
        id = ids[tid];
        bin = bin_of(id, n_adapters);
        o.tok_adapter[tid] = bin < n_adapters ? id : -1;
    }
    const unsigned bad = __ballot_sync(0xffffffffu, in && bin == n_adapters && id != -1);
    if (lane == 0 && bad) atomicAdd(&s_bad, __popc(bad));
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (in && lane == __ffs(peers) - 1) cnt[warp * nb + bin] = __popc(peers);
    __syncthreads();
    // column scan: offset of each warp inside every bin, and the histogram
    for (int b = tid; b < nb; b += blockDim.x) {
        int run = 0;
        for (int w = 0; w < nw; ++w) {
            const int c = cnt[w * nb + b];
            cnt[w * nb + b] = run;
            run += c;
        }
        hist[b] = run;
    }
    __syncthreads();
    finish_tables(hist, starts, n_adapters, max_tiles, s_bad, o);
    if (in) o.perm[starts[bin] + cnt[warp * nb + bin] + rank] = tid;
}

// Large batches: 1024 threads, shared memory = 2 * nb ints.
__global__ void __launch_bounds__(kMaxThreads, 1)
segments_large_kernel(const int32_t* __restrict__ ids, int T, int n_adapters, int max_tiles, SegOut o)
{
    extern __shared__ int32_t smem[];
    __shared__ int s_bad;
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    const int nb = n_adapters + 1;
    int32_t* hist = smem;         // [nb]
    int32_t* cursor = smem + nb;  // [nb] starts, then running cursors
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    for (int i = tid; i < nb; i += blockDim.x) hist[i] = 0;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    int bad = 0;
    for (int t = tid; t < T; t += blockDim.x) {
        const int id = ids[t];
        const int bin = bin_of(id, n_adapters);
        if (bin == n_adapters && id != -1) ++bad;
        o.tok_adapter[t] = bin < n_adapters ? id : -1;
        atomicAdd(&hist[bin], 1);
    }
    if (bad) atomicAdd(&s_bad, bad);
    __syncthreads();
    finish_tables(hist, cursor, n_adapters, max_tiles, s_bad, o);

    for (int t0 = 0; t0 < T; t0 += blockDim.x) {
        const int t = t0 + tid;
        const bool in = t < T;
        const int bin = in ? bin_of(ids[t], n_adapters) : -2 - lane;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        for (int w = 0; w < nw; ++w) {
            if (warp == w) {
                int p = 0;
                if (in && lane == leader) {
                    p = cursor[bin];
                    cursor[bin] = p + __popc(peers);
                }
                p = __shfl_sync(0xffffffffu, p, leader);
                if (in) o.perm[p + rank] = t;
            }
            __syncthreads();
        }
    }
}

}  // namespace

int tile_tokens_for(int T, int n_adapters)
{
    return (T <= LORA_DECODE_MAX_TOKENS && T <= 2 * n_adapters) ? LORA_DECODE_TILE_TOKENS : LORA_TILE_TOKENS;
}

int max_tiles_for(int T, int n_adapters)
{
    const long long t = tile_tokens_for(T, n_adapters);
    const long long m = n_adapters < T ? n_adapters : T;
    return (int)(((long long)T + (t - 1) * m) / t);
}

cudaError_t launch_build_segments(const int32_t* ids, int T, int n_adapters,
                                  const lora_segments_t& seg, cudaStream_t stream)
{
    SegOut o{seg.perm, seg.indptr, seg.active, seg.tiles, seg.tok_adapter, seg.counts, tile_tokens_for(T, n_adapters)};
    const int nb = n_adapters + 1;
    const int mt = max_tiles_for(T, n_adapters);
    const int threads_small = T <= 64 ? 64 : (T + 31) / 32 * 32;
    const size_t smem_small = sizeof(int32_t) * (size_t)(threads_small / 32 + 2) * nb;
    const bool small = T <= kMaxThreads && smem_small <= 96 * 1024;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = stream;
    cfg.gridDim = dim3(1, 1, 1);
    cudaError_t e;
    if (T <= kWarpMaxT && n_adapters <= kWarpMaxAdapters) {
        cfg.blockDim = dim3(32, 1, 1);
        cfg.dynamicSmemBytes = 0;
        return cudaLaunchKernelEx(&cfg, segments_warp_kernel, ids, T, n_adapters, mt, o);
    }
    if (small) {
        cfg.blockDim = dim3(threads_small, 1, 1);
        cfg.dynamicSmemBytes = smem_small;
        e = cudaFuncSetAttribute(segments_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 96 * 1024);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, segments_small_kernel, ids, T, n_adapters, mt, o);
    }
    cfg.blockDim = dim3(kMaxThreads, 1, 1);
    cfg.dynamicSmemBytes = sizeof(int32_t) * 2 * (size_t)nb;
    e = cudaFuncSetAttribute(segments_large_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             2 * (LORA_MAX_ADAPTERS + 1) * (int)sizeof(int32_t));
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, segments_large_kernel, ids, T, n_adapters, mt, o);
}

}  // namespace lora
