// sgmv_warp.cu -- the fused shrink + expand of SGMV (Punica README, "How?":
// y += s_a (x.A_a).B_a, tokens grouped by adapter) for the small tiles of a
// general batch: runs of at most kWarpTile tokens of one adapter, which is
// what most adapters of a many-tenant batch hold.
//
// Such a tile moves a whole adapter (A_a and B_a) for very few FMAs, so the
// cost is in moving bytes and in per-chunk latency, not in math. Every warp is
// an independent pipeline: it claims a work item from a global counter, issues
// its own tensor-map copies into a private ring of 3 shared-memory stages,
// and computes each chunk as soon as it lands, with no barrier across warps.
//   Shrink part (a span of h_in): each chunk is a box of A_a rows (only the
//   adapter's live columns) and the tile's x rows; lane (pair p, group q)
//   accumulates columns 2p, 2p+1 of v over rows q, q + G, ... for every token,
//   so the only reduction is over the G row groups at the end of the part,
//   which then adds its partial v into the workspace (stores when one part
//   spans h_in).
//   Expand part (a span of h_out): each chunk is a box of B_a (the rank's rows)
//   and the tile's y rows; each lane owns column pairs and sums v[t][j] B[j][n]
//   over the rank, then writes y[t][n..n+1] (bf16, one rounding).
// Two launches, like the pages' shrink-then-expand: the shrink parts, then the
// expand parts as a programmatic dependent whose copies start at once and whose
// warps wait for the shrink launch to complete before reading v.
//
// Tiles with more tokens are left to the cluster kernel (sgmv.cu), launched
// first; the tokens of the two sets are disjoint, so the shrink launch runs
// alongside it and only waits for it to complete before leaving.
//
// Every wait is bounded (limit from lora_debug_set_wait_limit, 2 s by
// default); on expiry the warp records a status word in lora_segments_t.counts,
// its CTA stops claiming work, and the copies in flight are drained.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kWarpTile = kWarpSmallTile;  // largest tile (tokens) of this kernel
constexpr int kWWarps = 8;          // independent pipelines per CTA
constexpr int kWThreads = kWWarps * 32;
constexpr int kWStages = 3;
constexpr int kWStage = 8192;       // bytes of one ring stage
constexpr unsigned long long kDrainNs = 2000000000ull;

// Rows of A per chunk for box width 8 << i, and columns of B per chunk for
// 16 (i + 1) rows, so that the box and the tile's x or y rows fill one stage.
__host__ __device__ constexpr int a_rows(int i) { return i == 0 ? 256 : (i == 1 ? 160 : (i == 2 ? 96 : 48)); }
__host__ __device__ constexpr int b_cols(int i) { return i == 0 ? 160 : (i == 1 ? 96 : (i == 2 ? 72 : 48)); }

struct WarpMaps {
    CUtensorMap a[4];  // A {r_max, h_in, slices * adapters}, box {8 << i, a_rows(i), 1}
    CUtensorMap b[4];  // B {h_out, r_max, slices * adapters}, box {b_cols(i), min(16 (i + 1), r_max), 1}
};

struct WarpParams {
    const uint16_t* x;
    long long x_slice_stride;
    const int32_t* ranks;
    const float* scales;
    const int32_t* perm;
    const int4* tiles;
    int32_t* counts;
    uint16_t* y;
    float* vbuf;  // fp32 [n_slices][T][r_max]
    int* ctr;     // [phase]: next item
    int T, n_adapters, h_in, h_out, r_max, n_slices;
    int Pk, Pn, kp, np;
    int phase;
    unsigned long long timeout_ns;
    int inject_stall;
};

__device__ __forceinline__ float bflo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bfhi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Bounded wait of one warp on a phase (lane 0 polls; the others acquire).
__device__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status, int code,
                          unsigned long long limit)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        if (!ptx::mbar_try_wait(bar, parity)) {
            const unsigned long long t0 = ptx::globaltimer();
            for (unsigned n = 1;; ++n) {
                if (ptx::mbar_try_wait(bar, parity)) break;
                if ((n & 63) == 0) {
                    if (*abort_flag) {
                        ok = false;
                        break;
                    }
                    if (ptx::globaltimer() - t0 > limit) {
                        *abort_flag = 1;
                        atomicOr(status, code);
                        ok = false;
                        break;
                    }
                }
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && (threadIdx.x & 31) != 0) ptx::mbar_try_wait(bar, parity);
    return ok;
}

__global__ void __launch_bounds__(kWThreads, 1)
sgmv_warp_kernel(const __grid_constant__ WarpMaps mp, const WarpParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t s_full[kWWarps][kWStages];
    __shared__ uint64_t s_stall;
    __shared__ int s_abort;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* ring = smem + (size_t)warp * (kWStages * kWStage + kWarpTile * 64 * 4);
    float* vsm = reinterpret_cast<float*>(ring + kWStages * kWStage);  // [kWarpTile][64]
    uint64_t* full = s_full[warp];
    volatile int* abort_flag = &s_abort;
    int32_t* status = p.counts + kSegStatusSlot;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int w = 0; w < kWWarps; ++w)
            for (int s = 0; s < kWStages; ++s) ptx::mbar_init(&s_full[w][s], 1);
        ptx::mbar_init(&s_stall, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    // the shrink launch overlaps the cluster kernel before it (disjoint tokens); the
    // expand launch's copies start at once and its warps wait before reading v
    ptx::pdl_launch_dependents();
    if (lane == 0) {
        for (int i = 0; i < 4; ++i)
            if ((8 << i) <= p.r_max) ptx::tma_prefetch_desc(&mp.a[i]);
        for (int i = 0; i < 4 && 16 * i < p.r_max; ++i) ptx::tma_prefetch_desc(&mp.b[i]);
    }
    bool ok = true;
    if (p.inject_stall && blockIdx.x == 0 && warp == 0)
        ok = warp_wait(&s_stall, 0, abort_flag, status, 0x2000, p.timeout_ns);
    const bool shrink = p.phase == 0;
    const long long used = p.counts[3];
    const int P = shrink ? p.Pk : p.Pn;
    const long long n_items = used * p.n_slices * P;
    bool v_ready = shrink;
    int st = 0;
    uint32_t ph = 0;
    long long issued = 0, consumed = 0;

    while (ok) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // the warp leaves as one
        long long item = 0;
        if (lane == 0) item = (long long)atomicAdd(p.ctr + p.phase, 1);
        item = __shfl_sync(0xffffffffu, item, 0);
        if (item >= n_items) break;
        const long long per_slice = used * P;
        const int slice = (int)(item / per_slice);
        long long rem = item - (long long)slice * per_slice;
        const int g = (int)(rem / P);
        const int part = (int)(rem - (long long)g * P);
        const int4 tl = p.tiles[g];
        const int nt = tl.z;
        if (nt <= 0 || nt > kWarpTile) continue;  // the cluster kernel's tile
        const int a = tl.x;
        int r = p.ranks ? p.ranks[a] : p.r_max;
        r = max(1, min(r, p.r_max));
        const float scale = p.scales ? p.scales[a] : 1.f;
        const int tok = lane < nt ? p.perm[tl.y + lane] : 0;
        int tk[kWarpTile];  // the tile's token ids in every lane (uniform shuffles, outside any divergence)
#pragma unroll
        for (int t = 0; t < kWarpTile; ++t) tk[t] = __shfl_sync(0xffffffffu, tok, t);
        const int r8 = (r + 7) & ~7;
        const int ai = r8 <= 8 ? 0 : 32 - __clz((r8 >> 3) - 1);  // A box width 8 << ai >= r
        const int rA = 8 << ai;
        const int bi = ((r + 15) >> 4) - 1;                       // B box rows 16 (bi + 1)
        const int rB = min(16 * (bi + 1), p.r_max);
        const int span = shrink ? p.kp : p.np;
        const int lim = shrink ? p.h_in : p.h_out;
        const int c_begin = part * span, c_end = min(lim, c_begin + span);
        const int wch = shrink ? a_rows(ai) : b_cols(bi);  // rows (shrink) or columns per chunk
        const int n_chunks = (c_end - c_begin + wch - 1) / wch;
        const int sa = slice * p.n_adapters + a;
        const uint16_t* xg = p.x + (size_t)slice * p.x_slice_stride;
        uint16_t* yg = p.y + (size_t)slice * p.T * p.h_out;
        // box bytes and the tile's row bytes of a chunk; the rows follow the box
        const int box_bytes = shrink ? wch * rA * 2 : rB * wch * 2;
        auto issue = [&](int c, int s) {
            const int c0 = c_begin + c * wch, cw = min(wch, c_end - c0);
            uint8_t* base = ring + s * kWStage;
            const uint32_t rows_u = ptx::smem_u32(base + box_bytes);
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)(box_bytes + nt * cw * 2));
                if (shrink)
                    ptx::tma_load_3d(ptx::smem_u32(base), &mp.a[ai], &full[s], 0, c0, sa);
                else
                    ptx::tma_load_3d(ptx::smem_u32(base), &mp.b[bi], &full[s], c0, 0, sa);
            }
            __syncwarp();
            if (lane < nt) {  // row t of x (or y) for the chunk's columns, one bulk copy per lane
                const uint16_t* src = shrink ? xg + (size_t)tok * p.h_in + c0 : yg + (size_t)tok * p.h_out + c0;
                ptx::bulk_g2s(rows_u + (uint32_t)(lane * wch * 2), src, (uint32_t)(cw * 2), &full[s]);
            }
        };
        // prologue: up to kWStages chunks in flight
        const int pre = min(n_chunks, kWStages);
        for (int c = 0; c < pre; ++c) {
            issue(c, (st + c) % kWStages);
            ++issued;
        }
        // expand: v of the tile's tokens (after the shrink launch has completed)
        if (!shrink) {
            if (!v_ready) {
                ptx::pdl_wait();
                v_ready = true;
            }
            const float* vrow = p.vbuf + (size_t)slice * p.T * p.r_max;
#pragma unroll
            for (int t = 0; t < kWarpTile; ++t)
                if (t < nt)
                    for (int j = lane; j < 64; j += 32)
                        vsm[t * 64 + j] = j < r ? __ldcg(vrow + (size_t)tk[t] * p.r_max + j) : 0.f;
            __syncwarp();
        }
        // shrink accumulators: lane (pair pp, group q); G groups of rows
        const int npair = rA >> 1;
        const int G = 32 / npair;
        const int pp = lane % npair, q = lane / npair;
        float acc[kWarpTile][2];
#pragma unroll
        for (int t = 0; t < kWarpTile; ++t) acc[t][0] = acc[t][1] = 0.f;
        for (int c = 0; c < n_chunks; ++c) {
            if (!warp_wait(&full[st], ph, abort_flag, status, 0x800, p.timeout_ns)) {
                ok = false;
                break;
            }
            ++consumed;
            const int c0 = c_begin + c * wch, cw = min(wch, c_end - c0);
            const uint8_t* base = ring + st * kWStage;
            const uint8_t* rows = base + box_bytes;
            if (shrink) {
                // A row k: rA bf16 at base + k * rA * 2; x row t: wch bf16 at rows + t * wch * 2
                for (int k = q; k < cw; k += G) {
                    const uint32_t a2 = *reinterpret_cast<const uint32_t*>(base + k * rA * 2 + pp * 4);
                    const float a0 = bflo(a2), a1 = bfhi(a2);
#pragma unroll
                    for (int t = 0; t < kWarpTile; ++t)
                        if (t < nt) {
                            const float xv =
                                __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(rows + (t * wch + k) * 2) << 16);
                            acc[t][0] = fmaf(xv, a0, acc[t][0]);
                            acc[t][1] = fmaf(xv, a1, acc[t][1]);
                        }
                }
            } else {
                // B row j: wch bf16 at base + j * wch * 2; y row t at rows + t * wch * 2
                for (int n = lane * 2; n < cw; n += 64) {
                    float s0[kWarpTile], s1[kWarpTile];
#pragma unroll
                    for (int t = 0; t < kWarpTile; ++t) s0[t] = s1[t] = 0.f;
                    for (int j = 0; j < r; ++j) {
                        const uint32_t b2 = *reinterpret_cast<const uint32_t*>(base + (j * wch + n) * 2);
                        const float b0 = bflo(b2), b1 = bfhi(b2);
#pragma unroll
                        for (int t = 0; t < kWarpTile; ++t)
                            if (t < nt) {
                                const float vv = vsm[t * 64 + j];
                                s0[t] = fmaf(vv, b0, s0[t]);
                                s1[t] = fmaf(vv, b1, s1[t]);
                            }
                    }
#pragma unroll
                    for (int t = 0; t < kWarpTile; ++t)
                        if (t < nt) {
                            const uint32_t yw = *reinterpret_cast<const uint32_t*>(rows + (t * wch + n) * 2);
                            *reinterpret_cast<__nv_bfloat162*>(yg + (size_t)tk[t] * p.h_out + c0 + n) =
                                __floats2bfloat162_rn(bflo(yw) + scale * s0[t], bfhi(yw) + scale * s1[t]);
                        }
                }
            }
            // the stage's reads are done: refill it with the chunk kWStages ahead
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (c + kWStages < n_chunks) {
                issue(c + kWStages, st);
                ++issued;
            }
            if (++st == kWStages) {
                st = 0;
                ph ^= 1;
            }
        }
        if (!ok) break;
        if (shrink) {
            // sum the row groups (lanes with the same pair), then lanes of group 0 add the
            // part's v for columns 2 pp, 2 pp + 1 (past the rank: the pool's padding, skipped)
            for (int off = npair; off < 32; off <<= 1)
#pragma unroll
                for (int t = 0; t < kWarpTile; ++t)
                    if (t < nt) {
                        acc[t][0] += __shfl_xor_sync(0xffffffffu, acc[t][0], off);
                        acc[t][1] += __shfl_xor_sync(0xffffffffu, acc[t][1], off);
                    }
            float* vrow = p.vbuf + (size_t)slice * p.T * p.r_max;
#pragma unroll
            for (int t = 0; t < kWarpTile; ++t) {
                if (t < nt && q == 0 && 2 * pp < r) {
                    float* dst = vrow + (size_t)tk[t] * p.r_max + 2 * pp;
                    if (p.Pk > 1) {
                        if (2 * pp + 1 < r) atomicAdd(reinterpret_cast<float2*>(dst), make_float2(acc[t][0], acc[t][1]));
                        else atomicAdd(dst, acc[t][0]);
                    } else {
                        if (2 * pp + 1 < r) *reinterpret_cast<float2*>(dst) = make_float2(acc[t][0], acc[t][1]);
                        else *dst = acc[t][0];
                    }
                }
            }
        }
    }
    // copies still in flight (a warp that stopped early): let them land
    if (lane == 0) {
        const unsigned long long t0 = ptx::globaltimer();
        for (long long it = consumed; it < issued; ++it) {
            const int s = (int)(it % kWStages);
            const uint32_t par = (uint32_t)((it / kWStages) & 1);
            while (!ptx::mbar_try_wait(&full[s], par) && ptx::globaltimer() - t0 < kDrainNs) {
            }
        }
    }
    __syncwarp();
    // the shrink launch leaves only once the kernel before it (the cluster kernel) is done,
    // so that the expand launch's completion implies every tile's completion
    if (shrink && threadIdx.x == 0) ptx::pdl_wait();
}

}  // namespace

// Parts per tile row: about three items per warp of the grid, counted on an
// estimate of the small tile rows (one per four tokens at most).
void warp_parts(int T, const lora_pool_t& pool, int* kp, int* np, int* Pk, int* Pn)
{
    const long long warps = (long long)device_sm_count() * kWWarps;
    const long long rows_est =
        (long long)std::max(1, std::min(max_tiles_for(T, pool.n_adapters), (T + 3) / 4)) * pool.n_slices;
    long long P = (3 * warps + rows_est - 1) / rows_est;
    P = P < 1 ? 1 : (P > 32 ? 32 : P);
    auto span = [&](int h) { return (int)(((h + P - 1) / P + 63) / 64 * 64); };
    *kp = span(pool.h_in);
    *np = span(pool.h_out);
    *Pk = (pool.h_in + *kp - 1) / *kp;
    *Pn = (pool.h_out + *np - 1) / *np;
}

// The item counters start at zero; so does v when several parts add into it. Issued
// before the cluster kernel, so that the warp kernel's launches can overlap that one.
cudaError_t sgmv_warp_zero(const lora_pool_t& pool, const lora_segments_t& seg, void* ws, cudaStream_t stream)
{
    if (seg.T == 0) return cudaSuccess;
    int kp, np, Pk, Pn;
    warp_parts(seg.T, pool, &kp, &np, &Pk, &Pn);
    const size_t v_bytes = (size_t)pool.n_slices * seg.T * pool.r_max * 4;
    return cudaMemsetAsync(ws, 0, Pk > 1 ? 256 + v_bytes : 256, stream);
}

size_t sgmv_warp_workspace_bytes(int T, const lora_pool_t& pool)
{
    const size_t v = (size_t)pool.n_slices * T * pool.r_max * 4;
    return 256 + (v + 255) / 256 * 256;  // the two item counters | v
}

cudaError_t launch_sgmv_warp(const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                             const lora_segments_t& seg, void* y, void* ws, cudaStream_t stream)
{
    if (seg.T == 0) return cudaSuccess;
    WarpParams p = {};
    p.x = static_cast<const uint16_t*>(x);
    p.x_slice_stride = x_slice_stride;
    p.ranks = pool.ranks;
    p.scales = pool.scales;
    p.perm = seg.perm;
    p.tiles = reinterpret_cast<const int4*>(seg.tiles);
    p.counts = seg.counts;
    p.y = static_cast<uint16_t*>(y);
    p.T = seg.T;
    p.n_adapters = pool.n_adapters;
    p.h_in = pool.h_in;
    p.h_out = pool.h_out;
    p.r_max = pool.r_max;
    p.n_slices = pool.n_slices;
    p.timeout_ns = debug_wait_limit_ns();
    p.inject_stall = debug_inject_stall();
    const int sms = device_sm_count();
    warp_parts(seg.T, pool, &p.kp, &p.np, &p.Pk, &p.Pn);
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.ctr = reinterpret_cast<int*>(w);
    p.vbuf = reinterpret_cast<float*>(w + 256);
    cudaError_t e = cudaSuccess;

    WarpMaps mp;
    memset(&mp, 0, sizeof(mp));
    {
        const uint64_t dims[3] = {(uint64_t)pool.r_max, (uint64_t)pool.h_in,
                                  (uint64_t)pool.n_slices * (uint64_t)pool.n_adapters};
        const uint64_t strides[2] = {(uint64_t)pool.r_max * 2, (uint64_t)pool.h_in * pool.r_max * 2};
        for (int i = 0; i < 4 && (8 << i) <= pool.r_max; ++i) {
            const uint32_t box[3] = {(uint32_t)(8 << i), (uint32_t)a_rows(i), 1};
            if (!encode_tmap_3d(&mp.a[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pool.A, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
                return cudaErrorInvalidValue;
        }
    }
    {
        const uint64_t dims[3] = {(uint64_t)pool.h_out, (uint64_t)pool.r_max,
                                  (uint64_t)pool.n_slices * (uint64_t)pool.n_adapters};
        const uint64_t strides[2] = {(uint64_t)pool.h_out * 2, (uint64_t)pool.r_max * pool.h_out * 2};
        for (int i = 0; i < 4 && 16 * i < pool.r_max; ++i) {
            const uint32_t rows = (uint32_t)std::min(16 * (i + 1), pool.r_max);
            const uint32_t box[3] = {(uint32_t)b_cols(i), rows, 1};
            if (!encode_tmap_3d(&mp.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pool.B, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
                return cudaErrorInvalidValue;
        }
    }
    const size_t smem = (size_t)kWWarps * (kWStages * kWStage + kWarpTile * 64 * 4);
    e = cudaFuncSetAttribute(sgmv_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    for (int phase = 0; phase < 2; ++phase) {
        p.phase = phase;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)sms, 1, 1);
        cfg.blockDim = dim3(kWThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, sgmv_warp_kernel, mp, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lora
