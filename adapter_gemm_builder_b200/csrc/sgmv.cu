// sgmv.cu -- Segmented Gather Matrix-Vector multiplication for multi-tenant
// LoRA (Punica README, "How?": the added term (x_i.A_i.B_i) for a batch whose
// tokens map to different adapters, computed for all adapters in one kernel).
//
// One kernel, three modes:
//   SHRINK  v = x.A_a            (fp32, written to global)
//   EXPAND  y += s_a * v.B_a     (v read from global, y bf16 read-modify-write)
//   APPLY   y += s_a * (x.A_a).B_a, with v kept on chip
//
// Work decomposition. The segment builder cuts every adapter's run of tokens
// into tiles of up to LORA_TILE_TOKENS tokens. A tile is handled by a
// thread-block cluster of C CTAs (C <= 8): in the shrink, CTA c owns the
// c-th slice of h_in (split-K) and produces a partial v for the tile's tokens;
// the partials are reduced through distributed shared memory (reduce-scatter
// then all-gather), so no global workspace and no second pass is needed; in
// the expand, CTA c owns the c-th slice of h_out. gridDim.y is the slice
// (projection) index, so q/k/v/o of one layer run in one launch.
//
// Memory path. Every operand streams global -> shared with 16-byte cp.async
// (zero-filling the bytes past an adapter's rank or past the end of a row,
// so the padding of the pool is never read) through a 4-stage ring of 16 KB
// stages. The stage shape adapts to the tile: a k-block holds BK rows of A_a
// (r8 columns) plus BK columns of the tile's x rows, with BK chosen so the
// stage is full whatever the rank and token count; decode tiles with one
// token therefore stream ~15 KB of A per stage. Shared layouts are chosen
// for conflict-free ldmatrix: A and B in 8-column blocks (each 8x8 matrix is
// 128 contiguous bytes), x and y rows with a 16-byte-chunk XOR swizzle.
//
// Math. bf16 tensor-core MMA (m16n8k16, fp32 accumulate) for both products.
// The expand's left operand v is fp32; it is split as v = hi + lo with hi, lo
// in bf16 and both halves are multiplied, which keeps ~16 mantissa bits of v
// (bf16 x bf16 products are exact in fp32).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 4;
constexpr int kStageBytes = 16384;
constexpr int kTT = LORA_TILE_TOKENS;  // 64
constexpr int kMaxCluster = 8;

struct SgmvParams {
    const uint16_t* x;
    long long x_slice_stride;
    const uint16_t* A;
    const uint16_t* B;
    const int32_t* ranks;
    const float* scales;
    const int32_t* perm;
    const int32_t* indptr;
    const int32_t* active;
    const int32_t* tile_ptr;
    const int32_t* counts;
    float* v;
    uint16_t* y;
    int T, n_adapters, h_in, h_out, r_max;
    int csize;     // CTAs per tile
    int kc, nc;    // h_in / h_out slice per CTA (multiples of 8)
    int rp;        // row pitch (floats) of the partial / reduced v buffers = round_up(r_max, 16)
    int vpitch;    // row pitch (bf16) of the hi/lo v operand = rp + 8
};

__device__ __forceinline__ int round_up(int a, int b) { return (a + b - 1) / b * b; }

// XOR-swizzled byte offset of 16-byte chunk `ch` of row `row` in a row-major
// tile of `row_bytes` per row (row_bytes a multiple of 128).
__device__ __forceinline__ uint32_t swz(int row, int ch, int row_bytes)
{
    return (uint32_t)(row * row_bytes + ((ch ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads)
sgmv_kernel(const SgmvParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_tok[kTT];
    __shared__ __align__(16) uint32_t s_zero[4];

    // Let a programmatic dependent (the FP8 GEMM) launch as early as possible.
    ptx::pdl_launch_dependents();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = p.csize;
    const int rank = (MODE == SGMV_EXPAND) ? (int)(blockIdx.x % C) : (int)ptx::cluster_ctarank();
    const int g = blockIdx.x / C;  // tile index
    const int slice = blockIdx.y;

    const int n_tiles = p.counts[3];
    if (g >= n_tiles) return;  // the whole cluster leaves together (same g)
    const int n_active = p.counts[1];

    // tile -> active segment (largest s with tile_ptr[s] <= g)
    int lo = 0, hi = n_active - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (p.tile_ptr[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int seg = lo;
    const int a = p.active[seg];
    const int seg_begin = p.indptr[a], seg_len = p.indptr[a + 1] - seg_begin;
    const int tok0 = seg_begin + (g - p.tile_ptr[seg]) * kTT;
    const int nt = min(kTT, seg_begin + seg_len - tok0);  // tokens in this tile, 1..64
    int r = p.ranks ? p.ranks[a] : p.r_max;
    r = max(0, min(r, p.r_max));
    const float scale = p.scales ? p.scales[a] : 1.0f;
    const int r8 = round_up(max(r, 1), 8), r16 = round_up(max(r, 1), 16);
    const int Mt = (nt + 15) >> 4;

    if (tid < kTT) s_tok[tid] = tid < nt ? p.perm[tok0 + tid] : 0;
    if (tid < 4) s_zero[tid] = 0u;

    uint8_t* ring = smem;
    // [sP partial v | hi/lo operand (aliases sP)] then [sR reduced v]
    float* sP = reinterpret_cast<float*>(smem + kStages * kStageBytes);  // [kTT][rp]
    uint16_t* sVh = reinterpret_cast<uint16_t*>(sP);                     // [kTT][vpitch]
    uint16_t* sVl = sVh + kTT * p.vpitch;                                // [kTT][vpitch]
    const int region0 = max(kTT * p.rp * 4, 2 * kTT * p.vpitch * 2);
    float* sR = reinterpret_cast<float*>(smem + kStages * kStageBytes + region0);  // [kTT][rp]
    const uint32_t ring_u = ptx::smem_u32(ring);
    const uint32_t zero_u = ptx::smem_u32(s_zero);

    // ---- shrink geometry: this CTA's slice of h_in
    const int k_begin = min(p.h_in, rank * p.kc);
    const int k_end = min(p.h_in, k_begin + p.kc);
    const int BK = ((kStageBytes / (2 * (r8 + nt))) / 64) * 64;  // >= 64
    const int nK = (MODE == SGMV_EXPAND) ? 0 : (k_end - k_begin + BK - 1) / BK;
    // ---- expand geometry: this CTA's slice of h_out
    const int n_begin = min(p.h_out, rank * p.nc);
    const int n_end = min(p.h_out, n_begin + p.nc);
    const int BN = ((kStageBytes / (2 * (r16 + nt))) / 64) * 64;  // >= 64
    const int nN = (MODE == SGMV_SHRINK) ? 0 : (n_end - n_begin + BN - 1) / BN;
    const int nItems = nK + nN;

    const size_t sa = (size_t)slice * p.n_adapters + a;
    const uint16_t* Ag = p.A + sa * (size_t)p.h_in * p.r_max;
    const uint16_t* Bg = p.B + sa * (size_t)p.r_max * p.h_out;
    const uint16_t* xg = p.x ? p.x + (size_t)slice * p.x_slice_stride : nullptr;
    uint16_t* yg = p.y ? p.y + (size_t)slice * p.T * p.h_out : nullptr;
    __syncthreads();

    // Issue the loads of work item `it` into ring stage `st`.
    auto load_item = [&](int it, int st) {
        const uint32_t base = ring_u + st * kStageBytes;
        if (it < nK) {
            const int k0 = k_begin + it * BK;
            const int kb = min(BK, k_end - k0);
            const int ncb = r8 >> 3;
            // A rows k0..k0+BK, column blocks of 8: smem [cb][BK][8]
            for (int i = tid; i < BK * ncb; i += kThreads) {
                const int kk = i / ncb, cb = i - kk * ncb;
                const int valid = (kk < kb) ? max(0, min(8, r - cb * 8)) : 0;
                const uint16_t* src = valid ? Ag + (size_t)(k0 + kk) * p.r_max + cb * 8 : Ag;
                ptx::cp_async16(base + (uint32_t)((cb * BK + kk) << 4), src, valid * 2);
            }
            // x rows of the tile: smem [nt][BK], swizzled
            const uint32_t xb = base + (uint32_t)(r8 * BK * 2);
            const int nch = BK >> 3;
            for (int i = tid; i < nt * nch; i += kThreads) {
                const int row = i / nch, ch = i - row * nch;
                const bool ok = ch * 8 < kb;
                const uint16_t* src =
                    ok ? xg + (size_t)s_tok[row] * p.h_in + k0 + ch * 8 : xg;
                ptx::cp_async16(xb + swz(row, ch, BK * 2), src, ok ? 16 : 0);
            }
        } else {
            const int n0 = n_begin + (it - nK) * BN;
            const int nb = min(BN, n_end - n0);
            const int ncb = BN >> 3;
            // B rows 0..r16, column blocks of 8: smem [cb][r16][8]
            for (int i = tid; i < r16 * ncb; i += kThreads) {
                const int j = i / ncb, cb = i - j * ncb;
                const bool ok = j < r && cb * 8 < nb;
                const uint16_t* src = ok ? Bg + (size_t)j * p.h_out + n0 + cb * 8 : Bg;
                ptx::cp_async16(base + (uint32_t)((cb * r16 + j) << 4), src, ok ? 16 : 0);
            }
            // y rows of the tile: smem [nt][BN], swizzled
            const uint32_t yb = base + (uint32_t)(r16 * BN * 2);
            for (int i = tid; i < nt * ncb; i += kThreads) {
                const int row = i / ncb, ch = i - row * ncb;
                const bool ok = ch * 8 < nb;
                const uint16_t* src =
                    ok ? yg + (size_t)s_tok[row] * p.h_out + n0 + ch * 8 : yg;
                ptx::cp_async16(yb + swz(row, ch, BN * 2), src, ok ? 16 : 0);
            }
        }
    };

    // Shrink accumulators: warp w owns output tiles [w*tpw, (w+1)*tpw) of the
    // (Mt x r8/8) grid of 16x8 tiles, row-major.
    const int nNT = r8 >> 3;
    const int tiles_s = Mt * nNT;
    const int tpw_s = (tiles_s + kWarps - 1) / kWarps;  // <= 4
    float acc[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[q][e] = 0.f;


    // Partial v of this CTA -> sP, then the cluster-wide reduction of v
    // (reduce-scatter by rows, then, for APPLY, all-gather as the bf16 hi/lo
    // operand of the expand). Called once by every CTA of a shrinking mode.
    auto finish_shrink = [&]() {
        {
            const int gq = lane >> 2, tq = lane & 3;
            const int q0 = warp * tpw_s;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = q0 + q;
                if (q < tpw_s && t < tiles_s) {
                    const int mt = t / nNT, ntl = t - mt * nNT;
                    const int row = mt * 16 + gq, col = ntl * 8 + tq * 2;
                    if (row < nt)
                        *reinterpret_cast<float2*>(&sP[row * p.rp + col]) =
                            make_float2(acc[q][0], acc[q][1]);
                    if (row + 8 < nt)
                        *reinterpret_cast<float2*>(&sP[(row + 8) * p.rp + col]) =
                            make_float2(acc[q][2], acc[q][3]);
                }
            }
        }
        ptx::cluster_sync();  // every CTA's partial is in its sP
        const uint32_t sP_u = ptx::smem_u32(sP);
        const uint32_t sR_u = ptx::smem_u32(sR);
        const int rows_mine = (nt > rank) ? (nt - rank + C - 1) / C : 0;
        const int cols = (MODE == SGMV_SHRINK) ? p.r_max : r8;
        for (int i = tid; i < rows_mine * cols; i += kThreads) {
            const int row = rank + (i / cols) * C, j = i % cols;
            float sum = 0.f;
            if (j < r8) {
                for (int c = 0; c < C; ++c)
                    sum += ptx::ld_dsmem_f32(ptx::mapa(sP_u + (uint32_t)((row * p.rp + j) * 4), c));
            }
            if (MODE == SGMV_SHRINK)
                p.v[((size_t)slice * p.T + s_tok[row]) * p.r_max + j] = (j < r) ? sum : 0.f;
            else
                sR[row * p.rp + j] = sum;
        }
        ptx::cluster_sync();  // reductions done; nobody reads sP any more
        if (MODE == SGMV_APPLY) {
            for (int i = tid; i < nt * r16; i += kThreads) {
                const int row = i / r16, j = i - row * r16;
                const float val =
                    j < r ? ptx::ld_dsmem_f32(
                                ptx::mapa(sR_u + (uint32_t)((row * p.rp + j) * 4), row % C))
                          : 0.f;
                const __nv_bfloat16 h = __float2bfloat16_rn(val);
                const __nv_bfloat16 l = __float2bfloat16_rn(val - __bfloat162float(h));
                sVh[row * p.vpitch + j] = *reinterpret_cast<const uint16_t*>(&h);
                sVl[row * p.vpitch + j] = *reinterpret_cast<const uint16_t*>(&l);
            }
            ptx::cluster_arrive();  // matched by the wait before exit
        }
    };

    // ---- prologue
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
        if (i < nItems) load_item(i, i);
        ptx::cp_async_commit();
    }

    if (MODE == SGMV_EXPAND) {
        // v (fp32, global) -> hi/lo bf16 operand
        for (int i = tid; i < nt * r16; i += kThreads) {
            const int row = i / r16, j = i - row * r16;
            const float val =
                j < r ? p.v[((size_t)slice * p.T + s_tok[row]) * p.r_max + j] : 0.f;
            const __nv_bfloat16 h = __float2bfloat16_rn(val);
            const __nv_bfloat16 l = __float2bfloat16_rn(val - __bfloat162float(h));
            sVh[row * p.vpitch + j] = *reinterpret_cast<const uint16_t*>(&h);
            sVl[row * p.vpitch + j] = *reinterpret_cast<const uint16_t*>(&l);
        }
    }

    if (MODE != SGMV_EXPAND && nK == 0) finish_shrink();

    for (int it = 0; it < nItems; ++it) {
        ptx::cp_async_wait<kStages - 2>();
        __syncthreads();
        {
            const int nx = it + kStages - 1;
            if (nx < nItems) load_item(nx, nx % kStages);
            ptx::cp_async_commit();
        }
        const int st = it % kStages;
        const uint32_t base = ring_u + st * kStageBytes;

        if (it < nK) {
            // ------------------------------------------------ shrink k-block
            const int k0 = k_begin + it * BK;
            const int kb = min(BK, k_end - k0);
            const uint32_t xb = base + (uint32_t)(r8 * BK * 2);
            const int ksteps = (kb + 15) >> 4;
            const int q0 = warp * tpw_s;
            for (int ks = 0; ks < ksteps; ++ks) {
                uint32_t af[4];
                int cur_mt = -1;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int t = q0 + q;
                    if (q < tpw_s && t < tiles_s) {
                        const int mt = t / nNT, ntl = t - mt * nNT;
                        if (mt != cur_mt) {
                            const int row = mt * 16 + (lane & 15);
                            const int ch = ks * 2 + (lane >> 4);
                            const uint32_t addr = row < nt ? xb + swz(row, ch, BK * 2) : zero_u;
                            ptx::ldsm_x4(addr, af[0], af[1], af[2], af[3]);
                            cur_mt = mt;
                        }
                        uint32_t b0, b1;
                        ptx::ldsm_x2_t(base + (uint32_t)((ntl * BK + ks * 16 + (lane & 15)) << 4),
                                       b0, b1);
                        ptx::mma_bf16_16816(acc[q], af, b0, b1);
                    }
                }
            }
        } else {
            // ------------------------------------------------ expand n-block
            const int n0 = n_begin + (it - nK) * BN;
            const int nb = min(BN, n_end - n0);
            const uint32_t yb = base + (uint32_t)(r16 * BN * 2);
            const int nNTe = BN >> 3;
            const int tiles_e = Mt * nNTe;
            const int tpw_e = (tiles_e + kWarps - 1) / kWarps;
            const int ksteps = r16 >> 4;
            const int gq = lane >> 2, tq = lane & 3;
            const uint32_t vh_u = ptx::smem_u32(sVh), vl_u = ptx::smem_u32(sVl);
            for (int q = 0; q < tpw_e; ++q) {
                const int t = warp * tpw_e + q;
                if (t >= tiles_e) break;
                const int mt = t / nNTe, ntl = t - mt * nNTe;
                if (ntl * 8 >= nb) continue;
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                for (int ks = 0; ks < ksteps; ++ks) {
                    const int row = mt * 16 + (lane & 15);
                    const uint32_t off = (uint32_t)((row * p.vpitch + ks * 16 + (lane >> 4) * 8) * 2);
                    uint32_t ah[4], al[4];
                    ptx::ldsm_x4(row < nt ? vh_u + off : zero_u, ah[0], ah[1], ah[2], ah[3]);
                    ptx::ldsm_x4(row < nt ? vl_u + off : zero_u, al[0], al[1], al[2], al[3]);
                    uint32_t b0, b1;
                    ptx::ldsm_x2_t(base + (uint32_t)((ntl * r16 + ks * 16 + (lane & 15)) << 4), b0,
                                   b1);
                    ptx::mma_bf16_16816(c, ah, b0, b1);
                    ptx::mma_bf16_16816(c, al, b0, b1);
                }
                // y(smem) = bf16(fp32(y) + s * c)
                const int col = ntl * 8 + tq * 2;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = mt * 16 + gq + h * 8;
                    if (row < nt) {
                        uint32_t* py = reinterpret_cast<uint32_t*>(
                            smem + (yb - ring_u) + swz(row, col >> 3, BN * 2) + (col & 7) * 2);
                        __nv_bfloat162 yv = *reinterpret_cast<__nv_bfloat162*>(py);
                        const float y0 = __bfloat162float(yv.x) + scale * c[h * 2 + 0];
                        const float y1 = __bfloat162float(yv.y) + scale * c[h * 2 + 1];
                        *py = pack_bf16x2(y0, y1);
                    }
                }
            }
            __syncthreads();
            // store the updated y rows (16 B per thread, coalesced per row)
            const int ncb = BN >> 3;
            for (int i = tid; i < nt * ncb; i += kThreads) {
                const int row = i / ncb, ch = i - row * ncb;
                if (ch * 8 < nb) {
                    const uint4 val =
                        *reinterpret_cast<const uint4*>(smem + (yb - ring_u) + swz(row, ch, BN * 2));
                    *reinterpret_cast<uint4*>(yg + (size_t)s_tok[row] * p.h_out + n0 + ch * 8) = val;
                }
            }
        }

        if (it == nK - 1 && MODE != SGMV_EXPAND) finish_shrink();
    }
    ptx::cp_async_wait<0>();
    if (MODE == SGMV_APPLY) ptx::cluster_wait();  // peers may read this CTA's sR until here
}

}  // namespace

cudaError_t launch_sgmv(int mode, const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                        const lora_segments_t& seg, float* v, void* y, cudaStream_t stream,
                        bool pdl_trigger)
{
    (void)pdl_trigger;
    SgmvParams p;
    p.x = static_cast<const uint16_t*>(x);
    p.x_slice_stride = x_slice_stride;
    p.A = static_cast<const uint16_t*>(pool.A);
    p.B = static_cast<const uint16_t*>(pool.B);
    p.ranks = pool.ranks;
    p.scales = pool.scales;
    p.perm = seg.perm;
    p.indptr = seg.indptr;
    p.active = seg.active;
    p.tile_ptr = seg.tile_ptr;
    p.counts = seg.counts;
    p.v = v;
    p.y = static_cast<uint16_t*>(y);
    p.T = seg.T;
    p.n_adapters = pool.n_adapters;
    p.h_in = pool.h_in;
    p.h_out = pool.h_out;
    p.r_max = pool.r_max;
    if (seg.T == 0) return cudaSuccess;

    // CTAs per tile: enough h_in per CTA to amortise the tile set-up
    int C = (pool.h_in + 255) / 256;
    C = C < 1 ? 1 : (C > kMaxCluster ? kMaxCluster : C);
    p.csize = C;
    p.kc = ((pool.h_in + C - 1) / C + 7) / 8 * 8;
    p.nc = ((pool.h_out + C - 1) / C + 7) / 8 * 8;
    p.rp = (pool.r_max + 15) / 16 * 16;
    p.vpitch = p.rp + 8;

    const int max_tiles = (pool.n_adapters < seg.T ? pool.n_adapters : seg.T) +
                          (seg.T + LORA_TILE_TOKENS - 1) / LORA_TILE_TOKENS;
    const size_t v_bytes = (size_t)kTT * p.rp * 4;                 // sP / sR
    const size_t vhl_bytes = (size_t)2 * kTT * p.vpitch * 2;       // hi + lo
    const size_t smem = kStages * kStageBytes + (v_bytes > vhl_bytes ? v_bytes : vhl_bytes) + v_bytes;
    // (layout: ring | sP or hi/lo v | sR; must match the kernel)

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(max_tiles * C), (unsigned)pool.n_slices, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    int nattr = 0;
    if (mode != SGMV_EXPAND) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        nattr = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = nattr;

    cudaError_t e;
    switch (mode) {
    case SGMV_SHRINK:
        e = cudaFuncSetAttribute(sgmv_kernel<SGMV_SHRINK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, sgmv_kernel<SGMV_SHRINK>, p);
    case SGMV_EXPAND:
        e = cudaFuncSetAttribute(sgmv_kernel<SGMV_EXPAND>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, sgmv_kernel<SGMV_EXPAND>, p);
    default:
        e = cudaFuncSetAttribute(sgmv_kernel<SGMV_APPLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, sgmv_kernel<SGMV_APPLY>, p);
    }
}

}  // namespace lora
