// sgmv_tc.cu -- SGMV (Punica README, "How?": the added term x_i.A_i.B_i of
// every adapter's segment) on the tcgen05 tensor cores, for batches whose
// segments are long (prefill-like: the 64-token tiles of lora_segments_t fill
// the MMAs): the expand y += s_a * v.B_a, and (at the end of the file) the
// shrink v = x.A_a into planes of v that the expand sums.
//
// Expand. One MMA per block of 128 output columns: D[t][n] = sum_j v[t][j] * B_a[j][n]
// (M = 128 rows, N = 128 columns, K = the adapter's rank rounded up to 16),
// accumulated in TMEM. A tile has at most 64 tokens, so v's rows fill M twice
// (rows 64..127 repeat rows 0..63): each of the four drain warps then reads
// valid TMEM lanes, two warps per half of the columns. B_a's rows (rank index
// j, columns contiguous) arrive by TMA as two 64-column boxes with the
// 128-byte swizzle, which is the MN-major operand layout as it stands, so
// B_a is read straight from the pool. v (fp32) is split, once per tile row a
// CTA works on, into bf16 halves v = hi + lo (~16 bits of v), kept as K-major
// 128-byte-swizzled operands; both halves go into the same accumulator.
//
// y rows of a block come into shared memory as 16-byte cp.async copies from
// all lanes of the producer (two 256-byte rows per instruction; a 1-D bulk
// copy per row would queue 64 small requests on the SM's copy engine), their
// 16-byte chunks XOR-swizzled by the row so that a warp whose lanes are rows
// reads without bank conflicts. A drain thread owns one token row and 64
// columns: it adds s_a D to its 128 bytes of y in place, then its warp writes
// its 32 rows back with coalesced 16-byte stores (8 lanes per 128-byte row).
// Gathered (unsorted) tokens cost nothing extra.
//
// Roles (192 threads): warp 0 fills a ring of two stages (B boxes by TMA, y
// rows by cp.async) on mbarriers; warp 1 owns TMEM (two accumulators of 128
// columns) and its lane 0 issues the MMAs; warps 2..5 build v's operands,
// then drain each accumulator into y (warp w reads TMEM lanes 32 (w % 4) ..
// + 31). The persistent grid (two CTAs per SM) splits the sequence of (tile
// row, slice, column block) units evenly, a CTA's run crossing rows where it
// must. Every wait is bounded; on expiry the CTA records a status word in
// lora_segments_t.counts, drains what it issued and leaves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "internal.h"
#include "ptx.cuh"
#include "sgmv_common.cuh"

namespace lora {
namespace {

constexpr int kTcThreads = 192;
constexpr int kTcStages = 2;
constexpr int kTcBlockN = 128;             // output columns per MMA (the N of the MMA)
constexpr int kTcMinCtas = 2;              // CTAs per SM the shared memory is sized for
constexpr int kTcChunks = kTcBlockN / 8;   // 16-byte chunks of a y row of one block
constexpr int kTcSwz = (kTcChunks < 16 ? kTcChunks : 16) - 1;
constexpr int kTcVBytes = 2 * kTT * 128;   // one bf16 half of v: 128 rows (64 twice) x 128 bytes
constexpr int kTcBBytes = (kTcBlockN / 64) * 64 * 128;  // 64-column boxes of up to 64 rank rows
constexpr int kTcYBytes = kTT * kTcBlockN * 2;          // the tile's y rows of one block
constexpr int kTcStageBytes = kTcBBytes + kTcYBytes;
constexpr int kTcTmemCols = 2 * kTcBlockN;              // two accumulators
constexpr int kTcMaxPlanes = 8;                         // planes of v the expand sums

struct TcExpandParams {
    const float* v;        // v_parts planes of v, v_part_stride floats apart; v is their sum
    long long v_part_stride;
    int v_parts;
    uint16_t* y;
    const int32_t* ranks;
    const float* scales;
    const int32_t* perm;
    const int4* tiles;
    int32_t* counts;
    int T, n_adapters, h_out, r_max, n_slices;
    int max_rows;  // rows of the tile table
    int nblk;      // column blocks of kTcBlockN per row
    unsigned long long timeout_ns;
    int inject_stall;
};

// UMMA shared-memory descriptor of an MN-major bf16 operand as TMA leaves
// 64-column boxes with the 128-byte swizzle (one 128-byte row per k): 8-row
// groups 1024 bytes apart along K (stride byte offset), 64-column atoms
// `atom_bytes` apart along M / N (leading byte offset), version 1.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t atom_bytes)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((atom_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// The same for a K-major operand with 128-byte rows (64 bf16 of K), 128-byte
// swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: A = B = bf16, A K-major, B MN-major,
// D fp32, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_mn_b(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

// Byte offset of 16-byte chunk c of token row t in a stage's y block (256-byte
// rows; the chunk index XORed with the row's low four bits).
__device__ __forceinline__ int y_chunk(int t, int c) { return t * (kTcBlockN * 2) + ((c ^ (t & kTcSwz)) << 4); }

// One tile row of one slice as every role sees it.
struct TcRow {
    int nt, nt16, tok0, r, r16, b_map, rB, sa;
    float scale;
    uint32_t atom;
    bool live;  // 1 <= nt <= 64
};

__device__ __forceinline__ TcRow tc_row(const TcExpandParams& p, int row, int slice)
{
    const int4 tl = p.tiles[row];
    TcRow w;
    w.nt = tl.z;
    w.live = tl.z >= 1 && tl.z <= kTT && tl.x >= 0 && tl.x < p.n_adapters;
    const int a = w.live ? tl.x : 0;
    int r = p.ranks ? p.ranks[a] : p.r_max;
    w.r = max(1, min(r, p.r_max));
    w.r16 = round_up(w.r, 16);
    w.nt16 = round_up(max(w.nt, 1), 16);
    w.tok0 = tl.y;
    w.b_map = (w.r16 >> 4) - 1;
    w.rB = min(w.r16, p.r_max);
    w.atom = (uint32_t)(w.r16 * 128);
    w.sa = slice * p.n_adapters + a;
    w.scale = p.scales ? p.scales[a] : 1.0f;
    return w;
}

// The grid splits the sequence of (tile row, slice, column block) units evenly:
// CTA c takes units [c U / G, (c + 1) U / G), U = tile rows x slices x blocks,
// so every SM gets the same number of blocks whatever the segment lengths. A
// CTA whose run crosses into another (row, slice) rebuilds v's operands once
// the previous row's last accumulator is drained (its MMAs are then complete).
__global__ void __launch_bounds__(kTcThreads, kTcMinCtas)
sgmv_expand_tc_kernel(const __grid_constant__ AMaps am, const TcExpandParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ int s_ptok[kTT];  // the producer's token table of its current row
    __shared__ int s_abort;
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // the previous kernel in the stream (the shrink, the segment builder) may still run
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    const int n_rows = min(p.counts[3], p.max_rows);
    const long long total = (long long)max(n_rows, 0) * p.n_slices * p.nblk;
    const long long u0 = (long long)blockIdx.x * total / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * total / gridDim.x;
    if (u0 >= u1) return;
    int32_t* status = p.counts + kSegStatusSlot;
    const int rs_per = p.nblk;  // units per (row, slice)

    const uint32_t raw_u = ptx::smem_u32(smem_raw);
    const uint32_t base_u = (raw_u + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base_u - raw_u);
    const uint32_t vhi_u = base_u, vlo_u = base_u + kTcVBytes;
    const uint32_t ring_u = base_u + 2 * kTcVBytes;
    uint8_t* ring = smem + 2 * kTcVBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kTcStages * kTcStageBytes);
    uint64_t* empty = full + kTcStages;
    uint64_t* tfull = empty + kTcStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* vready = tempty + 2;
    uint64_t* mdone = vready + 1;
    uint64_t* stall = mdone + 1;  // test hook: never completed
    volatile int* abort_flag = &s_abort;

    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < kTcStages; ++s) {
            ptx::mbar_init(&full[s], 1 + 32);  // lane 0's expect_tx + every producer lane's copies
            ptx::mbar_init(&empty[s], 1 + 4);  // the MMAs' commit + the four drain warps
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], 4);
        }
        ptx::mbar_init(vready, 4);
        ptx::mbar_init(mdone, 1);
        ptx::mbar_init(stall, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&s_tmem, kTcTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ================================================================ producer
        int issued[kTcStages] = {};
        bool go = true;
        if (p.inject_stall && u0 == 0)  // test hook (the CTA of the first unit): a wait that runs out
            go = wait_all<false>(stall, 0, abort_flag, status, 0x2000, p.timeout_ns);
        long long cur = -1;
        TcRow w{};
        const uint16_t* yg = p.y;
        int i = 0;  // live blocks so far
        for (long long u = u0; u < u1 && go; ++u) {
            const long long rs = u / rs_per;
            if (rs != cur) {
                cur = rs;
                const int row = (int)(rs / p.n_slices), slice = (int)(rs - (long long)row * p.n_slices);
                w = tc_row(p, row, slice);
                yg = p.y + (size_t)slice * p.T * p.h_out;
                __syncwarp();  // the previous row's copies were issued from s_ptok
                if (w.live)
                    for (int t = lane; t < w.nt; t += 32) s_ptok[t] = p.perm[w.tok0 + t];
                __syncwarp();
                if (lane == 0 && w.live) ptx::tma_prefetch_desc(&am.b[w.b_map]);
            }
            if (!w.live) continue;
            const int st = i % kTcStages;
            if (i >= kTcStages &&
                !wait_all<false>(&empty[st], (uint32_t)(((i / kTcStages) - 1) & 1), abort_flag, status, 0x100,
                                 p.timeout_ns))
                break;
            const int n0 = (int)(u - rs * rs_per) * kTcBlockN;
            const int wc = min(kTcBlockN, p.h_out - n0);
            const int nbox = (wc + 63) >> 6;
            const uint32_t sb = ring_u + (uint32_t)(st * kTcStageBytes);
            const uint32_t sy = sb + kTcBBytes;
            if (lane == 0) ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)(nbox * 64 * w.rB * 2));
            __syncwarp();
            // boxes of 64 columns x rB rank rows, placed r16 rows apart (rows past h_out read as zero)
            if (lane < nbox)
                ptx::tma_load_3d(sb + (uint32_t)lane * w.atom, &am.b[w.b_map], &full[st], n0 + lane * 64, 0, w.sa);
            // the tile's y rows, 16 bytes per lane (several rows per instruction: one small
            // copy instruction per row would serialise on the copy engine)
            const int cpr = wc >> 3;
            if (cpr == kTcChunks) {
                constexpr int kRowsPer = 32 / kTcChunks;
                const int c = lane % kTcChunks;
                for (int t = lane / kTcChunks; t < w.nt; t += kRowsPer)
                    ptx::cp_async16(sy + (uint32_t)y_chunk(t, c), yg + (size_t)s_ptok[t] * p.h_out + n0 + c * 8, 16);
            } else {
                for (int idx = lane; idx < w.nt * cpr; idx += 32) {
                    const int t = idx / cpr, c = idx - t * cpr;
                    ptx::cp_async16(sy + (uint32_t)y_chunk(t, c), yg + (size_t)s_ptok[t] * p.h_out + n0 + c * 8, 16);
                }
            }
            ptx::cp_async_arrive_noinc(&full[st]);
            ++issued[st];
            ++i;
        }
        // let every copy this CTA issued land before it leaves
        for (int st = 0; st < kTcStages; ++st)
            if (issued[st]) wait_all<false, false>(&full[st], (uint32_t)((issued[st] - 1) & 1), abort_flag, status,
                                                   0x800, p.timeout_ns);
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        const uint32_t idesc = idesc_mn_b(kTcBlockN);
        long long cur = -1;
        TcRow w{};
        int i = 0, nv = 0;
        bool ok = true;
        for (long long u = u0; u < u1 && ok; ++u) {
            const long long rs = u / rs_per;
            if (rs != cur) {
                cur = rs;
                const int row = (int)(rs / p.n_slices), slice = (int)(rs - (long long)row * p.n_slices);
                w = tc_row(p, row, slice);
                if (!w.live) {
                    if (lane == 0 && w.nt > kTT) atomicOr(status, kSegTooLarge);
                    continue;
                }
                // v's operands of this row are built
                ok = wait_all<false>(vready, (uint32_t)(nv & 1), abort_flag, status, 0x200, p.timeout_ns);
                ++nv;
                if (!ok) break;
            }
            if (!w.live) continue;
            const int st = i % kTcStages, buf = i & 1;
            if (!wait_all<false>(&full[st], (uint32_t)((i / kTcStages) & 1), abort_flag, status, 0x800,
                                 p.timeout_ns))
                break;
            const uint32_t sb = ring_u + (uint32_t)(st * kTcStageBytes);
            if (w.r != w.r16) {  // rank rows r..r16 of every box: pool padding or nothing; zero them
                const int zr = w.r16 - w.r;
                for (int c = lane; c < (kTcBlockN / 64) * zr * 8; c += 32) {
                    const int bx = c / (zr * 8), rem = c - bx * zr * 8;
                    *reinterpret_cast<uint4*>(ring + st * kTcStageBytes + bx * (int)w.atom + (w.r + (rem >> 3)) * 128 +
                                              (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
                ptx::fence_proxy_async_smem();
            }
            __syncwarp();
            if (i >= 2 && !wait_all<false>(&tempty[buf], (uint32_t)(((i >> 1) - 1) & 1), abort_flag, status, 0x200,
                                           p.timeout_ns))
                break;
            if (lane == 0) {
                ptx::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * kTcBlockN);
                for (int h = 0; h < 2; ++h) {
                    const uint32_t vb = h ? vlo_u : vhi_u;
                    for (int ks = 0; ks < (w.r16 >> 4); ++ks)
                        ptx::tc_mma_f16(d, desc_k_sw128(vb + (uint32_t)(ks * 32)),
                                        desc_mn_sw128(sb + (uint32_t)(ks * 2048), w.atom), idesc, (h | ks) ? 1u : 0u);
                }
                ptx::tc_commit(&empty[st]);  // the B boxes may be refilled once these MMAs are done
                ptx::tc_commit(&tfull[buf]);
            }
            __syncwarp();
            ++i;
        }
        // every MMA this thread issued is complete before TMEM is released
        if (lane == 0) ptx::tc_commit(mdone);
        __syncwarp();
        wait_all<false, false>(mdone, 0, abort_flag, status, 0x200, p.timeout_ns);
    } else {
        // ================================================================ v operands, then drains
        const int q = warp & 3;             // TMEM lane quarter this warp may read
        const int et = (warp - 2) * 32 + lane;
        const int t = (q & 1) * 32 + lane, hf = q >> 1;  // this thread: token row t, half hf of a block
        const int rbase = (q & 1) * 32;                  // the warp's 32 rows
        constexpr int kLanesPerRow = kTcChunks / 2, kRowsPer = 32 / kLanesPerRow, kStoreRows = 32 / kRowsPer;
        long long yoff[kStoreRows];  // y offsets of the rows this lane stores
        long long cur = -1;
        TcRow w{};
        int i = 0;
        bool ok = true;
        for (long long u = u0; u < u1 && ok; ++u) {
            const long long rs = u / rs_per;
            if (rs != cur) {
                cur = rs;
                const int row = (int)(rs / p.n_slices), slice = (int)(rs - (long long)row * p.n_slices);
                w = tc_row(p, row, slice);
                if (!w.live) continue;
                // v rows t < nt16 as bf16 hi / lo halves, K-major, 128-byte rows, 128-byte
                // swizzle, at rows t and t + 64; columns j >= r (and rows t >= nt) are zero.
                // Every MMA of the previous row is complete (its last block was drained).
                const int cpr = w.r16 >> 3;
                const int n_items = w.nt16 * cpr;
                // the items' token indices first (independent loads), then each item's planes
                int tokv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int idx = et + 128 * k, tv = idx / cpr;
                    tokv[k] = idx < n_items && tv < w.nt ? p.perm[w.tok0 + tv] : 0;
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int idx = et + 128 * k;
                    if (idx >= n_items) break;
                    const int tv = idx / cpr, c = idx - tv * cpr;
                    float fv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (tv < w.nt && 8 * c < w.r) {
                        // the planes' loads first, then their sum in plane order
                        const float4* src = reinterpret_cast<const float4*>(
                            p.v + ((size_t)slice * p.T + tokv[k]) * p.r_max + 8 * c);
                        float4 g[kTcMaxPlanes][2];
#pragma unroll
                        for (int pl = 0; pl < kTcMaxPlanes; ++pl)
                            if (pl < p.v_parts) {
                                const float4* sp = src + (size_t)pl * (p.v_part_stride >> 2);
                                g[pl][0] = sp[0];
                                g[pl][1] = sp[1];
                            }
#pragma unroll
                        for (int pl = 0; pl < kTcMaxPlanes; ++pl)
                            if (pl < p.v_parts) {
                                fv[0] += g[pl][0].x; fv[1] += g[pl][0].y; fv[2] += g[pl][0].z; fv[3] += g[pl][0].w;
                                fv[4] += g[pl][1].x; fv[5] += g[pl][1].y; fv[6] += g[pl][1].z; fv[7] += g[pl][1].w;
                            }
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (8 * c + e >= w.r) fv[e] = 0.f;
                    }
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        hi[e] = pack_bf16x2(fv[2 * e], fv[2 * e + 1]);
                        lo[e] = pack_bf16x2(fv[2 * e] - bf16_lo(hi[e]), fv[2 * e + 1] - bf16_hi(hi[e]));
                    }
#pragma unroll
                    for (int rep = 0; rep < 2; ++rep) {
                        const int vrow = tv + rep * kTT;
                        const int off = vrow * 128 + ((c ^ (vrow & 7)) << 4);
                        *reinterpret_cast<uint4*>(smem + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4*>(smem + kTcVBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(vready);
#pragma unroll
                for (int k = 0; k < kStoreRows; ++k) {
                    const int srow = rbase + lane / kLanesPerRow + kRowsPer * k;
                    yoff[k] = srow < w.nt ? ((long long)slice * p.T + p.perm[w.tok0 + srow]) * p.h_out : 0;
                }
            }
            if (!w.live) continue;
            const int st = i % kTcStages, buf = i & 1;
            ok = wait_all<false>(&full[st], (uint32_t)((i / kTcStages) & 1), abort_flag, status, 0x800,
                                 p.timeout_ns);
            ok = ok && wait_all<false>(&tfull[buf], (uint32_t)((i >> 1) & 1), abort_flag, status, 0x200,
                                       p.timeout_ns);
            if (!ok) break;
            ptx::tc_fence_after();
            const int n0 = (int)(u - rs * rs_per) * kTcBlockN;
            const int wc = min(kTcBlockN, p.h_out - n0);
            uint8_t* sy = ring + st * kTcStageBytes + kTcBBytes;
            const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kTcBlockN + hf * (kTcBlockN / 2));
            // y[t][n] += s_a D[t][n] in place, for this thread's row and half block
#pragma unroll
            for (int c4 = 0; c4 < kTcBlockN / 32; ++c4) {
                float d[16];
                ptx::tmem_ld16(ta + (uint32_t)(c4 * 16), d);
                if (t < w.nt) {
#pragma unroll
                    for (int hc = 0; hc < 2; ++hc) {
                        uint4* yp = reinterpret_cast<uint4*>(sy + y_chunk(t, hf * (kTcChunks / 2) + c4 * 2 + hc));
                        uint4 uy = *yp;
                        uint32_t* w4 = reinterpret_cast<uint32_t*>(&uy);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            w4[k] = pack_bf16x2(bf16_lo(w4[k]) + w.scale * d[hc * 8 + 2 * k],
                                                bf16_hi(w4[k]) + w.scale * d[hc * 8 + 2 * k + 1]);
                        *yp = uy;
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
            // the warp's 32 rows of this half back to y: kLanesPerRow lanes per row, 16 bytes
            // each (coalesced 128-byte row pieces)
            {
                const int cc = hf * kLanesPerRow + lane % kLanesPerRow;
                if (cc * 8 < wc)
#pragma unroll
                    for (int k = 0; k < kStoreRows; ++k) {
                        const int srow = rbase + lane / kLanesPerRow + kRowsPer * k;
                        if (srow < w.nt)
                            *reinterpret_cast<uint4*>(p.y + yoff[k] + n0 + cc * 8) =
                                *reinterpret_cast<const uint4*>(sy + y_chunk(srow, cc));
                    }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[st]);
            ++i;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTcTmemCols);
    }
}

// ---------------------------------------------------------------------------- shrink
// Planes of v = x.A_a for the same batches: CTA (tile row, slice, part) sums the
// k-blocks [part nkb / P, (part + 1) nkb / P) of 64 h_in columns into plane `part`
// (P <= 8 planes; the expand adds them in plane order, so the result does not depend
// on timing). D[t][j] = sum_k x[t][k] A_a[k][j] with M = 128, N = 64, K = 16 per MMA:
// the tile's tokens are rows 64..127 of the x operand, whose descriptor starts 8 KB
// before the x tile (rows 0..63 read the stage's A box as filler and their results
// are dropped), so drain warps 2 and 3 read valid TMEM lanes. A_a's k rows arrive by
// TMA as one 64-column box with the 128-byte swizzle (the MN-major operand; columns
// past the rank, pool padding or past r_max, are dropped from the result); the
// tile's x rows by cp.async into the K-major 128-byte-swizzled layout.
constexpr int kShThreads = 128;
constexpr int kShStages = 4;
constexpr int kShBox = 64 * 64 * 2;           // 64 k rows x 64 columns of A_a, or 64 tokens x 64 k of x
constexpr int kShStageBytes = 2 * kShBox;     // A box, then the x tile
constexpr int kShTmemCols = 64;

struct TcShrinkParams {
    const uint16_t* x;
    long long x_slice_stride;
    const int32_t* ranks;
    const int32_t* perm;
    const int4* tiles;
    int32_t* counts;
    float* v;  // parts planes of [n_slices][T][r_max]
    long long v_part_stride;
    int T, n_adapters, h_in, r_max, n_slices;
    int parts, nkb;  // planes; 64-column k-blocks of h_in
    unsigned long long timeout_ns;
    int inject_stall;
};

__global__ void __launch_bounds__(kShThreads, 3)
sgmv_shrink_tc_kernel(const __grid_constant__ CUtensorMap a_map, const TcShrinkParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ int s_tok[kTT];
    __shared__ int s_abort;
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per_row = p.n_slices * p.parts;
    const int g = blockIdx.x / per_row;
    const int slice = (blockIdx.x - g * per_row) / p.parts;
    const int part = blockIdx.x - g * per_row - slice * p.parts;

    // the previous kernel in the stream (the segment builder, the producer of x) may still run
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    const int4 tl = p.tiles[g];
    const int nt = tl.z;
    if (nt <= 0) return;  // unused tile row
    int32_t* status = p.counts + kSegStatusSlot;
    if (nt > kTT || tl.x < 0 || tl.x >= p.n_adapters) {  // segments not built for this batch size
        if (tid == 0 && part == 0 && slice == 0) atomicOr(status, kSegTooLarge);
        return;
    }
    const int kb0 = (int)((long long)part * p.nkb / p.parts);
    const int nkb = (int)((long long)(part + 1) * p.nkb / p.parts) - kb0;  // >= 1 (parts <= nkb)
    const int a = tl.x, tok0 = tl.y;
    int r = p.ranks ? p.ranks[a] : p.r_max;
    r = max(1, min(r, p.r_max));
    const int sa = slice * p.n_adapters + a;

    const uint32_t raw_u = ptx::smem_u32(smem_raw);
    const uint32_t base_u = (raw_u + 1023u) & ~1023u;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + (base_u - raw_u) + kShStages * kShStageBytes);
    uint64_t* empty = full + kShStages;
    uint64_t* dfull = empty + kShStages;
    uint64_t* stall = dfull + 1;  // test hook: never completed
    volatile int* abort_flag = &s_abort;

    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < kShStages; ++s) {
            ptx::mbar_init(&full[s], 1 + 32);  // lane 0's expect_tx + every producer lane's copies
            ptx::mbar_init(&empty[s], 1);      // the MMAs' commit
        }
        ptx::mbar_init(dfull, 1);
        ptx::mbar_init(stall, 1);
        ptx::fence_mbar_init();
    }
    if (tid < nt) s_tok[tid] = p.perm[tok0 + tid];
    if (warp == 1) {
        ptx::tmem_alloc(&s_tmem, kShTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) ptx::tma_prefetch_desc(&a_map);
        const uint16_t* xs = p.x + (size_t)(p.x_slice_stride ? slice : 0) * p.x_slice_stride;
        int issued[kShStages] = {};
        bool go = true;
        if (p.inject_stall && blockIdx.x == 0)  // test hook: a wait that runs out
            go = wait_all<false>(stall, 0, abort_flag, status, 0x2000, p.timeout_ns);
        for (int i = 0; i < nkb && go; ++i) {
            const int st = i % kShStages;
            if (i >= kShStages &&
                !wait_all<false>(&empty[st], (uint32_t)(((i / kShStages) - 1) & 1), abort_flag, status, 0x100,
                                 p.timeout_ns))
                break;
            const int k0 = (kb0 + i) * 64;
            const uint32_t sA = base_u + (uint32_t)(st * kShStageBytes), sx = sA + kShBox;
            if (lane == 0) ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)kShBox);
            __syncwarp();
            // k rows past h_in and columns past r_max read as zero
            if (lane == 0) ptx::tma_load_3d(sA, &a_map, &full[st], 0, k0, sa);
            // x rows: 8 chunks of 16 bytes each, chunk index XOR row (the 128-byte swizzle);
            // chunks past h_in are zero-filled
            for (int idx = lane; idx < nt * 8; idx += 32) {
                const int t = idx >> 3, c = idx & 7, col = k0 + 8 * c;
                const uint16_t* src = xs + (size_t)s_tok[t] * p.h_in + (col < p.h_in ? col : 0);
                ptx::cp_async16(sx + (uint32_t)(t * 128 + ((c ^ (t & 7)) << 4)), src, col < p.h_in ? 16u : 0u);
            }
            ptx::cp_async_arrive_noinc(&full[st]);
            ++issued[st];
        }
        // let every copy this CTA issued land before it leaves
        for (int st = 0; st < kShStages; ++st)
            if (issued[st]) wait_all<false, false>(&full[st], (uint32_t)((issued[st] - 1) & 1), abort_flag, status,
                                                   0x800, p.timeout_ns);
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        const uint32_t idesc = idesc_mn_b(64);
        for (int i = 0; i < nkb; ++i) {
            const int st = i % kShStages;
            if (!wait_all<false>(&full[st], (uint32_t)((i / kShStages) & 1), abort_flag, status, 0x800,
                                 p.timeout_ns))
                break;
            if (lane == 0) {
                ptx::tc_fence_after();
                const uint32_t sA = base_u + (uint32_t)(st * kShStageBytes);
                for (int ks = 0; ks < 4; ++ks)
                    ptx::tc_mma_f16(tmem, desc_k_sw128(sA + (uint32_t)(ks * 32)),
                                    desc_mn_sw128(sA + (uint32_t)(ks * 2048), (uint32_t)kShBox), idesc,
                                    (i | ks) ? 1u : 0u);
                ptx::tc_commit(&empty[st]);
            }
            __syncwarp();
        }
        // the accumulator is complete (or, after an abort, every issued MMA is)
        if (lane == 0) ptx::tc_commit(dfull);
        __syncwarp();
    } else {
        // ================================================================ drain: plane rows
        const int q = warp & 3;  // 2 or 3: TMEM lanes 64..127, the tile's tokens
        const int t = (q - 2) * 32 + lane;
        const bool ok = wait_all<false, false>(dfull, 0, abort_flag, status, 0x200, p.timeout_ns);
        ptx::tc_fence_after();
        float d[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 16), d + c * 16);
        if (ok && !*abort_flag && t < nt) {
            float* dst = p.v + (size_t)part * p.v_part_stride + ((size_t)slice * p.T + s_tok[t]) * p.r_max;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                if (j >= p.r_max) break;
                float4 o;
                o.x = j < r ? d[j] : 0.f;
                o.y = j + 1 < r ? d[j + 1] : 0.f;
                o.z = j + 2 < r ? d[j + 2] : 0.f;
                o.w = j + 3 < r ? d[j + 3] : 0.f;
                *reinterpret_cast<float4*>(dst + j) = o;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kShTmemCols);
    }
}

}  // namespace

bool sgmv_expand_tc_eligible(int T, const lora_pool_t& pool)
{
    // long segments (on average at least half a tile per adapter and slice) and a
    // y row of at least one block
    return tile_tokens_for(T, pool.n_adapters) == kTT && T >= 32LL * pool.n_adapters &&
           pool.h_out >= kTcBlockN;
}

cudaError_t launch_sgmv_expand_tc(const float* v, int v_parts, const lora_pool_t& pool, const lora_segments_t& seg,
                                  void* y, cudaStream_t stream)
{
    if (seg.T == 0) return cudaSuccess;
    TcExpandParams p = {};
    p.v = v;
    p.v_parts = v_parts;
    p.v_part_stride = (long long)pool.n_slices * seg.T * pool.r_max;
    p.y = static_cast<uint16_t*>(y);
    p.ranks = pool.ranks;
    p.scales = pool.scales;
    p.perm = seg.perm;
    p.tiles = reinterpret_cast<const int4*>(seg.tiles);
    p.counts = seg.counts;
    p.T = seg.T;
    p.n_adapters = pool.n_adapters;
    p.h_out = pool.h_out;
    p.r_max = pool.r_max;
    p.n_slices = pool.n_slices;
    p.timeout_ns = debug_wait_limit_ns();
    p.inject_stall = debug_inject_stall();
    p.nblk = (pool.h_out + kTcBlockN - 1) / kTcBlockN;
    p.max_rows = max_tiles_for(seg.T, pool.n_adapters);
    // persistent: one wave of kTcMinCtas CTAs per SM (or one per unit when there are fewer)
    const long long units = (long long)p.max_rows * pool.n_slices * p.nblk;
    long long grid = (long long)kTcMinCtas * device_sm_count();
    if (grid > units) grid = units;

    AMaps am;
    if (!build_pool_maps(am, pool, false, true)) return cudaErrorInvalidValue;
    const size_t smem = 2 * kTcVBytes + (size_t)kTcStages * kTcStageBytes + 8 * (4 * kTcStages + 8) + 1024;
    auto kern = sgmv_expand_tc_kernel;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, am, p);
}

int sgmv_shrink_tc_parts(const lora_pool_t& pool)
{
    const int nkb = (pool.h_in + 63) / 64;
    return nkb < kTcMaxPlanes ? nkb : kTcMaxPlanes;
}

cudaError_t launch_sgmv_shrink_tc(const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                                  const lora_segments_t& seg, float* v, int parts, cudaStream_t stream)
{
    if (seg.T == 0) return cudaSuccess;
    TcShrinkParams p = {};
    p.x = static_cast<const uint16_t*>(x);
    p.x_slice_stride = x_slice_stride;
    p.ranks = pool.ranks;
    p.perm = seg.perm;
    p.tiles = reinterpret_cast<const int4*>(seg.tiles);
    p.counts = seg.counts;
    p.v = v;
    p.v_part_stride = (long long)pool.n_slices * seg.T * pool.r_max;
    p.T = seg.T;
    p.n_adapters = pool.n_adapters;
    p.h_in = pool.h_in;
    p.r_max = pool.r_max;
    p.n_slices = pool.n_slices;
    p.nkb = (pool.h_in + 63) / 64;
    p.parts = parts < 1 ? 1 : (parts > p.nkb ? p.nkb : parts);
    p.timeout_ns = debug_wait_limit_ns();
    p.inject_stall = debug_inject_stall();
    // A as {r_max, h_in, slices x adapters}, box {64, 64, 1}, 128-byte swizzle (columns past
    // r_max and rows past h_in read as zero)
    CUtensorMap a_map;
    const uint64_t dims[3] = {(uint64_t)pool.r_max, (uint64_t)pool.h_in,
                              (uint64_t)pool.n_slices * (uint64_t)pool.n_adapters};
    const uint64_t strides[2] = {(uint64_t)pool.r_max * 2, (uint64_t)pool.h_in * pool.r_max * 2};
    const uint32_t box[3] = {64, 64, 1};
    if (!encode_tmap_3d(&a_map, CU_TENSOR_MAP_DATA_TYPE_UINT16, pool.A, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)kShStages * kShStageBytes + 8 * (2 * kShStages + 2) + 1024;
    auto kern = sgmv_shrink_tc_kernel;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)max_tiles_for(seg.T, pool.n_adapters) * pool.n_slices * p.parts), 1, 1);
    cfg.blockDim = dim3(kShThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a_map, p);
}

}  // namespace lora
