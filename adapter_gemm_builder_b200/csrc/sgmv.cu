// sgmv.cu -- Segmented Gather Matrix-Vector multiplication for multi-tenant
// LoRA (Punica README, "How?": the added term (x_i.A_i.B_i) for a batch whose
// tokens map to different adapters, for all adapters in one kernel).
//
// One kernel, three modes:
//   SHRINK  v = x.A_a            (fp32, written to global)
//   EXPAND  y += s_a * v.B_a     (v read from global, y bf16 read-modify-write)
//   APPLY   y += s_a * (x.A_a).B_a, with v kept on chip
//
// Work. The segment builder cuts every adapter's run of tokens into tiles of
// at most lora_tile_tokens_for(T, n_adapters) tokens (one row of
// lora_segments_t.tiles each): 4 for a decode-like batch, which then runs
// the kernel variant built for such tiles alone (no tensor-core path: a
// smaller kernel whose short-lived CTAs wait less on instruction fetch), else
// LORA_TILE_TOKENS. A
// tile is handled by a thread-block cluster of C CTAs: in the shrink CTA c
// owns the c-th slice of h_in (split-K) and computes a partial v for the
// tile's tokens; in the expand it owns the c-th slice of h_out. The grid covers
// every (tile row, slice) pair, the slices of a row adjacent, so q/k/v/o run in
// one launch.
//
// Memory path (the kernel is bound by HBM bytes and by latency). A producer
// warp fills a ring of 3 stages whose copies all complete on the stage's
// mbarrier. The k rows of A_a come as tensor-map boxes of only the adapter's
// live columns (128-, 64- or 32-byte swizzled rows: the pool's padding past
// the rank is never read and the tensor-core reads are free of bank
// conflicts) or, for a decode tile whose rank rounds to r_max, as one
// contiguous 1-D bulk copy. Decode tiles take their few x, B and y rows as
// 1-D bulk copies, issued from all lanes in parallel (a copy instruction
// costs ~35 ns of issue, so one lane issuing many small copies would
// serialise). Tensor-core tiles keep x, B_a and y in blocks of 64 columns
// whose 128-byte rows are swizzled (bank-conflict free for ldmatrix): B_a
// comes as tensor-map boxes, and so do x and y when the tile's tokens are
// consecutive rows (pre-sorted batches); otherwise the rows are gathered with
// 16-byte cp.async spread over all 32 lanes, written in the same layout.
//
// Math. Tiles of at most 4 tokens (decode) use CUDA-core FMAs: the products
// are few and a 16-row MMA would be mostly padding. Larger tiles use bf16
// tensor-core MMA (m16n8k16, fp32 accumulate) with all tile-invariant
// addressing hoisted out of the k loop; their expand operand v (fp32) is
// split as v = hi + lo in bf16 and both halves are multiplied (~16 bits of v).
//
// Reduction of v. Partials travel by distributed shared memory with st.async:
// each store lands in a peer's shared memory and counts as transaction bytes
// on that peer's mbarrier, which expects exactly the bytes it must receive.
// With few rows all CTAs receive all partials (one exchange); with many rows
// a reduce-scatter by row is followed by an all-gather. Every wait is
// bounded (2 s); on expiry the kernel records a status word in
// lora_segments_t.counts and stops computing, but still takes part in every
// barrier.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "internal.h"
#include "ptx.cuh"
#include "sgmv_common.cuh"

namespace lora {
namespace {

constexpr int kMaxCluster = 8;
constexpr int kOnePhaseBytes = 8192;     // all-to-all exchange of v up to this size per CTA

struct SgmvParams {
    const uint16_t* x;
    long long x_slice_stride;
    const uint16_t* A;
    const uint16_t* B;
    const int32_t* ranks;
    const float* scales;
    const int32_t* perm;
    const int4* tiles;  // the segments' tile rows, or the same rows in cost order (tile_order_kernel)
    int32_t* counts;
    float* v;
    uint16_t* y;
    int T, n_adapters, h_in, h_out, r_max;
    int n_slices;
    int csize;       // CTAs per tile
    int kc, nc;      // h_in / h_out slice per CTA (kc a multiple of 128, nc of 64)
    int rp;          // round_up(r_max, 16): row pitch (floats) of the v buffers
    int stage_bytes; // one ring stage
    int xy_maps;     // tensor maps of x and y are valid (consecutive-row tiles use them)
    uint32_t off_rb, off_vf, off_bar;
    unsigned long long timeout_ns;  // limit of every bounded wait (2 s unless a test lowers it)
    int inject_stall;  // test hook: one CTA's producer first waits on a barrier nothing completes
};

// kSmallOnly: every tile holds <= kSmallTile tokens (the tiles of a decode-like
// batch), so the tensor-core path for larger tiles is left out of this variant:
// a smaller kernel, whose dependent steps wait less on instruction fetch.
template <int MODE, bool kSmallOnly>
__global__ void __launch_bounds__(kThreads, 2)
sgmv_kernel(const __grid_constant__ AMaps am, const SgmvParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ int s_tok[kTT];
    __shared__ int s_abort;

    constexpr bool kClustered = MODE != SGMV_EXPAND;
    const uint32_t raw_u = ptx::smem_u32(smem_raw);
    const uint32_t base_u = (raw_u + 1023u) & ~1023u;  // swizzled boxes need 1024-byte alignment
    uint8_t* smem = smem_raw + (base_u - raw_u);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = p.csize;
    const int rank = kClustered ? (int)ptx::cluster_ctarank() : (int)(blockIdx.x % C);
    // blockIdx.x = ((tile row * n_slices) + slice) * C + rank: the slices of a tile row
    // launch together (with the rows in cost order, every slice's long rows start first)
    const int g = (blockIdx.x / C) / p.n_slices;
    const int slice = (blockIdx.x / C) - g * p.n_slices;
    const int SB = p.stage_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
    uint64_t* empty = full + kStages;
    uint64_t* red1 = empty + kStages;
    uint64_t* red2 = red1 + 1;
    uint64_t* stall = red2 + 1;  // test hook: never completed
    volatile int* abort_flag = &s_abort;
    int32_t* status = p.counts + kSegStatusSlot;

    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 33);  // lane 0's expect_tx + one arrival per producer lane
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(red1, 1);
        ptx::mbar_init(red2, 1);
        ptx::mbar_init(stall, 1);
        ptx::fence_mbar_init();
    }
    __syncwarp();  // __syncthreads is an aligned barrier: warps reach it converged
    // Cluster barrier, phase 0: this CTA's mbarriers exist (peers wait for it before
    // their first remote store); phase 1: this CTA makes no more remote accesses (every
    // CTA waits for it before leaving). Phase 0 is announced before the wait on the
    // previous kernel, so it overlaps that kernel's tail.
    __syncthreads();
    if (kClustered) ptx::cluster_arrive();
    // the previous kernel in the stream (e.g. the segment builder) may still run
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();

    const int4 tl = p.tiles[g];
    const int nt = tl.z;
    if (nt <= 0) return;  // unused row: the cluster leaves together
    const int a = tl.x, tok0 = tl.y;
    int r = p.ranks ? p.ranks[a] : p.r_max;
    r = max(1, min(r, p.r_max));
    const float scale = p.scales ? p.scales[a] : 1.0f;
    const int r8 = round_up(r, 8), r16 = round_up(r, 16);
    if (kSmallOnly && nt > kSmallTile) {  // segments not built for this batch size: the
        if (tid == 0 && rank == 0) atomicOr(status, kSegTooLarge);  // whole cluster leaves
        return;
    }
    const bool small = kSmallOnly || nt <= kSmallTile;
    const int Mt = (nt + 15) >> 4;
    const int Mtr = small ? nt : Mt * 16;  // x / y rows held per stage (tail rows zero)
    if (tid < nt) s_tok[tid] = p.perm[tok0 + tid];

    // ---- geometry (identical in every role)
    // A rows in shared memory: tensor-map boxes of rA >= r live columns (rA the power of
    // two >= r8; dense, swizzled when rA >= 16), or for decode tiles whose rank rounds to
    // r_max the pool's contiguous rows
    const int a_map = r8 <= 8 ? 0 : 32 - __clz((r8 >> 3) - 1);  // log2(rA / 8)
    const int rA = 8 << a_map;
    const bool a_tma = !small || rA < p.r_max;
    const int apitch = a_tma ? rA * 2 : p.r_max * 2;
    const int a_swz = (a_tma && rA >= 16) ? (rA >> 3) - 1 : 0;
    const int k_begin = min(p.h_in, rank * p.kc);
    const int k_len = min(p.h_in, k_begin + p.kc) - k_begin;
    int BK;
    if (small) {
        BK = ((SB - 16 * Mtr) / (apitch + 2 * Mtr)) / 64 * 64;
        BK = min(BK, round_up(max(k_len, 1), 64));
    } else {
        // a divisor of kc (a multiple of 128), so only the last block of h_in is partial
        BK = 64;
        for (int b = 256; b > 64; b >>= 1)
            if (p.kc % b == 0 && b * (apitch + 2 * Mtr) <= SB) {
                BK = b;
                break;
            }
    }
    const int nK = (MODE == SGMV_EXPAND) ? 0 : (k_len + BK - 1) / BK;
    const int xp = BK * 2 + 16;  // x row pitch of decode tiles (bytes)
    const int n_begin = min(p.h_out, rank * p.nc);
    const int n_len = min(p.h_out, n_begin + p.nc) - n_begin;
    // expand blocks: small tiles keep B in unswizzled boxes of kSmallBoxCols columns (r16
    // rows each) and their y rows at the padded pitch bp;
    // tensor-core tiles keep B (r16 rows) and y (Mtr rows) in swizzled 64-column blocks
    int BN;
    if (small) {
        // whole boxes of kSmallBoxCols columns (B arrives in such boxes)
        BN = ((SB / (r16 + Mtr) - 16) / 2) / kSmallBoxCols * kSmallBoxCols;
    } else {
        BN = 64;  // a power of two, so the gathers need no division
        while (BN < 256 && 2 * BN * (2 * r16 + 2 * Mtr) <= SB) BN *= 2;
    }
    BN = min(BN, round_up(max(n_len, 1), small ? kSmallBoxCols : 64));
    const int nN = (MODE == SGMV_SHRINK) ? 0 : (n_len + BN - 1) / BN;
    const int bp = BN * 2 + 16;  // y row pitch (and B row pitch of decode tiles), bytes
    const int b_map = (r16 >> 4) - 1;
    const int rB = min(r16, p.r_max);                               // rows per B box
    const uint32_t y_off = small ? (uint32_t)(r16 * bp) : (uint32_t)((BN >> 6) * r16 * 128);
    const int nItems = nK + nN;
    const size_t sa = (size_t)slice * p.n_adapters + a;
    const uint16_t* Ag = p.A + sa * (size_t)p.h_in * p.r_max;
    const uint16_t* Bg = p.B + sa * (size_t)p.r_max * p.h_out;
    const uint16_t* xg = p.x ? p.x + (size_t)slice * p.x_slice_stride : nullptr;
    uint16_t* yg = p.y ? p.y + (size_t)slice * p.T * p.h_out : nullptr;

    // bytes this CTA receives in the v exchange
    const bool one_phase = C * nt * r8 * 4 <= kOnePhaseBytes;
    const int rows_per = (nt + C - 1) / C;
    const int mine = nt > rank ? (nt - rank + C - 1) / C : 0;
    if (kClustered && tid == 0) {
        ptx::mbar_arrive_expect_tx(red1, (uint32_t)((one_phase ? C * nt : C * mine) * r8 * 4));
        ptx::mbar_arrive_expect_tx(red2, one_phase ? 0u : (uint32_t)(nt * r8 * 4));
    }
    // a decode tile's first A block is one contiguous copy that needs nothing but the
    // geometry: the producer's lane 0 issues it now, ahead of the barrier (its bytes
    // join stage 0's count; the item-0 pass below leaves it out)
    const bool a_early = small && !a_tma && nK > 0;
    if (a_early && warp == kComputeWarps && lane == 0) {
        const uint32_t bytes = (uint32_t)(min(BK, k_len) * apitch);
        ptx::mbar_expect_tx(&full[0], bytes);
        ptx::bulk_g2s(base_u, Ag + (size_t)k_begin * p.r_max, bytes, &full[0]);
    }
    __syncwarp();
    __syncthreads();

    if (warp == kComputeWarps) {
        // ================================================================ producer warp
        if (lane == 0 && a_tma && nK > 0) ptx::tma_prefetch_desc(&am.m[a_map]);
        if (lane == 0 && nN > 0) ptx::tma_prefetch_desc(small ? &am.bs[b_map] : &am.b[b_map]);
        // consecutive token rows (a pre-sorted batch): x and y rows come as tensor-map boxes
        bool contig = false;
        if (!small && p.xy_maps) {
            const int t0 = s_tok[0];
            contig = __all_sync(0xffffffffu, (lane >= nt || s_tok[lane] == t0 + lane) &&
                                                 (lane + 32 >= nt || s_tok[lane + 32] == t0 + lane + 32));
        }
        const int xs = p.x_slice_stride ? slice : 0;
        int issued = 0;
        // test hook: the first CTA of the first tile row waits, before its first copy, on
        // a barrier that nothing completes; the bounded wait runs out and the CTA takes
        // its abort path (not with an early A copy in flight, which that path cannot drain)
        bool go = true;
        if (p.inject_stall && g == 0 && slice == 0 && rank == 0 && !a_early)
            go = wait_all<false>(stall, 0, abort_flag, status, 0x2000, p.timeout_ns);
        for (int it = 0; it < nItems && go; ++it) {
            const int st = it % kStages;
            const uint32_t ph = (uint32_t)((it / kStages) & 1);
            if (!wait_all<false>(&empty[st], ph ^ 1, abort_flag, status, 0x100, p.timeout_ns)) break;
            const uint32_t base = base_u + st * SB;
            // lane 0 announces the stage's tensor-map / bulk bytes before any lane issues a
            // copy; then every lane arrives once its own copies have landed (33 arrivals)
            if (it < nK) {
                const int k0 = k_begin + it * BK;
                const int kb = min(BK, k_begin + k_len - k0);
                const int nbox = (kb + 63) >> 6;  // 64-row boxes; rows past h_in read as zero
                const uint32_t xb = base + (uint32_t)(BK * apitch);
                const bool a_done = a_early && it == 0;  // issued with the geometry
                if (lane == 0) {
                    uint32_t bytes = a_done ? 0u : (a_tma ? (uint32_t)(nbox * 64 * apitch) : (uint32_t)(kb * apitch));
                    if (small) bytes += (uint32_t)(nt * kb * 2);
                    else if (contig) bytes += (uint32_t)(nbox * Mt * 16 * 128);
                    ptx::mbar_arrive_expect_tx(&full[st], bytes);
                }
                __syncwarp();
                // one copy instruction per lane (a copy costs ~150 ns of issue to its thread):
                // lanes 0..nA-1 the A boxes (or the one A bulk copy), then the x boxes or rows
                const int nA = a_done ? 0 : (a_tma ? nbox : 1);
                if (lane < nA) {
                    if (a_tma)
                        ptx::tma_load_3d(base + (uint32_t)(lane * 64 * apitch), &am.m[a_map], &full[st], 0,
                                         k0 + lane * 64, (int)sa);
                    else
                        ptx::bulk_g2s(base, Ag + (size_t)k0 * p.r_max, (uint32_t)(kb * apitch), &full[st]);
                }
                if (small) {
                    for (int row = lane - nA; row < nt; row += 32)
                        if (row >= 0)
                            ptx::bulk_g2s(xb + row * xp, xg + (size_t)s_tok[row] * p.h_in + k0, (uint32_t)(kb * 2),
                                          &full[st]);
                    ptx::mbar_arrive(&full[st]);
                } else {
                    if (contig)  // columns past h_in read as zero
                        for (int i = lane - nA; i < nbox * Mt; i += 32)
                            if (i >= 0)
                                ptx::tma_load_3d(xb + (uint32_t)(((i / Mt) * Mtr + (i % Mt) * 16) * 128), &am.x, &full[st],
                                                 k0 + (i / Mt) * 64, s_tok[0] + (i % Mt) * 16, xs);
                    if (!contig) gather_rows(xb, xg + k0, (size_t)p.h_in, s_tok, nt, kb >> 3, Mtr, lane);
                    ptx::cp_async_arrive_noinc(&full[st]);
                }
            } else {
                const int n0 = n_begin + (it - nK) * BN;
                const int nb = min(BN, n_begin + n_len - n0);
                const uint32_t yb = base + y_off;
                if (small) {
                    // B as tensor-map boxes of kSmallBoxCols columns x rB rows (one request per
                    // box, 256 contiguous bytes of each rank row), the tile's y rows as 1-D copies
                    const int nbox = (nb + kSmallBoxCols - 1) / kSmallBoxCols;
                    if (lane == 0)
                        ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)(nbox * kSmallBoxCols * rB * 2 + nt * nb * 2));
                    __syncwarp();
                    if (lane < nbox)
                        ptx::tma_load_3d(base + (uint32_t)(lane * r16 * kSmallBoxCols * 2), &am.bs[b_map], &full[st],
                                         n0 + lane * kSmallBoxCols, 0, (int)sa);
                    for (int i = lane; i < nt; i += 32)
                        ptx::bulk_g2s(yb + i * bp, yg + (size_t)s_tok[i] * p.h_out + n0, (uint32_t)(nb * 2),
                                      &full[st]);
                    ptx::mbar_arrive(&full[st]);
                } else {
                    const int nbox = (nb + 63) >> 6;
                    if (lane == 0)
                        ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)(nbox * 64 * rB * 2) +
                                                                  (contig ? (uint32_t)(nbox * Mt * 16 * 128) : 0u));
                    __syncwarp();
                    if (lane < nbox)
                        ptx::tma_load_3d(base + (uint32_t)(lane * r16 * 128), &am.b[b_map], &full[st], n0 + lane * 64,
                                         0, (int)sa);
                    if (contig)
                        for (int i = lane - nbox; i < nbox * Mt; i += 32)
                            if (i >= 0)
                                ptx::tma_load_3d(yb + (uint32_t)(((i / Mt) * Mtr + (i % Mt) * 16) * 128), &am.y,
                                                 &full[st], n0 + (i / Mt) * 64, s_tok[0] + (i % Mt) * 16, slice);
                    if (!contig) gather_rows(yb, yg + n0, (size_t)p.h_out, s_tok, nt, nb >> 3, Mtr, lane);
                    ptx::cp_async_arrive_noinc(&full[st]);
                }
            }
            ++issued;
        }
        ptx::cp_async_commit();
        ptx::cp_async_wait<0>();
        if (lane == 0 && *abort_flag) {  // let the copies that were issued land before leaving
            const unsigned long long t0 = ptx::globaltimer();
            for (int it = (issued > kStages ? issued - kStages : 0); it < issued; ++it)
                while (!ptx::mbar_try_wait(&full[it % kStages], (uint32_t)((it / kStages) & 1)) &&
                       ptx::globaltimer() - t0 < kTimeoutNs) {
                }
        }
        __syncwarp();
        if (kClustered) {  // no remote accesses from this warp
            ptx::cluster_wait();
            ptx::cluster_arrive();
        }
    } else {
        // ================================================================ compute warps
        float* VF = reinterpret_cast<float*>(smem + p.off_vf);       // [kTT][rp]: partial, then v
        float* RB = reinterpret_cast<float*>(smem + p.off_rb);       // exchange receive buffer
        uint16_t* Vh = reinterpret_cast<uint16_t*>(smem + p.off_rb); // [kTT][rp+8] (aliases RB)
        uint16_t* Vl = Vh + kTT * (p.rp + 8);
        const int vpitch = p.rp + 8;
        const uint32_t vf_u = base_u + p.off_vf, rb_u = base_u + p.off_rb;
        const uint32_t red1_u = ptx::smem_u32(red1), red2_u = ptx::smem_u32(red2);

        // small tiles, chunks of 8 columns per token padded to a power of two (ncbp).
        // Decode variant: warp w owns the (token, chunk) pairs w, w + 8, ... and its lanes
        // stride over the rows (SACC(i, e): column e of its i-th pair), so no reduction
        // across warps is needed. Otherwise: thread (c_own, rg) owns chunk c_own over rows
        // rg, rg + rstride, ... for every token (SACC(t, e)), one read of A for all tokens.
        const int ncb = r8 >> 3;
        const int lg = ncb <= 1 ? 0 : (ncb <= 2 ? 1 : (ncb <= 4 ? 2 : 3));
        const int ncbp = 1 << lg;
        const int c_own = tid & (ncbp - 1), rg = tid >> lg, rstride = kCompute >> lg;
        // large tiles: warp w owns 16x8 output tiles [w*tpw, (w+1)*tpw) of the (Mt x r8/8) grid
        const int nNT = r8 >> 3;
        const int tiles_s = Mt * nNT;
        const int tpw_s = (tiles_s + kComputeWarps - 1) / kComputeWarps;  // <= 4
        // one register file for both paths (a tile takes exactly one of them):
        // small: R[i*8+e] (see above); large: R[q*4+e] = MMA tile q
        float R[kSmallTile * 8];
#pragma unroll
        for (int i = 0; i < kSmallTile * 8; ++i) R[i] = 0.f;
#define SACC(t, e) R[(t) * 8 + (e)]
#define ACC(q) (&R[(q) * 4])

        // ---- v for the expand: hi/lo operand (large tiles) or VF as is (small tiles)
        auto stage_v = [&](auto get) {
            if (small) {
                for (int i = tid; i < nt * r16; i += kCompute) {
                    const int row = i / r16, j = i - row * r16;
                    VF[row * p.rp + j] = j < r ? get(row, j) : 0.f;
                }
            } else {
                for (int i = tid; i < Mtr * r16; i += kCompute) {
                    const int row = i / r16, j = i - row * r16;
                    const float val = (j < r && row < nt) ? get(row, j) : 0.f;
                    const __nv_bfloat16 h = __float2bfloat16_rn(val);
                    const __nv_bfloat16 l = __float2bfloat16_rn(val - __bfloat162float(h));
                    Vh[row * vpitch + j] = *reinterpret_cast<const uint16_t*>(&h);
                    Vl[row * vpitch + j] = *reinterpret_cast<const uint16_t*>(&l);
                }
            }
            ptx::named_sync(1, kCompute);
        };

        // ---- partial v of this CTA -> VF, cluster exchange, v in VF (all rows)
        auto reduce_v = [&]() {
            if (small) {
                if constexpr (kSmallOnly) {
                    // each pair of a warp: a shuffle tree over the lanes, then lane 0 writes its 8 sums
#pragma unroll
                    for (int i = 0; i < kSmallTile * 8 / kComputeWarps; ++i) {
                        const int q = warp + kComputeWarps * i;
                        if (q >= nt * ncbp) break;  // uniform per warp
                        const int t = q >> lg, c = q & (ncbp - 1);
                        if (c >= ncb) continue;
                        for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
                            for (int e = 0; e < 8; ++e) SACC(i, e) += __shfl_xor_sync(0xffffffffu, SACC(i, e), off);
                        if (lane == 0) {
                            float4* dst = reinterpret_cast<float4*>(&VF[t * p.rp + c * 8]);
                            dst[0] = make_float4(SACC(i, 0), SACC(i, 1), SACC(i, 2), SACC(i, 3));
                            dst[1] = make_float4(SACC(i, 4), SACC(i, 5), SACC(i, 6), SACC(i, 7));
                        }
                    }
                } else {
                    // lanes sharing a chunk (lane % ncbp) reduce by shuffles, then warps through VF
                    for (int off = 16; off >= ncbp; off >>= 1)
#pragma unroll
                        for (int t = 0; t < kSmallTile; ++t)
                            if (t < nt)  // uniform
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    SACC(t, e) += __shfl_xor_sync(0xffffffffu, SACC(t, e), off);
                    if (lane < ncbp) {
#pragma unroll
                        for (int t = 0; t < kSmallTile; ++t)
#pragma unroll
                            for (int e = 0; e < 8; ++e) VF[((warp * ncbp + lane) * kSmallTile + t) * 8 + e] = SACC(t, e);
                    }
                    ptx::named_sync(1, kCompute);
                    // column j = c*8+e of token t: sum the slots of the threads that own chunk c
                    float part[2] = {0.f, 0.f};
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int idx = tid + h * kCompute;
                        if (idx < nt * r8) {
                            const int t = idx / r8, j = idx - t * r8, c = j >> 3, e = j & 7;
                            for (int w = 0; w < kComputeWarps; ++w)
                                part[h] += VF[((w * ncbp + c) * kSmallTile + t) * 8 + e];
                        }
                    }
                    ptx::named_sync(1, kCompute);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int idx = tid + h * kCompute;
                        if (idx < nt * r8) VF[(idx / r8) * p.rp + idx % r8] = part[h];
                    }
                }
            } else {
                const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int t = warp * tpw_s + q;
                    if (q < tpw_s && t < tiles_s) {
                        const int mt = t / nNT, ntl = t - mt * nNT;
                        const int row = mt * 16 + gq, col = ntl * 8 + tq * 2;
                        if (row < nt)
                            *reinterpret_cast<float2*>(&VF[row * p.rp + col]) = make_float2(ACC(q)[0], ACC(q)[1]);
                        if (row + 8 < nt)
                            *reinterpret_cast<float2*>(&VF[(row + 8) * p.rp + col]) =
                                make_float2(ACC(q)[2], ACC(q)[3]);
                    }
                }
            }
            ptx::named_sync(1, kCompute);
            ptx::cluster_wait();  // every CTA of the cluster has initialised its barriers
            // 16-byte pieces: 4 consecutive columns j of one row
            const int q8 = r8 >> 2;
            auto add4 = [](float4 a4, float4 b4) {
                return make_float4(a4.x + b4.x, a4.y + b4.y, a4.z + b4.z, a4.w + b4.w);
            };
            if (one_phase) {
                for (int i = tid; i < nt * q8; i += kCompute) {
                    const int row = i / q8, j = (i - row * q8) * 4;
                    const float4 val = *reinterpret_cast<const float4*>(&VF[row * p.rp + j]);
                    const uint32_t off = (uint32_t)(((rank * nt + row) * r8 + j) * 4);
                    for (int d = 0; d < C; ++d)
                        ptx::st_async_f32x4(ptx::mapa(rb_u + off, d), val, ptx::mapa(red1_u, d));
                }
            } else {
                for (int i = tid; i < nt * q8; i += kCompute) {
                    const int row = i / q8, j = (i - row * q8) * 4;
                    const uint32_t off = (uint32_t)(((rank * rows_per + row / C) * r8 + j) * 4);
                    ptx::st_async_f32x4(ptx::mapa(rb_u + off, row % C),
                                        *reinterpret_cast<const float4*>(&VF[row * p.rp + j]), ptx::mapa(red1_u, row % C));
                }
            }
            if (one_phase) ptx::cluster_arrive();  // phase 1: this thread's remote stores are issued
            wait_all<true, false>(red1, 0, abort_flag, status, 0x200, p.timeout_ns);
            ptx::named_sync(1, kCompute);  // every thread of this CTA has sent its share
            if (one_phase) {
                for (int i = tid; i < nt * q8; i += kCompute) {
                    const int row = i / q8, j = (i - row * q8) * 4;
                    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int c = 0; c < C; ++c)
                        s4 = add4(s4, *reinterpret_cast<const float4*>(&RB[(c * nt + row) * r8 + j]));
                    *reinterpret_cast<float4*>(&VF[row * p.rp + j]) = s4;
                }
            } else {
                // VF is written by the peers from here on; this CTA's partial was sent already
                for (int i = tid; i < mine * q8; i += kCompute) {
                    const int li = i / q8, j = (i - li * q8) * 4;
                    const int row = rank + li * C;
                    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int c = 0; c < C; ++c)
                        s4 = add4(s4, *reinterpret_cast<const float4*>(&RB[(c * rows_per + li) * r8 + j]));
                    const uint32_t off = (uint32_t)((row * p.rp + j) * 4);
                    for (int d = 0; d < C; ++d)
                        ptx::st_async_f32x4(ptx::mapa(vf_u + off, d), s4, ptx::mapa(red2_u, d));
                }
                ptx::cluster_arrive();  // phase 1: this thread's remote stores are issued
                wait_all<true, false>(red2, 0, abort_flag, status, 0x400, p.timeout_ns);
            }
            ptx::named_sync(1, kCompute);
            if (MODE == SGMV_SHRINK) {
                for (int i = tid; i < nt * p.r_max; i += kCompute) {
                    const int row = i / p.r_max, j = i - row * p.r_max;
                    if (row % C == rank)
                        p.v[((size_t)slice * p.T + s_tok[row]) * p.r_max + j] = j < r ? VF[row * p.rp + j] : 0.f;
                }
            } else if (!small) {
                stage_v([&](int row, int j) { return VF[row * p.rp + j]; });
            }
        };

        if (MODE == SGMV_EXPAND)
            stage_v([&](int row, int j) { return p.v[((size_t)slice * p.T + s_tok[row]) * p.r_max + j]; });

        // hoisted large-tile shrink addressing: warp tiles (mt, ntl)
        int l_mt[4], l_ntl[4];
        bool l_ok[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int t = warp * tpw_s + q;
            l_ok[q] = q < tpw_s && t < tiles_s;
            l_mt[q] = l_ok[q] ? t / nNT : 0;
            l_ntl[q] = l_ok[q] ? t - l_mt[q] * nNT : 0;
        }

        for (int it = 0; it < nK; ++it) {
            // -------------------------------------------------------- shrink k-block
            const int st = it % kStages;
            const uint32_t ph = (uint32_t)((it / kStages) & 1);
            const uint32_t base = base_u + st * SB;
            const bool ok = wait_all<false>(&full[st], ph, abort_flag, status, 0x800, p.timeout_ns) && !*abort_flag;
            const int k0 = k_begin + it * BK;
            const int kb = min(BK, k_begin + k_len - k0);
            const uint32_t xb = base + (uint32_t)(BK * apitch);
            if (ok && small) {
                if constexpr (kSmallOnly) {
                    // warp w owns the (token, 8-column chunk) pairs w, w + 8, ...: its lanes
                    // stride over the block's rows, so one shuffle tree finishes each pair
#pragma unroll
                    for (int i = 0; i < kSmallTile * 8 / kComputeWarps; ++i) {
                        const int q = warp + kComputeWarps * i;
                        if (q >= nt * ncbp) break;  // uniform per warp
                        const int t = q >> lg, c = q & (ncbp - 1);
                        if (c >= ncb) continue;
                        for (int k = lane; k < kb; k += 32) {
                            const uint4 av =
                                *reinterpret_cast<const uint4*>(smem + (base - base_u) + a_chunk(k, c, apitch, a_swz));
                            const float xv = __uint_as_float(
                                (uint32_t)(*reinterpret_cast<const uint16_t*>(smem + (xb - base_u) + t * xp + k * 2)) << 16);
                            const float af[8] = {bf16_lo(av.x), bf16_hi(av.x), bf16_lo(av.y), bf16_hi(av.y),
                                                 bf16_lo(av.z), bf16_hi(av.z), bf16_lo(av.w), bf16_hi(av.w)};
#pragma unroll
                            for (int e = 0; e < 8; ++e) SACC(i, e) = fmaf(xv, af[e], SACC(i, e));
                        }
                    }
                } else {
                    // thread owns 8 columns (chunk c_own) over rows k = rg, rg + rstride, ...
                    if (c_own < ncb) {
                        for (int k = rg; k < kb; k += rstride) {
                            const uint4 av =
                                *reinterpret_cast<const uint4*>(smem + (base - base_u) + a_chunk(k, c_own, apitch, a_swz));
                            const float af[8] = {bf16_lo(av.x), bf16_hi(av.x), bf16_lo(av.y), bf16_hi(av.y),
                                                 bf16_lo(av.z), bf16_hi(av.z), bf16_lo(av.w), bf16_hi(av.w)};
#pragma unroll
                            for (int t = 0; t < kSmallTile; ++t) {
                                if (t < nt) {
                                    const float xv = __uint_as_float(
                                        (uint32_t)(*reinterpret_cast<const uint16_t*>(smem + (xb - base_u) + t * xp + k * 2))
                                        << 16);
#pragma unroll
                                    for (int e = 0; e < 8; ++e) SACC(t, e) = fmaf(xv, af[e], SACC(t, e));
                                }
                            }
                        }
                    }
                }
            } else if (!small && (kb & 15)) {
                // last block of h_in: x columns kb..kb+8 may hold stale bytes; zero them (the
                // barrier does not depend on ok, so every compute thread meets it)
                if (ok && tid < nt)
                    *reinterpret_cast<uint4*>(smem + (xb - base_u) + blk_chunk(tid, kb >> 3, Mtr)) =
                        make_uint4(0, 0, 0, 0);
                ptx::fence_proxy_async_smem();  // generic writes to a stage that bulk copies refill
                ptx::named_sync(1, kCompute);
            }
            if (ok && !small) {
                const int ksteps = (kb + 15) >> 4;
                // x rows in swizzled 64-column blocks: row (l_mt*16 + lane%16), k chunk 2*ks + lane/16
                uint32_t xrow[4], aaddr[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    xrow[q] = xb + (uint32_t)((l_mt[q] * 16 + (lane & 15)) * 128);
                    aaddr[q] = base + a_chunk(lane & 15, l_ntl[q], apitch, a_swz);
                }
                const int xr7 = lane & 7, xhi = lane >> 4;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint32_t xoff =
                        (uint32_t)((ks >> 2) * Mtr * 128 + (((((ks & 3) << 1) | xhi) ^ xr7) << 4));
                    uint32_t af[4][4], bf[4][2];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (l_ok[q]) {
                            if (q == 0 || l_mt[q] != l_mt[q - 1])
                                ptx::ldsm_x4(xrow[q] + xoff, af[q][0], af[q][1], af[q][2], af[q][3]);
                            else
#pragma unroll
                                for (int e = 0; e < 4; ++e) af[q][e] = af[q - 1][e];
                            ptx::ldsm_x2_t(aaddr[q] + (uint32_t)(ks * 16 * apitch), bf[q][0], bf[q][1]);
                        }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (l_ok[q]) ptx::mma_bf16_16816(ACC(q), af[q], bf[q][0], bf[q][1]);
                }
            }
            ptx::named_sync(1, kCompute);
            if (tid == 0) ptx::mbar_arrive(&empty[st]);
        }
        if (MODE != SGMV_EXPAND) reduce_v();

        // tensor-core expand: warp w owns m-tile mt_w = w % Mt (rows mt_w*16 ..) and the
        // n-tiles ntl = w / Mt + k * nw_mt of every n-block; its V fragments (hi and lo,
        // all rank steps) are loaded once here and stay in registers for every n-block
        const int mt_w = warp % Mt;
        const int nw_mt = (kComputeWarps - mt_w + Mt - 1) / Mt;
        const int ntl0 = warp / Mt;
        const int ksteps_e = r16 >> 4;
        uint32_t vah[4][4], val[4][4];
        if (!small && nN > 0) {
            const uint32_t voff = (uint32_t)(((mt_w * 16 + (lane & 15)) * vpitch + (lane >> 4) * 8) * 2);
            const uint32_t vh_u = ptx::smem_u32(Vh), vl_u = ptx::smem_u32(Vl);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                if (ks < ksteps_e) {
                    ptx::ldsm_x4(vh_u + voff + ks * 32, vah[ks][0], vah[ks][1], vah[ks][2], vah[ks][3]);
                    ptx::ldsm_x4(vl_u + voff + ks * 32, val[ks][0], val[ks][1], val[ks][2], val[ks][3]);
                }
        }

        for (int it = nK; it < nItems; ++it) {
            // -------------------------------------------------------- expand n-block
            const int st = it % kStages;
            const uint32_t ph = (uint32_t)((it / kStages) & 1);
            const uint32_t base = base_u + st * SB;
            const bool ok = wait_all<false>(&full[st], ph, abort_flag, status, 0x800, p.timeout_ns) && !*abort_flag;
            const int n0 = n_begin + (it - nK) * BN;
            const int nb = min(BN, n_begin + n_len - n0);
            const uint32_t yb = base + y_off;
            if (ok && small) {
                // one column pair per thread: y[t][n..n+1] += s * sum_j v[t][j] * B[j][n..n+1]
                for (int pp = tid; pp < (nb >> 1); pp += kCompute) {
                    const int n = pp * 2;
                    float s0[kSmallTile], s1[kSmallTile];
#pragma unroll
                    for (int t = 0; t < kSmallTile; ++t) s0[t] = s1[t] = 0.f;
                    // B(j, n..n+1) in its box of kSmallBoxCols columns: rows of 2 kSmallBoxCols bytes
                    const uint8_t* bbox = smem + (base - base_u) + (n / kSmallBoxCols) * r16 * kSmallBoxCols * 2 +
                                          (n % kSmallBoxCols) * 2;
                    for (int j = 0; j < r; ++j) {
                        const uint32_t bw = *reinterpret_cast<const uint32_t*>(bbox + j * kSmallBoxCols * 2);
                        const float b0 = bf16_lo(bw), b1 = bf16_hi(bw);
#pragma unroll
                        for (int t = 0; t < kSmallTile; ++t)
                            if (t < nt) {
                                const float vv = VF[t * p.rp + j];
                                s0[t] = fmaf(vv, b0, s0[t]);
                                s1[t] = fmaf(vv, b1, s1[t]);
                            }
                    }
#pragma unroll
                    for (int t = 0; t < kSmallTile; ++t)
                        if (t < nt) {
                            const uint32_t yw = *reinterpret_cast<const uint32_t*>(smem + (yb - base_u) + t * bp + n * 2);
                            *reinterpret_cast<uint32_t*>(yg + (size_t)s_tok[t] * p.h_out + n0 + n) =
                                pack_bf16x2(bf16_lo(yw) + scale * s0[t], bf16_hi(yw) + scale * s1[t]);
                        }
                }
            } else if (!small) {
                if (r != r16) {  // B rows r..r16 of every box hold padding or nothing: zero them
                    const int zr = r16 - r, nbx = (nb + 63) >> 6;
                    for (int i = tid; ok && i < nbx * zr * 8; i += kCompute) {
                        const int bx = i / (zr * 8), rem = i - bx * zr * 8;
                        *reinterpret_cast<uint4*>(smem + (base - base_u) + bx * r16 * 128 + (r + (rem >> 3)) * 128 +
                                                  (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();  // generic writes to a stage that bulk copies refill
                    ptx::named_sync(1, kCompute);    // met by every compute thread, whatever ok
                }
                const int nNTe = ok ? (nb + 7) >> 3 : 0;
                const int gq = lane >> 2, tq = lane & 3;
                for (int ntl = ntl0; ntl < nNTe; ntl += nw_mt) {
                    // row j = ks*16 + (lane & 15) of box ntl/8, 16-byte chunk ntl%8 XOR (j & 7)
                    const uint32_t bbase = base + (uint32_t)((ntl >> 3) * r16 * 128 + (lane & 15) * 128 +
                                                             ((((ntl & 7) ^ (lane & 7))) << 4));
                    uint32_t b[4][2];
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        if (ks < ksteps_e) ptx::ldsm_x2_t(bbase + ks * 16 * 128, b[ks][0], b[ks][1]);
                    float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        if (ks < ksteps_e) {
                            ptx::mma_bf16_16816(c[0], vah[ks], b[ks][0], b[ks][1]);
                            ptx::mma_bf16_16816(c[1], val[ks], b[ks][0], b[ks][1]);
                        }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int rr = mt_w * 16 + gq + h * 8;
                        if (rr < nt) {
                            uint32_t* py =
                                reinterpret_cast<uint32_t*>(smem + (yb - base_u) + blk_chunk(rr, ntl, Mtr) + tq * 4);
                            const uint32_t yw = *py;
                            *py = pack_bf16x2(bf16_lo(yw) + scale * (c[0][h * 2] + c[1][h * 2]),
                                              bf16_hi(yw) + scale * (c[0][h * 2 + 1] + c[1][h * 2 + 1]));
                        }
                    }
                }
            }
            // large tiles: updated y rows -> global, 16 bytes per thread, coalesced (uniform branch)
            if (!small) {
                ptx::fence_proxy_async_smem();  // the RMW wrote a stage that bulk copies refill
                ptx::named_sync(1, kCompute);
                if (ok) {
                    const int nch = nb >> 3;
                    auto put = [&](int rr, int ch) {
                        *reinterpret_cast<uint4*>(yg + (size_t)s_tok[rr] * p.h_out + n0 + ch * 8) =
                            *reinterpret_cast<const uint4*>(smem + (yb - base_u) + blk_chunk(rr, ch, Mtr));
                    };
                    if ((nch & (nch - 1)) == 0 && nch <= 32) {
                        const int lg = __ffs(nch) - 1;
                        for (int rr = tid >> lg; rr < nt; rr += kCompute >> lg) put(rr, tid & (nch - 1));
                    } else {
                        for (int i = tid; i < nt * nch; i += kCompute) put(i / nch, i % nch);
                    }
                }
            }
            ptx::named_sync(1, kCompute);
            if (tid == 0) ptx::mbar_arrive(&empty[st]);
        }
    }
    // no CTA leaves while a peer may still address its shared memory
    if (kClustered) ptx::cluster_wait();
}
#undef SACC
#undef ACC

// The tile rows of a general batch in descending cost, so that the long rows start
// first and the grid has no tail of a few long CTAs: the tensor-core rows (more than
// kSmallTile tokens), then the small rows by descending rank (round_up(r, 8)), each
// class in table order (a stable counting sort, one CTA). Results do not depend on
// the order: every row writes only its own tokens' outputs. The unused rows keep
// their places after the last used one; above kOrderMax used rows the table is copied
// as it is.
constexpr int kOrderThreads = 1024;
constexpr int kOrderMax = kOrderThreads;
constexpr int kOrderClasses = 9;
__global__ void __launch_bounds__(kOrderThreads)
tile_order_kernel(const int4* tiles, const int32_t* counts, const int32_t* ranks, int r_max, int max_tiles, int4* out)
{
    __shared__ int s_cnt[kOrderClasses][kOrderThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    ptx::pdl_wait();  // the segment builder wrote the tile rows
    const int n = min(max(counts[3], 0), max_tiles);
    if (n > kOrderMax) {
        for (int i = tid; i < max_tiles; i += kOrderThreads) out[i] = tiles[i];
        ptx::pdl_launch_dependents();
        return;
    }
    const bool valid = tid < n;
    const int4 tl = valid ? tiles[tid] : make_int4(-1, 0, 0, -1);
    int key = kOrderClasses;  // none
    if (valid) {
        int r = ranks ? ranks[tl.x] : r_max;
        r = max(1, min(r, r_max));
        key = tl.z > kSmallTile ? 0 : 1 + (64 - ((r + 7) & ~7)) / 8;  // 0 .. 8
    }
    unsigned mine = 0;
    for (int c = 0; c < kOrderClasses; ++c) {
        const unsigned b = __ballot_sync(0xffffffffu, key == c);
        if (key == c) mine = b;
        if (lane == 0) s_cnt[c][warp] = __popc(b);
    }
    __syncthreads();
    if (tid == 0) {  // exclusive prefix in (class, warp) order
        int run = 0;
        for (int c = 0; c < kOrderClasses; ++c)
            for (int w = 0; w < kOrderThreads / 32; ++w) {
                const int v = s_cnt[c][w];
                s_cnt[c][w] = run;
                run += v;
            }
    }
    __syncthreads();
    if (valid) out[s_cnt[key][warp] + __popc(mine & ((1u << lane) - 1u))] = tl;
    for (int i = n + tid; i < max_tiles; i += kOrderThreads) out[i] = tiles[i];
    ptx::pdl_launch_dependents();
}

template <int MODE, bool kSmallOnly>
cudaError_t launch_mode(const AMaps& am, const SgmvParams& p, dim3 grid, int C, size_t smem, cudaStream_t stream)
{
    auto kern = sgmv_kernel<MODE, kSmallOnly>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (MODE != SGMV_EXPAND) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)C;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, am, p);
}

// Dynamic shared memory one CTA may take so that two fit on an SM (per device).
size_t sgmv_smem_per_cta()
{
    int dev = 0;
    cudaGetDevice(&dev);
    static size_t cached[64] = {0};
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
    cudaFuncAttributes fa;
    size_t stat = 1024;
    if (cudaFuncGetAttributes(&fa, sgmv_kernel<SGMV_APPLY, false>) == cudaSuccess) stat = fa.sharedSizeBytes;
    const size_t b = smem_two_per_sm(stat);
    if (dev >= 0 && dev < 64) cached[dev] = b;
    return b;
}

}  // namespace

size_t sgmv_order_bytes(int T, int n_adapters)
{
    return (size_t)max_tiles_for(T, n_adapters) * sizeof(int4);
}

cudaError_t launch_sgmv(int mode, const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                        const lora_segments_t& seg, float* v, void* y, cudaStream_t stream,
                        bool pdl_trigger, void* order)
{
    (void)pdl_trigger;
    if (seg.T == 0) return cudaSuccess;
    SgmvParams p = {};
    p.x = static_cast<const uint16_t*>(x);
    p.x_slice_stride = x_slice_stride;
    p.A = static_cast<const uint16_t*>(pool.A);
    p.B = static_cast<const uint16_t*>(pool.B);
    p.ranks = pool.ranks;
    p.scales = pool.scales;
    p.perm = seg.perm;
    p.tiles = reinterpret_cast<const int4*>(seg.tiles);
    p.counts = seg.counts;
    p.v = v;
    p.y = static_cast<uint16_t*>(y);
    p.T = seg.T;
    p.n_adapters = pool.n_adapters;
    p.h_in = pool.h_in;
    p.h_out = pool.h_out;
    p.r_max = pool.r_max;
    p.timeout_ns = debug_wait_limit_ns();
    p.inject_stall = debug_inject_stall();
    // CTAs per tile: up to one per 512 columns of h_in (at most 8). When that would
    // need more than one wave of two CTAs per SM but the tile rows alone fit in one,
    // take as many per tile as keep one wave (no near-empty last wave: prefill gets 5),
    // but not fewer than 2 (one CTA per row makes long chains); with more tile rows than
    // that (many tenants), 2 per tile, then 1 beyond eight waves
    int C = (pool.h_in + 511) / 512;
    C = C < 1 ? 1 : (C > kMaxCluster ? kMaxCluster : C);
    const long long rows = (long long)max_tiles_for(seg.T, pool.n_adapters) * pool.n_slices;
    const long long slots = 2LL * device_sm_count();
    if (rows * C > slots) {
        if (rows <= slots) {
            const int c1 = (int)(slots / rows), c2 = C < 2 ? C : 2;
            C = c1 > c2 ? c1 : c2;
        } else {
            C = C < 2 ? C : 2;
            if (rows * C > 8 * slots) C = 1;
        }
    }
    // the tile rows in cost order first (one small CTA, a programmatic dependent), when
    // their CTAs need more than one wave of two per SM (else the order cannot help)
    if (order && rows * C <= slots) order = nullptr;
    if (order) {
        const int mt = max_tiles_for(seg.T, pool.n_adapters);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1, 1, 1);
        cfg.blockDim = dim3(kOrderThreads, 1, 1);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, tile_order_kernel, p.tiles, (const int32_t*)seg.counts,
                                                 pool.ranks, pool.r_max, mt, static_cast<int4*>(order));
        if (e != cudaSuccess) return e;
        p.tiles = static_cast<const int4*>(order);
    }
    p.csize = C;
    p.kc = ((pool.h_in + C - 1) / C + 127) / 128 * 128;
    p.nc = ((pool.h_out + C - 1) / C + 63) / 64 * 64;
    p.rp = (pool.r_max + 15) / 16 * 16;

    // shared memory: ring | exchange buffer (aliased by the hi/lo operand) | v | barriers
    const size_t rows_per = (kTT + C - 1) / C;
    size_t rb = (size_t)C * rows_per * p.rp * 4;
    if (rb < (size_t)kOnePhaseBytes) rb = kOnePhaseBytes;
    const size_t hilo = (size_t)2 * kTT * (p.rp + 8) * 2;
    if (rb < hilo) rb = hilo;
    rb = (rb + 127) / 128 * 128;
    size_t vf = (size_t)kTT * p.rp * 4;
    const size_t partials = (size_t)kComputeWarps * 8 * kSmallTile * 8 * 4;  // small-tile warp partials
    if (vf < partials) vf = partials;
    // stages (multiples of 1024 bytes, at most 32 KB) sized so that two CTAs fit on an SM
    const size_t bars = 8 * (2 * kStages + 3);
    const size_t fixed = rb + vf + bars + 1024;  // + base alignment slack
    const size_t budget = sgmv_smem_per_cta();
    if (budget <= fixed + (size_t)kStages * 8192) return cudaErrorInvalidConfiguration;
    size_t sb = (budget - fixed) / kStages / 1024 * 1024;
    p.stage_bytes = (int)(sb > 32768 ? 32768 : sb);
    // a tensor-core tile (64 tokens, rank 64) needs 64-column blocks and 64-row k-blocks
    if (p.stage_bytes < 20480) return cudaErrorInvalidConfiguration;
    const size_t ring = (size_t)kStages * p.stage_bytes;
    p.off_rb = (uint32_t)ring;
    p.off_vf = (uint32_t)(ring + rb);
    p.off_bar = (uint32_t)(ring + rb + vf);
    const size_t smem = p.off_bar + bars + 1024;  // + base alignment slack

    AMaps am;
    if (!build_pool_maps(am, pool, mode != SGMV_EXPAND, mode != SGMV_SHRINK)) return cudaErrorInvalidValue;
    p.xy_maps = build_xy_maps(am, pool, seg.T, x, x_slice_stride, y, mode != SGMV_EXPAND, mode != SGMV_SHRINK) ? 1 : 0;

    p.n_slices = pool.n_slices;
    const dim3 grid((unsigned)((long long)max_tiles_for(seg.T, pool.n_adapters) * pool.n_slices * C), 1, 1);
    // segments of a decode-like batch come in tiles of <= kSmallTile tokens
    if (tile_tokens_for(seg.T, seg.n_adapters) <= kSmallTile) {
        switch (mode) {
        case SGMV_SHRINK: return launch_mode<SGMV_SHRINK, true>(am, p, grid, C, smem, stream);
        case SGMV_EXPAND: return launch_mode<SGMV_EXPAND, true>(am, p, grid, C, smem, stream);
        default: return launch_mode<SGMV_APPLY, true>(am, p, grid, C, smem, stream);
        }
    }
    switch (mode) {
    case SGMV_SHRINK: return launch_mode<SGMV_SHRINK, false>(am, p, grid, C, smem, stream);
    case SGMV_EXPAND: return launch_mode<SGMV_EXPAND, false>(am, p, grid, C, smem, stream);
    default: return launch_mode<SGMV_APPLY, false>(am, p, grid, C, smem, stream);
    }
}

}  // namespace lora
