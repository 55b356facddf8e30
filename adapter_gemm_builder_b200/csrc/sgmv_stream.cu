// sgmv_stream.cu -- the fused shrink + expand of SGMV (Punica README, "How?":
// y += s_a (x.A_a).B_a for every token, grouped by adapter into segments) for
// batches whose segments come in tiles of up to 64 tokens (many tenants,
// prefill), as a persistent grid that streams work items.
//
// Work items. Every tile row (one run of <= 64 tokens of one adapter, in one
// slice) is split into Pk shrink parts (spans of h_in) and Pn expand parts
// (spans of h_out). The call makes two launches of the kernel, each handing
// its items out from a global counter: the first runs every shrink part, which
// computes its span's partial v = x.A_a for the tile's tokens and adds it into
// a v buffer in the workspace (plain stores when Pk == 1); the second, a
// programmatic dependent of the first, runs every expand part: its copies of
// B_a and y start while the first launch finishes, and its compute warps wait
// for the first launch to complete before they read v.
//
// Pipeline. A producer warp claims items, cuts them into chunks of columns
// sized to one ring stage (wider chunks for small ranks and few tokens) and
// fills a ring of 3 stages: the rows of A_a (or B_a) by tensor-map boxes of
// the adapter's live columns, and the tile's x (or y) rows gathered with
// 16-byte cp.async, or by tensor-map boxes when the tokens are consecutive
// rows. Each stage carries a header (item, chunk, tokens) for the compute
// warps, so the next chunks' copies -- of the same item or of the next one --
// are in flight while the compute warps work on the current chunk. Two CTAs
// share an SM.
//
// Math, as in the cluster kernel: tiles of <= 4 tokens on CUDA cores, larger
// ones with bf16 mma.sync (fp32 accumulate); the expand operand v is split
// into bf16 hi + lo halves (~16 bits of v).
//
// Every wait is bounded; on expiry the kernel records a status word in
// lora_segments_t.counts, drains the copies it issued and leaves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"
#include "sgmv_common.cuh"

namespace lora {
namespace {

constexpr int kMaxChunk = 1024;  // widest chunk of columns

struct StreamParams {
    const uint16_t* x;
    long long x_slice_stride;
    const uint16_t* A;
    const uint16_t* B;
    const int32_t* ranks;
    const float* scales;
    const int32_t* perm;
    const int4* tiles;
    int32_t* counts;
    uint16_t* y;
    float* vbuf;  // fp32 [n_slices][T][r_max]
    int* ctr;     // [phase]: the next item of this launch
    int phase;    // 0: the shrink parts; 1: the expand parts (a programmatic dependent of 0)
    int T, n_adapters, h_in, h_out, r_max, n_slices, n_rows;
    int Pk, Pn, kp, np;  // parts per tile row and their spans (multiples of 64)
    int stage_bytes;
    int xy_maps;
    uint32_t off_vf, off_bar;
    unsigned long long timeout_ns;
    int inject_stall;
};

// What a ring stage holds, written by the producer before it arrives on the
// stage's barrier.
struct __align__(16) StageHdr {
    int kind;  // 0 shrink chunk, 1 expand chunk, 2 end of work
    int slice, g, a;
    int nt, r, a_map, wb;  // tokens, rank, A map (log2 of box width / 8), allocated width
    int c0, cw, first, last;  // first column and width of the chunk; first / last of its item
    float scale;
    int pad[3];
    int tok[kTT];
};

enum { kShrinkChunk = 0, kExpandChunk = 1, kEnd = 2 };

// Columns per chunk: the widest power of two times 64 (<= 1024) whose rows of
// `per_col` bytes fit a stage.
__device__ __forceinline__ int chunk_width(int per_col, int sb)
{
    int w = kMaxChunk;
    while (w > 64 && w * per_col > sb) w >>= 1;
    return w;
}

__global__ void __launch_bounds__(kThreads, 2)
sgmv_stream_kernel(const __grid_constant__ AMaps am, const StreamParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ StageHdr s_hdr[kStages];
    __shared__ int s_abort;

    const uint32_t raw_u = ptx::smem_u32(smem_raw);
    const uint32_t base_u = (raw_u + 1023u) & ~1023u;  // swizzled boxes need 1024-byte alignment
    uint8_t* smem = smem_raw + (base_u - raw_u);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int SB = p.stage_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
    uint64_t* empty = full + kStages;
    uint64_t* stall = empty + kStages;  // test hook: never completed
    volatile int* abort_flag = &s_abort;
    int32_t* status = p.counts + kSegStatusSlot;

    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 33);  // lane 0's expect_tx + one arrival per producer lane
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(stall, 1);
        ptx::fence_mbar_init();
    }
    __syncwarp();
    __syncthreads();
    // Shrink launch: the segment builder (the previous kernel in the stream) may still
    // run; the expand launch may start as soon as this one has passed this point. Expand
    // launch: its copies (B_a and y, which the shrink does not write) start at once; the
    // compute warps wait for the shrink launch to complete before they read v.
    if (p.phase == 0) ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    bool v_ready = p.phase == 0;

    if (warp == kComputeWarps) {
        // ================================================================ producer warp
        int st = 0;
        uint32_t ph = 0;
        long long issued = 0;
        bool ok = true;
        if (p.inject_stall && blockIdx.x == 0)
            ok = wait_all<false>(stall, 0, abort_flag, status, 0x2000, p.timeout_ns);
        if (lane == 0) {
            for (int i = 0; i < 4; ++i)
                if ((8 << i) <= p.r_max) ptx::tma_prefetch_desc(&am.m[i]);
            for (int i = 0; i < 4 && 16 * i < p.r_max; ++i) ptx::tma_prefetch_desc(&am.b[i]);
        }
        // Items are enumerated over the tile rows in use (the segment builder's count).
        // The producer's per-item metadata is a chain of dependent loads (claim -> tile
        // row -> rank, scale, token ids); it is software-pipelined so that each link is
        // consumed one item after it was issued, while the current item's copies go out:
        // claims run two items ahead, tile rows one item ahead.
        const long long used = p.counts[3];
        const long long n_shrink = p.phase == 0 ? used * p.n_slices * p.Pk : 0;
        const long long n_items = p.phase == 0 ? n_shrink : used * p.n_slices * p.Pn;
        struct Meta {
            long long item;
            int shrink, slice, g, part;
            int4 tl;
            int r, t_lo, t_hi;
            float scale;
        };
        auto decode = [&](long long item, Meta& m) {  // issues the tile-row load
            m.item = item;
            if (item >= n_items) return;
            m.shrink = item < n_shrink;
            long long rem = m.shrink ? item : item - n_shrink;
            const int P = m.shrink ? p.Pk : p.Pn;
            const long long per_slice = used * P;
            m.slice = (int)(rem / per_slice);
            rem -= (long long)m.slice * per_slice;
            m.g = (int)(rem / P);
            m.part = (int)(rem - (long long)m.g * P);
            m.tl = p.tiles[m.g];
        };
        auto resolve = [&](Meta& m) {  // issues the loads that need the tile row
            if (m.item >= n_items) return;
            const int a = m.tl.x, nt = m.tl.z;
            m.r = p.ranks ? p.ranks[a] : p.r_max;
            m.scale = p.scales ? p.scales[a] : 1.0f;
            m.t_lo = lane < nt ? p.perm[m.tl.y + lane] : 0;
            m.t_hi = lane + 32 < nt ? p.perm[m.tl.y + lane + 32] : 0;
        };
        long long claim = 0;
        Meta m0, m1;
        if (lane == 0) claim = (long long)atomicAdd(p.ctr + p.phase, 1);
        decode(__shfl_sync(0xffffffffu, claim, 0), m0);
        if (lane == 0) claim = (long long)atomicAdd(p.ctr + p.phase, 1);
        decode(__shfl_sync(0xffffffffu, claim, 0), m1);
        if (lane == 0 && m1.item < n_items) claim = (long long)atomicAdd(p.ctr + p.phase, 1);
        resolve(m0);
        while (ok && m0.item < n_items) {
            resolve(m1);
            Meta m2;
            m2.item = n_items;
            if (m1.item < n_items) {
                decode(__shfl_sync(0xffffffffu, claim, 0), m2);
                if (lane == 0 && m2.item < n_items) claim = (long long)atomicAdd(p.ctr + p.phase, 1);
            }
            const bool shrink = m0.shrink;
            const int slice = m0.slice, g = m0.g, part = m0.part;
            const int nt = m0.tl.z;
            const int a = m0.tl.x;
            const int r = max(1, min(m0.r, p.r_max));
            const float scale = m0.scale;
            const int t_lo = m0.t_lo, t_hi = m0.t_hi;
            m0 = m1;
            m1 = m2;
            const bool small = nt <= kSmallTile;
            const int Mt = (nt + 15) >> 4;
            const int Mtr = small ? nt : Mt * 16;
            const int r8 = round_up(r, 8), r16 = round_up(r, 16);
            const int a_map = r8 <= 8 ? 0 : 32 - __clz((r8 >> 3) - 1);
            const int rA = 8 << a_map;
            const int rB = min(r16, p.r_max);
            // consecutive token rows (a pre-sorted batch): x / y rows as tensor-map boxes
            const int t_first = __shfl_sync(0xffffffffu, t_lo, 0);
            bool contig = false;
            if (!small && p.xy_maps)
                contig = __all_sync(0xffffffffu, (lane >= nt || t_lo == t_first + lane) &&
                                                     (lane + 32 >= nt || t_hi == t_first + lane + 32));
            const int span = shrink ? p.kp : p.np;
            const int lim = shrink ? p.h_in : p.h_out;
            const int c_begin = part * span, c_end = min(lim, c_begin + span);
            const int wb = shrink ? chunk_width(rA * 2 + Mtr * 2, SB) : chunk_width(r16 * 2 + Mtr * 2, SB);
            const int n_chunks = (c_end - c_begin + wb - 1) / wb;
            const size_t sa = (size_t)slice * p.n_adapters + a;
            const uint16_t* xg = p.x + (size_t)slice * p.x_slice_stride;
            const uint16_t* yg = p.y + (size_t)slice * p.T * p.h_out;
            const int xs = p.x_slice_stride ? slice : 0;
            for (int c = 0; c < n_chunks; ++c) {
                if (!wait_all<false>(&empty[st], ph ^ 1, abort_flag, status, 0x100, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t base = base_u + (uint32_t)(st * SB);
                const int c0 = c_begin + c * wb;
                const int cw = min(wb, c_end - c0);
                const int nbox = (cw + 63) >> 6;
                StageHdr& h = s_hdr[st];
                if (lane == 0) {
                    h.kind = shrink ? kShrinkChunk : kExpandChunk;
                    h.slice = slice;
                    h.g = g;
                    h.a = a;
                    h.nt = nt;
                    h.r = r;
                    h.a_map = a_map;
                    h.wb = wb;
                    h.c0 = c0;
                    h.cw = cw;
                    h.first = c == 0;
                    h.last = c == n_chunks - 1;
                    h.scale = scale;
                }
                h.tok[lane] = t_lo;
                h.tok[lane + 32] = t_hi;
                // lane 0 announces the stage's tensor-map bytes before any lane issues a copy;
                // every lane then arrives once its own cp.async copies have landed
                uint32_t bytes;
                if (shrink) bytes = (uint32_t)(nbox * 64 * rA * 2);
                else bytes = (uint32_t)(nbox * 64 * rB * 2);
                if (contig) bytes += (uint32_t)(nbox * Mt * 2048);
                if (lane == 0) ptx::mbar_arrive_expect_tx(&full[st], bytes);
                __syncwarp();
                if (shrink) {
                    const uint32_t xb = base + (uint32_t)(wb * rA * 2);
                    if (lane < nbox)
                        ptx::tma_load_3d(base + (uint32_t)(lane * 64 * rA * 2), &am.m[a_map], &full[st], 0,
                                         c0 + lane * 64, (int)sa);
                    if (contig) {
                        for (int i = lane - nbox; i < nbox * Mt; i += 32)
                            if (i >= 0)
                                ptx::tma_load_3d(xb + (uint32_t)(((i / Mt) * Mtr + (i % Mt) * 16) * 128), &am.x,
                                                 &full[st], c0 + (i / Mt) * 64, t_first + (i % Mt) * 16, xs);
                    } else {
                        // 16-byte chunks (cw / 8 per row) of the tile's x rows, all lanes
                        const int cpr = cw >> 3;
                        for (int i = lane; i < nt * cpr; i += 32) {
                            const int row = i / cpr, cc = i - row * cpr;
                            ptx::cp_async16(xb + blk_chunk(row, cc, Mtr), xg + (size_t)h.tok[row] * p.h_in + c0 + cc * 8, 16);
                        }
                    }
                } else {
                    const uint32_t yb = base + (uint32_t)((wb >> 6) * r16 * 128);
                    if (lane < nbox)
                        ptx::tma_load_3d(base + (uint32_t)(lane * r16 * 128), &am.b[(r16 >> 4) - 1], &full[st],
                                         c0 + lane * 64, 0, (int)sa);
                    if (contig) {
                        for (int i = lane - nbox; i < nbox * Mt; i += 32)
                            if (i >= 0)
                                ptx::tma_load_3d(yb + (uint32_t)(((i / Mt) * Mtr + (i % Mt) * 16) * 128), &am.y,
                                                 &full[st], c0 + (i / Mt) * 64, t_first + (i % Mt) * 16, slice);
                    } else {
                        const int cpr = cw >> 3;
                        for (int i = lane; i < nt * cpr; i += 32) {
                            const int row = i / cpr, cc = i - row * cpr;
                            ptx::cp_async16(yb + blk_chunk(row, cc, Mtr), yg + (size_t)h.tok[row] * p.h_out + c0 + cc * 8, 16);
                        }
                    }
                }
                ptx::cp_async_arrive_noinc(&full[st]);
                ++issued;
                if (++st == kStages) {
                    st = 0;
                    ph ^= 1;
                }
            }
        }
        if (ok) {  // the end marker, in the next stage
            if (wait_all<false>(&empty[st], ph ^ 1, abort_flag, status, 0x100, p.timeout_ns)) {
                if (lane == 0) {
                    s_hdr[st].kind = kEnd;
                    ptx::mbar_arrive_expect_tx(&full[st], 0u);
                }
                __syncwarp();
                ptx::cp_async_arrive_noinc(&full[st]);
            }
        }
        ptx::cp_async_commit();
        ptx::cp_async_wait<0>();
        if (lane == 0 && *abort_flag) {  // let the copies that were issued land before leaving
            const unsigned long long t0 = ptx::globaltimer();
            const long long from = issued > kStages ? issued - kStages : 0;
            for (long long it = from; it < issued; ++it)
                while (!ptx::mbar_try_wait(&full[it % kStages], (uint32_t)((it / kStages) & 1)) &&
                       ptx::globaltimer() - t0 < kTimeoutNs) {
                }
        }
        __syncwarp();
    } else {
        // ================================================================ compute warps
        float* VF = reinterpret_cast<float*>(smem + p.off_vf);  // small tiles: warp partials / v rows
        // One register file for the state a consumer keeps across the chunks of an item:
        // a shrink's accumulators (small tiles: SACC(t, e); large: ACC(q), 4 MMA tiles) or,
        // for a large tile's expand, the bf16 hi / lo fragments of v (VAH(ks, i), VAL(ks, i)).
        float R[kSmallTile * 8];
#pragma unroll
        for (int i = 0; i < kSmallTile * 8; ++i) R[i] = 0.f;
#define SACC(t, e) R[(t) * 8 + (e)]
#define ACC(q) (&R[(q) * 4])
#define VAH(ks, i) R[(ks) * 4 + (i)]
#define VAL(ks, i) R[16 + (ks) * 4 + (i)]
        int st = 0;
        uint32_t ph = 0;
        while (true) {
            // every compute thread takes the same decision to leave (they meet in named barriers)
            const bool got = wait_all<false>(&full[st], ph, abort_flag, status, 0x800, p.timeout_ns);
            if (ptx::named_sync_or(2, kCompute, !got || *abort_flag)) break;
            const StageHdr& h = s_hdr[st];
            const int kind = h.kind;
            if (kind == kEnd) break;
            const int slice = h.slice, nt = h.nt, r = h.r, wb = h.wb, c0 = h.c0, cw = h.cw;
            const bool first = h.first, last = h.last;
            const bool small = nt <= kSmallTile;
            const int Mt = (nt + 15) >> 4;
            const int Mtr = small ? nt : Mt * 16;
            const int r8 = round_up(r, 8), r16 = round_up(r, 16);
            const int rA = 8 << h.a_map;
            const int apitch = rA * 2;
            const int a_swz = rA >= 16 ? (rA >> 3) - 1 : 0;
            const uint32_t base = base_u + (uint32_t)(st * SB);
            float* vrow = p.vbuf + (size_t)slice * p.T * p.r_max;
            // small tiles: thread (c_own, rg) owns 8-column chunk c_own of v over rows rg, rg + rstride, ...
            const int ncb = r8 >> 3;
            const int lg = ncb <= 1 ? 0 : (ncb <= 2 ? 1 : (ncb <= 4 ? 2 : 3));
            const int ncbp = 1 << lg;
            const int c_own = tid & (ncbp - 1), rg = tid >> lg, rstride = kCompute >> lg;
            // large tiles: warp w owns MMA tiles [w * tpw, (w + 1) * tpw) of the (Mt x r8 / 8) grid
            const int nNT = r8 >> 3;
            const int tiles_s = Mt * nNT;
            const int tpw_s = (tiles_s + kComputeWarps - 1) / kComputeWarps;
            bool live = true;

            if (kind == kShrinkChunk) {
                // ---------------------------------------------------------- shrink chunk
                if (first) {
#pragma unroll
                    for (int i = 0; i < kSmallTile * 8; ++i) R[i] = 0.f;
                }
                const uint32_t xb = base + (uint32_t)(wb * apitch);
                if (small) {
                    if (c_own < ncb) {
                        for (int k = rg; k < cw; k += rstride) {
                            const uint4 av = *reinterpret_cast<const uint4*>(smem + (base - base_u) +
                                                                               a_chunk(k, c_own, apitch, a_swz));
                            const float af[8] = {bf16_lo(av.x), bf16_hi(av.x), bf16_lo(av.y), bf16_hi(av.y),
                                                 bf16_lo(av.z), bf16_hi(av.z), bf16_lo(av.w), bf16_hi(av.w)};
#pragma unroll
                            for (int t = 0; t < kSmallTile; ++t) {
                                if (t < nt) {
                                    const float xv = __uint_as_float(
                                        (uint32_t)(*reinterpret_cast<const uint16_t*>(
                                            smem + (xb - base_u) + blk_chunk(t, k >> 3, Mtr) + (k & 7) * 2))
                                        << 16);
#pragma unroll
                                    for (int e = 0; e < 8; ++e) SACC(t, e) = fmaf(xv, af[e], SACC(t, e));
                                }
                            }
                        }
                    }
                } else {
                    const int ksteps = (cw + 15) >> 4;
                    if (cw & 15) {  // x columns cw..cw+8 of the last k-step hold stale bytes: zero them
                        if (tid < nt)
                            *reinterpret_cast<uint4*>(smem + (xb - base_u) + blk_chunk(tid, cw >> 3, Mtr)) =
                                make_uint4(0, 0, 0, 0);
                        ptx::fence_proxy_async_smem();  // generic writes to a stage that copies refill
                        ptx::named_sync(1, kCompute);
                    }
                    uint32_t xrow[4], aaddr[4];
                    int l_mt[4], l_ntl[4];
                    bool l_ok[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int t = warp * tpw_s + q;
                        l_ok[q] = q < tpw_s && t < tiles_s;
                        l_mt[q] = l_ok[q] ? t / nNT : 0;
                        l_ntl[q] = l_ok[q] ? t - l_mt[q] * nNT : 0;
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
                if (last) {
                    // this part's v for the tile's tokens -> the v buffer (added when several
                    // parts share the tile), then the part is counted done
                    const bool add = p.Pk > 1;
                    if (small) {
                        for (int off = 16; off >= ncbp; off >>= 1)
#pragma unroll
                            for (int t = 0; t < kSmallTile; ++t)
                                if (t < nt)
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
                        for (int idx = tid; idx < nt * r8; idx += kCompute) {
                            const int t = idx / r8, j = idx - t * r8, c = j >> 3, e = j & 7;
                            if (j >= r) continue;
                            float sum = 0.f;
                            for (int w = 0; w < kComputeWarps; ++w) sum += VF[((w * ncbp + c) * kSmallTile + t) * 8 + e];
                            float* dst = vrow + (size_t)h.tok[t] * p.r_max + j;
                            if (add) atomicAdd(dst, sum);
                            else *dst = sum;
                        }
                    } else {
                        const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int t = warp * tpw_s + q;
                            if (q < tpw_s && t < tiles_s) {
                                const int mt = t / nNT, ntl = t - mt * nNT;
                                const int col = ntl * 8 + tq * 2;
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const int row = mt * 16 + gq + hh * 8;
                                    if (row >= nt) continue;
                                    float* dst = vrow + (size_t)h.tok[row] * p.r_max + col;
                                    const float v0 = ACC(q)[2 * hh], v1 = ACC(q)[2 * hh + 1];
                                    if (col + 1 < r) {
                                        if (add) atomicAdd(reinterpret_cast<float2*>(dst), make_float2(v0, v1));
                                        else *reinterpret_cast<float2*>(dst) = make_float2(v0, v1);
                                    } else if (col < r) {
                                        if (add) atomicAdd(dst, v0);
                                        else *dst = v0;
                                    }
                                }
                            }
                        }
                    }
                    ptx::named_sync(1, kCompute);
                }
            } else {
                // ---------------------------------------------------------- expand chunk
                const float scale = h.scale;
                if (first) {
                    // the shrink launch has completed: v of every token is in the buffer
                    if (!v_ready) {
                        ptx::pdl_wait();
                        v_ready = true;
                    }
                    if (live) {
                        if (small) {
                            for (int idx = tid; idx < nt * r16; idx += kCompute) {
                                const int t = idx / r16, j = idx - t * r16;
                                VF[t * 64 + j] = j < r ? __ldcg(vrow + (size_t)h.tok[t] * p.r_max + j) : 0.f;
                            }
                        } else {
                            // mma.sync A fragments of v (rows = tokens of this warp's m-tile,
                            // columns = rank), split into bf16 hi + lo
                            const int mt_w = warp % Mt;
                            const int gq = lane >> 2, tq = lane & 3;
                            const int row0 = mt_w * 16 + gq, row1 = row0 + 8;
                            const float* v0p = row0 < nt ? vrow + (size_t)h.tok[row0] * p.r_max : nullptr;
                            const float* v1p = row1 < nt ? vrow + (size_t)h.tok[row1] * p.r_max : nullptr;
                            auto ld2 = [&](const float* rp, int j) -> float2 {
                                if (!rp || j >= r) return make_float2(0.f, 0.f);
                                float2 f = __ldcg(reinterpret_cast<const float2*>(rp + j));
                                if (j + 1 >= r) f.y = 0.f;
                                return f;
                            };
                            auto split = [](float2 f, float& hi, float& lo) {
                                const __nv_bfloat162 hh = __floats2bfloat162_rn(f.x, f.y);
                                const float2 hf = __bfloat1622float2(hh);
                                const __nv_bfloat162 ll = __floats2bfloat162_rn(f.x - hf.x, f.y - hf.y);
                                hi = __uint_as_float(*reinterpret_cast<const uint32_t*>(&hh));
                                lo = __uint_as_float(*reinterpret_cast<const uint32_t*>(&ll));
                            };
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks) {
                                if (ks * 16 < r16) {
                                    const int j0 = ks * 16 + tq * 2;
                                    split(ld2(v0p, j0), VAH(ks, 0), VAL(ks, 0));
                                    split(ld2(v1p, j0), VAH(ks, 1), VAL(ks, 1));
                                    split(ld2(v0p, j0 + 8), VAH(ks, 2), VAL(ks, 2));
                                    split(ld2(v1p, j0 + 8), VAH(ks, 3), VAL(ks, 3));
                                }
                            }
                        }
                    }
                    ptx::named_sync(1, kCompute);
                }
                const uint32_t yb = base + (uint32_t)((wb >> 6) * r16 * 128);
                uint16_t* yg = p.y + (size_t)slice * p.T * p.h_out;
                if (live && small) {
                    // four lanes per column pair, each over every fourth rank index j (its
                    // loads unrolled by two), then a two-step shuffle sum:
                    // y[t][n..n+1] += s * sum_j v[t][j] * B[j][n..n+1]
                    const int jq = tid & 3;
                    const int npairs = cw >> 1;
                    for (int pb = 0; pb < npairs; pb += kCompute / 4) {  // uniform trip count
                        const int pp = pb + (tid >> 2);
                        const bool on = pp < npairs;
                        const int n = on ? pp * 2 : 0;
                        float s0[kSmallTile], s1[kSmallTile];
#pragma unroll
                        for (int t = 0; t < kSmallTile; ++t) s0[t] = s1[t] = 0.f;
                        const uint8_t* bcol = smem + (base - base_u) + (n >> 6) * r16 * 128 + (n & 7) * 2;
                        const int nc = (n >> 3) & 7;
                        for (int j = jq; j < r; j += 8) {
                            const uint32_t bw0 = *reinterpret_cast<const uint32_t*>(bcol + j * 128 + ((nc ^ (j & 7)) << 4));
                            const int j1 = j + 4;
                            const uint32_t bw1 = j1 < r ? *reinterpret_cast<const uint32_t*>(
                                                              bcol + j1 * 128 + ((nc ^ (j1 & 7)) << 4))
                                                        : 0u;
#pragma unroll
                            for (int t = 0; t < kSmallTile; ++t)
                                if (t < nt) {
                                    const float v0 = VF[t * 64 + j], v1 = j1 < r ? VF[t * 64 + j1] : 0.f;
                                    s0[t] = fmaf(v0, bf16_lo(bw0), fmaf(v1, bf16_lo(bw1), s0[t]));
                                    s1[t] = fmaf(v0, bf16_hi(bw0), fmaf(v1, bf16_hi(bw1), s1[t]));
                                }
                        }
#pragma unroll
                        for (int t = 0; t < kSmallTile; ++t) {
                            s0[t] += __shfl_xor_sync(0xffffffffu, s0[t], 1);
                            s1[t] += __shfl_xor_sync(0xffffffffu, s1[t], 1);
                            s0[t] += __shfl_xor_sync(0xffffffffu, s0[t], 2);
                            s1[t] += __shfl_xor_sync(0xffffffffu, s1[t], 2);
                        }
                        if (on && jq < nt) {  // lane jq of the four stores token jq
#pragma unroll
                            for (int t = 0; t < kSmallTile; ++t)
                                if (t == jq) {
                                    const uint32_t yw = *reinterpret_cast<const uint32_t*>(
                                        smem + (yb - base_u) + blk_chunk(t, n >> 3, Mtr) + (n & 7) * 2);
                                    *reinterpret_cast<uint32_t*>(yg + (size_t)h.tok[t] * p.h_out + c0 + n) =
                                        pack_bf16x2(bf16_lo(yw) + scale * s0[t], bf16_hi(yw) + scale * s1[t]);
                                }
                        }
                    }
                } else if (live) {
                    if (r != r16) {  // B rows r..r16 of every box hold padding or nothing: zero them
                        const int zr = r16 - r, nbx = (cw + 63) >> 6;
                        for (int i = tid; i < nbx * zr * 8; i += kCompute) {
                            const int bx = i / (zr * 8), rr = i - bx * zr * 8;
                            *reinterpret_cast<uint4*>(smem + (base - base_u) + bx * r16 * 128 + (r + (rr >> 3)) * 128 +
                                                      (rr & 7) * 16) = make_uint4(0, 0, 0, 0);
                        }
                        ptx::fence_proxy_async_smem();
                        ptx::named_sync(1, kCompute);
                    }
                    const int mt_w = warp % Mt;
                    const int nw_mt = (kComputeWarps - mt_w + Mt - 1) / Mt;
                    const int ntl0 = warp / Mt;
                    const int ksteps_e = r16 >> 4;
                    const int nNTe = (cw + 7) >> 3;
                    const int gq = lane >> 2, tq = lane & 3;
                    for (int ntl = ntl0; ntl < nNTe; ntl += nw_mt) {
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
                                const uint32_t ah[4] = {__float_as_uint(VAH(ks, 0)), __float_as_uint(VAH(ks, 1)),
                                                        __float_as_uint(VAH(ks, 2)), __float_as_uint(VAH(ks, 3))};
                                const uint32_t al[4] = {__float_as_uint(VAL(ks, 0)), __float_as_uint(VAL(ks, 1)),
                                                        __float_as_uint(VAL(ks, 2)), __float_as_uint(VAL(ks, 3))};
                                ptx::mma_bf16_16816(c[0], ah, b[ks][0], b[ks][1]);
                                ptx::mma_bf16_16816(c[1], al, b[ks][0], b[ks][1]);
                            }
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int rr = mt_w * 16 + gq + hh * 8;
                            if (rr < nt) {
                                uint32_t* py =
                                    reinterpret_cast<uint32_t*>(smem + (yb - base_u) + blk_chunk(rr, ntl, Mtr) + tq * 4);
                                const uint32_t yw = *py;
                                *py = pack_bf16x2(bf16_lo(yw) + scale * (c[0][hh * 2] + c[1][hh * 2]),
                                                  bf16_hi(yw) + scale * (c[0][hh * 2 + 1] + c[1][hh * 2 + 1]));
                            }
                        }
                    }
                    ptx::fence_proxy_async_smem();  // the RMW wrote a stage that copies refill
                    ptx::named_sync(1, kCompute);
                    // updated y rows -> global, 16 bytes per thread, coalesced
                    const int nch = cw >> 3;
                    for (int i = tid; i < nt * nch; i += kCompute) {
                        const int rr = i / nch, ch = i - rr * nch;
                        *reinterpret_cast<uint4*>(yg + (size_t)h.tok[rr] * p.h_out + c0 + ch * 8) =
                            *reinterpret_cast<const uint4*>(smem + (yb - base_u) + blk_chunk(rr, ch, Mtr));
                    }
                }
            }
            ptx::named_sync(1, kCompute);
            if (tid == 0) ptx::mbar_arrive(&empty[st]);
            if (++st == kStages) {
                st = 0;
                ph ^= 1;
            }
        }
#undef SACC
#undef ACC
#undef VAH
#undef VAL
    }
}

}  // namespace

size_t sgmv_stream_workspace_bytes(int T, const lora_pool_t& pool)
{
    const size_t v = (size_t)pool.n_slices * T * pool.r_max * 4;
    return 256 + (v + 255) / 256 * 256;  // the two item counters | v
}

cudaError_t launch_sgmv_stream(const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                               const lora_segments_t& seg, void* y, void* ws, cudaStream_t stream)
{
    if (seg.T == 0) return cudaSuccess;
    StreamParams p = {};
    p.x = static_cast<const uint16_t*>(x);
    p.x_slice_stride = x_slice_stride;
    p.A = static_cast<const uint16_t*>(pool.A);
    p.B = static_cast<const uint16_t*>(pool.B);
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
    p.n_rows = max_tiles_for(seg.T, pool.n_adapters);
    p.timeout_ns = debug_wait_limit_ns();
    p.inject_stall = debug_inject_stall();

    // Parts per tile row: about three shrink and three expand items per CTA of the
    // grid, counted on an estimate of the tile rows in use (at most the bound, and
    // at most one row per 4 tokens: many adapters hold only a few tokens each).
    const int sms = device_sm_count();
    const long long G = 2LL * sms;
    const long long rows = (long long)p.n_rows * pool.n_slices;
    const long long rows_est = (long long)min(p.n_rows, (seg.T + 3) / 4) * pool.n_slices;
    long long P = (3 * G + rows_est - 1) / rows_est;
    P = P < 1 ? 1 : (P > 16 ? 16 : P);
    auto span = [&](int h) { return (int)(((h + P - 1) / P + 63) / 64 * 64); };
    p.kp = span(pool.h_in);
    p.np = span(pool.h_out);
    p.Pk = (pool.h_in + p.kp - 1) / p.kp;
    p.Pn = (pool.h_out + p.np - 1) / p.np;

    uint8_t* w = static_cast<uint8_t*>(ws);
    const size_t ctr_bytes = 256;
    p.ctr = reinterpret_cast<int*>(w);
    p.vbuf = reinterpret_cast<float*>(w + ctr_bytes);
    const size_t v_bytes = (size_t)pool.n_slices * seg.T * pool.r_max * 4;
    // the item counters start at zero; so does v when several parts add into it
    cudaError_t e = cudaMemsetAsync(w, 0, p.Pk > 1 ? ctr_bytes + v_bytes : ctr_bytes, stream);
    if (e != cudaSuccess) return e;

    // shared memory: ring | small-tile partials | barriers; two CTAs per SM
    const size_t vf = (size_t)kComputeWarps * 8 * kSmallTile * 8 * 4;  // >= kSmallTile * 64 floats
    const size_t bars = 8 * (2 * kStages + 1);
    static size_t budget_cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    size_t budget = (dev >= 0 && dev < 64) ? budget_cache[dev] : 0;
    if (!budget) {
        cudaFuncAttributes fa;
        size_t stat = 2048;
        if (cudaFuncGetAttributes(&fa, sgmv_stream_kernel) == cudaSuccess) stat = fa.sharedSizeBytes;
        budget = smem_two_per_sm(stat);
        if (dev >= 0 && dev < 64) budget_cache[dev] = budget;
    }
    const size_t fixed = vf + bars + 1024;  // + base alignment slack
    if (budget <= fixed + (size_t)kStages * 16384) return cudaErrorInvalidConfiguration;
    size_t sb = (budget - fixed) / kStages / 1024 * 1024;
    p.stage_bytes = (int)(sb > 32768 ? 32768 : sb);
    const size_t ring = (size_t)kStages * p.stage_bytes;
    p.off_vf = (uint32_t)ring;
    p.off_bar = (uint32_t)(ring + vf);
    const size_t smem = p.off_bar + bars + 1024;

    AMaps am;
    if (!build_pool_maps(am, pool, true, true)) return cudaErrorInvalidValue;
    p.xy_maps = build_xy_maps(am, pool, seg.T, x, x_slice_stride, y, true, true) ? 1 : 0;

    e = cudaFuncSetAttribute(sgmv_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // two launches of the persistent kernel: the shrink parts, then the expand parts as
    // its programmatic dependent
    for (int phase = 0; phase < 2; ++phase) {
        p.phase = phase;
        long long grid = G;
        const long long items = rows * (phase == 0 ? p.Pk : p.Pn);
        if (grid > items) grid = items;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, sgmv_stream_kernel, am, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lora
