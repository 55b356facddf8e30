// fp8_gemm.cu -- 8-bit (E4M3) base GEMM with the multi-tenant LoRA term fused
// into it, on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// The EpiLoRA abstract (sentences 3-4) observes that the GEMM needs the
// adapter's down-projection only in its epilogue, so the down-projection can
// run while the weights stream:
//   y[m][n] = sx[m] * sw[n] * sum_k xq[m][k] Wq[n][k] + s_a * sum_j v[m][j] B[a][j][n],
//   v[m][j] = sum_k x[m][k] A[a][k][j]       (a = adapter of token m, bf16 x).
//
// Design for decode-sized M (tokens) and large N x K weights:
//  * swap-AB: the MMA's M dimension is 128 rows of W, its N dimension the
//    tokens (16..256 per tile), so W -- the bytes that bound the kernel -- is
//    read exactly once while all tokens ride along in one MMA.
//  * stream-K: the (tile, k-block) units are split evenly over one persistent
//    CTA per SM, so no SM idles in a last partial wave. A tile cut between two
//    CTAs is finished by the CTA holding its first k-blocks (the last work of
//    that CTA): the others store fp32 partial accumulators to the workspace
//    first thing and raise a flag; the finisher adds them before its epilogue.
//  * warp roles in each CTA:
//      warp 0  TMA producer: W and xq k-blocks into a ring of stages
//              (128- or 64-byte swizzle, matching the MMA descriptors); W's
//              tiles carry an L2 evict-first policy (read once); its first W
//              loads are issued before the wait on the quantiser;
//      warp 1  TMEM allocator and single-thread tcgen05.mma issuer
//              (kind::f8f6f4, fp32 accumulators in TMEM, double-buffered so the
//              epilogue of one segment overlaps the mainloop of the next); it
//              also issues the LoRA up-projection (kind::f16) of a segment in
//              phases between that segment's own k-blocks;
//      warp 2  B stager: TMA-loads the [r x 128] slices of B_a of the adapters
//              of the tile's token block into a few shared-memory slots, one
//              phase of slots at a time (the MMAs of a phase free the slots);
//      warps 3..10 the down-projection first -- while the first weights
//              stream, each CTA computes v over its own 64-column slice of K
//              for every token (bf16 x, fp32 sums, vector atomics spread over
//              8 copies of v, then a completion count) -- then, per segment,
//              the LoRA operands (V' = s_a v / sx per token block, B' = B / sw
//              per phase) and the epilogue: tcgen05.ld of the accumulator,
//              stream-K partials, per-token and per-channel scales, bf16 rows
//              stored 16 bytes at a time.
//  * tokens are processed in segment order (rows of xq are permuted by the
//    quantiser, v is kept in that order), so the adapter changes only at
//    segment boundaries.
//  * every wait (mbarrier, flag, count) is bounded (2 s); on expiry the CTA
//    records a status word in the workspace, drains what it issued and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kBlockM = 128;  // W rows per tile (MMA M)
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = (3 + kEpiWarps) * 32;
constexpr int kCvtWarps = 8;                      // weight converter warps: half a W row per lane
constexpr int kThreadsW4 = (3 + kEpiWarps + kCvtWarps) * 32;
constexpr int kPackStage = 5120;                  // packed E2M1 tile (128 x 32 B) + scales (2 x 128 B), 1 KB aligned
constexpr int kCodeStage = 8192;                  // E4M3 tile of the 8-bit weights under bf16 activations (128 x 64 B)
// Weight converter modes of the 16-bit MMA path: none (the weights are bf16), MX FP4
// codes with E8M0 block scales, E4M3 codes with a per-channel scale (W8A16).
enum { kWcNone = 0, kWcMxfp4 = 1, kWcE4m3 = 2 };
__host__ __device__ constexpr int wc_stage_bytes(int wc) { return wc == 1 ? kPackStage : (wc == 2 ? kCodeStage : 0); }
// MX FP4: the byte-permute tables of all 256 block scales (uint4 each), built once per CTA
constexpr int kE2m1TabBytes = 256 * 16;
// W8A16: the converter writes each E4M3 weight as bf16 times 2^-112 (the exponent of its
// exact f16 form read as a bf16 exponent), and the per-channel scale carries the 2^112
__host__ __device__ constexpr float e4m3_bf16_shift() { return 5.192296858534828e33f; }  // 2^112
constexpr int kMaxStages = 8;
constexpr int kShrinkCols = 64;  // K columns of the down-projection per work item
constexpr int kShrinkTok = 64;   // tokens of the down-projection per work item
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // drains after an abort

struct GemmParams {
    int M, N, K, BN, n_tb, n_nb, num_tiles, k_blocks, stages;
    long long units;  // num_tiles * k_blocks, split evenly over the grid
    const float* sx;
    const float* sw;
    const uint8_t* wsc;  // MX FP4 block scales (kW4)
    const uint8_t* Wpk;  // MX FP4 codes in 128 x 64 tiles of 4096 bytes
    uint16_t* y;
    uint32_t* status;
    float* partials;  // fp32 stream-K partial accumulators, [gridDim.x][BN/16][4][128][4]
                      // (per 16-token chunk: four float4 planes over the 128 rows)
    int* flags;       // [gridDim.x] partial of CTA c stored
    int* v_done;      // down-projection items finished
    int lora;
    const uint16_t* x;  // bf16 [M][K] (unquantised, by token index)
    const uint16_t* A;  // bf16 [n_adapters][K][r_max]
    const int32_t* perm;
    const int32_t* tok_adapter;
    const int32_t* indptr;
    const int32_t* active;
    const int32_t* counts;
    int v_adapters;  // adapters of a token block whose V' tiles fit (the rest: CUDA cores)
    float* v;  // fp32 [v_rep][M][r_max], segment (perm) order, zeroed by the quantiser: the
               // down-projection of K chunk q adds into copy q % v_rep (fewer atomics per address)
    int v_rep, lg_rep;  // copies of v (a power of two), log2
    int lg_lanes;       // log2 of the lanes that sum one token's copies in the V' build
    const uint16_t* B;
    const int32_t* ranks;
    const float* scales;
    int n_adapters, r_max, r8, r16;
    int n_slots;
    uint32_t ring_off, slots_off, v_off, meta_off, bar_off, tab_off;
    unsigned long long timeout_ns;  // limit of every bounded wait (2 s unless a test lowers it)
    int inject_stall;  // test hook: CTA 0's producer first waits on a barrier nothing completes
};

using ptx::globaltimer;

// Transpose an 8x8 matrix of 32-bit words held by 8 consecutive lanes (lane j of
// the group holds row j in w[0..7]); afterwards lane j holds column j. Three
// butterfly stages swap the off-diagonal blocks of 4x4, 2x2 and 1x1 words.
__device__ __forceinline__ void transpose8x8(uint32_t (&w)[8], int lane)
{
#pragma unroll
    for (int s = 4; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k & s) continue;
            const uint32_t send = upper ? w[k] : w[k | s];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, s);
            if (upper) w[k] = recv; else w[k | s] = recv;
        }
    }
}

// Bounded wait on an mbarrier phase. Returns false if the CTA is aborting
// (another role gave up) or if this wait itself timed out (then it raises the
// abort flag and records `code` in the status word).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             uint32_t* status, uint32_t code, unsigned long long limit)
{
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit) {
            *abort_flag = 1;
            if (status) atomicOr(status, code);
            return false;
        }
    }
}
// Bounded wait used while draining after an abort (no abort check).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity)
{
    const unsigned long long t0 = globaltimer();
    while (!ptx::mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > kTimeoutNs) return;
}

// Bounded wait until the global counter reaches `target` (acquire, GPU scope).
__device__ __forceinline__ bool wait_count(const int* ctr, int target, volatile int* abort_flag,
                                           uint32_t* status, uint32_t code, unsigned long long limit)
{
    const unsigned long long t0 = globaltimer();
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit) {
            *abort_flag = 1;
            if (status) atomicOr(status, code);
            return false;
        }
        __nanosleep(64);
    }
}

// UMMA shared-memory descriptor for a K-major operand tile whose rows are
// SW bytes long (SW = 128 or 64), swizzled by TMA with the same width:
// 8-row core groups SW*8 bytes apart (stride byte offset), version 1.
template <int SW>
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr)
{
    constexpr uint64_t layout = (SW == 128) ? 2ull : 4ull;  // SWIZZLE_128B / SWIZZLE_64B
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
           ((uint64_t)((SW * 8) >> 4) << 32) | ((uint64_t)1 << 46) | (layout << 61);
}

// Instruction descriptor: kind::f8f6f4, A = B = E4M3, both K-major, D fp32,
// M = 128, N = n.
__device__ __forceinline__ uint32_t make_idesc(int n)
{
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBlockM >> 4) << 24);
}

// Instruction descriptor: kind::f16 with A = B = bf16, both K-major, D fp32,
// M = 128, N = n.
__device__ __forceinline__ uint32_t make_idesc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBlockM >> 4) << 24);
}

// UMMA descriptor for a K-major bf16 tile without swizzle: 8-row x 16-byte
// core matrices of 128 contiguous bytes, 128 bytes apart along K (leading
// byte offset) and kg * 128 bytes apart along M / N (stride byte offset).
__device__ __forceinline__ uint64_t make_desc_kmajor(uint32_t saddr, int kg)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
           ((uint64_t)((kg * 128) >> 4) << 32) | ((uint64_t)1 << 46);
}

// Byte offset of (row, 8-column group kg) in such a tile with kg_n groups per row.
__device__ __forceinline__ uint32_t kmajor_off(int row, int kg, int kg_n)
{
    return (uint32_t)((((row >> 3) * kg_n + kg) << 7) + ((row & 7) << 4));
}

// bf16 bit patterns of the 8 E2M1 magnitudes times the block scale 2^(E - 127)
// (exact: at most two significant bits), split into low and high byte tables
// of 8 entries for byte permutes.
__device__ __forceinline__ void e2m1_tables(uint32_t E, uint32_t& lo0, uint32_t& lo1, uint32_t& hi0, uint32_t& hi1)
{
    const float S = E == 0 ? __uint_as_float(0x00400000u) : (E == 255 ? __uint_as_float(0x7fc00000u) : __uint_as_float(E << 23));
    const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = __float_as_uint(mag[i] * S) >> 16;
    lo0 = (b[0] & 0xffu) | ((b[1] & 0xffu) << 8) | ((b[2] & 0xffu) << 16) | ((b[3] & 0xffu) << 24);
    lo1 = (b[4] & 0xffu) | ((b[5] & 0xffu) << 8) | ((b[6] & 0xffu) << 16) | ((b[7] & 0xffu) << 24);
    hi0 = (b[0] >> 8) | ((b[1] >> 8) << 8) | ((b[2] >> 8) << 16) | ((b[3] >> 8) << 24);
    hi1 = (b[4] >> 8) | ((b[5] >> 8) << 8) | ((b[6] >> 8) << 16) | ((b[7] >> 8) << 24);
}

// Eight E2M1 codes (one 32-bit word, element i in nibble i) -> eight bf16 values:
// byte permutes pick each code's magnitude bytes from the tables, the code's
// sign bit becomes the bf16 sign, and the low / high bytes are interleaved.
__device__ __forceinline__ uint4 e2m1x8_to_bf16(uint32_t w, uint32_t lo0, uint32_t lo1, uint32_t hi0, uint32_t hi1)
{
    const uint32_t s0 = w & 0x7777u, s1 = (w >> 16) & 0x7777u;
    const uint32_t w4 = w << 4;
    const uint32_t L0 = __byte_perm(lo0, lo1, s0), L1 = __byte_perm(lo0, lo1, s1);
    const uint32_t H0 = __byte_perm(hi0, hi1, s0) | (__byte_perm(w, w4, 0x1504) & 0x80808080u);
    const uint32_t H1 = __byte_perm(hi0, hi1, s1) | (__byte_perm(w, w4, 0x3726) & 0x80808080u);
    return make_uint4(__byte_perm(L0, H0, 0x5140), __byte_perm(L0, H0, 0x7362), __byte_perm(L1, H1, 0x5140),
                      __byte_perm(L1, H1, 0x7362));
}

// Two E4M3 codes (byte 0 the first) -> two bf16 (the first in the low half):
// E4M3 -> f16 -> f32 -> bf16, every step exact.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t c2)
{
    uint32_t h2, r;
    float lo, hi;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c2));
    asm("{\n.reg .f16 l, h;\nmov.b32 {l, h}, %2;\ncvt.f32.f16 %0, l;\ncvt.f32.f16 %1, h;\n}" : "=f"(lo), "=f"(hi) : "r"(h2));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four E4M3 codes (byte i the i-th) -> four bf16 equal to the codes' values times
// 2^-112: each pair goes to f16 (exact; every E4M3 value, subnormals included, is a
// normal f16 or zero), whose exponent and top mantissa bits, shifted into bf16
// position, read as value * 2^(15 - 127) (E4M3 has 3 mantissa bits, so none is lost).
__device__ __forceinline__ uint2 e4m3x4_to_bf16_shifted(uint32_t w)
{
    uint32_t h0, h1;
    asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %2;\ncvt.rn.f16x2.e4m3x2 %0, lo;\ncvt.rn.f16x2.e4m3x2 %1, hi;\n}"
        : "=r"(h0), "=r"(h1) : "r"(w));
    return make_uint2(((h0 >> 3) & 0x0fff0fffu) | (h0 & 0x80008000u), ((h1 >> 3) & 0x0fff0fffu) | (h1 & 0x80008000u));
}

// Stream-K schedule: CTA c owns units [c*U/G, (c+1)*U/G) of the (tile,
// k-block) sequence; a segment is the part of one tile inside that range.
struct Seg {
    int tile, kb0, kb1;
};
__device__ __forceinline__ long long unit_begin(long long U, int c, int G) { return U * c / G; }

// Next segment starting at unit u (< u_end).
__device__ __forceinline__ Seg seg_at(long long u, long long u_end, int KB)
{
    Seg s;
    s.tile = (int)(u / KB);
    s.kb0 = (int)(u - (long long)s.tile * KB);
    const long long left = u_end - u;
    s.kb1 = (left < (long long)(KB - s.kb0)) ? s.kb0 + (int)left : KB;
    return s;
}

// ESZ: bytes per operand element -- 1 for E4M3 (kind::f8f6f4), 2 for bf16
// (kind::f16). BK is the k-block in bytes either way (128: 128-byte swizzle,
// 64: 64-byte swizzle), so the shared-memory layouts are the same.
// kW4 (a weight converter mode, with ESZ 2 and BK 128): the weights arrive as
// codes -- OCP MX FP4 (packed E2M1 codes and E8M0 block scales) or E4M3 (whose
// per-channel scale the epilogue applies, as on the 8-bit path) -- and eight
// converter warps turn each k-block's codes into the bf16 tile the MMA reads
// (half a row per thread), signalling it on conv[stage].
template <int BK, int MAXR, int ESZ, int kW4 = kWcNone>
__global__ void __launch_bounds__(kW4 != kWcNone ? kThreadsW4 : kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmB, const GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_nact;  // adapters of the current token block on the tensor cores
    __shared__ int s_slot_adapter[256];
    __shared__ int s_slot_rank[256];
    __shared__ int4 s_lq[256];  // per slot: first / end token (block-relative), V' byte offset

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the swizzled TMA tiles need a 1024-byte aligned base
    const uint32_t raw_u = ptx::smem_u32(smem_raw);
    const uint32_t smem_u = (raw_u + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (smem_u - raw_u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* full = bars;                      // [stages]
    uint64_t* empty = bars + kMaxStages;        // [stages]
    uint64_t* tfull = bars + 2 * kMaxStages;    // [2]
    uint64_t* tempty = tfull + 2;               // [2]
    uint64_t* bfull = tempty + 2;               // [1]
    uint64_t* bempty = bfull + 1;               // [1]
    uint64_t* drain = bempty + 1;               // [1]
    uint64_t* epibar = drain + 1;               // [1] epilogue-warps barrier
    uint64_t* lready = epibar + 1;              // [1] LoRA operands of the segment built
    uint64_t* stall = lready + 1;               // [1] test hook: never completed
    uint64_t* conv = stall + 1;                 // [stages] converter paths: the k-block's bf16 W tile built
    volatile int* abort_flag = &s_abort;

    constexpr int kStageW = kBlockM * BK;
    const int stage_bytes = kStageW + p.BN * BK + wc_stage_bytes(kW4);
    constexpr float kWShift = kW4 == kWcE4m3 ? e4m3_bf16_shift() : 1.f;  // see e4m3x4_to_bf16_shifted
    const uint32_t ncols = (uint32_t)(2 * p.BN <= 32 ? 32 : (2 * p.BN <= 64 ? 64 : (2 * p.BN <= 128 ? 128 : (2 * p.BN <= 256 ? 256 : 512))));
    const int G = gridDim.x, cta = blockIdx.x, KB = p.k_blocks;
    const long long u_begin = unit_begin(p.units, cta, G), u_end = unit_begin(p.units, cta + 1, G);

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_nact = 0;
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
            if (kW4 != kWcNone) ptx::mbar_init(&conv[s], kCvtWarps);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], kEpiWarps);
        }
        ptx::mbar_init(bfull, 1);
        ptx::mbar_init(bempty, 1);  // tcgen05.commit of a LoRA phase
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(epibar, kEpiWarps);
        ptx::mbar_init(lready, 1);
        ptx::mbar_init(stall, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&s_tmem, ncols);
        ptx::tmem_relinquish();
    }
    // __syncthreads is an aligned barrier: every warp reaches it converged
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tmW);
            ptx::tma_prefetch_desc(&tmX);
            // W is read exactly once: first out of L2, which then keeps the reused data
            // (xq, the stream-K partials, v, the adapters)
            const uint64_t w_policy = ptx::l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_phase[kMaxStages];
            bool issued[kMaxStages];
            for (int s = 0; s < kMaxStages; ++s) issued[s] = false;
            // the first ring of W loads goes out before the wait on the quantiser
            // (xq is its output, W is not); their xq loads follow the wait
            bool waited = false;
            int n_def = 0, def_kb[kMaxStages], def_tb[kMaxStages];
            auto flush_deferred = [&]() {
                ptx::pdl_wait();
                waited = true;
                for (int d = 0; d < n_def; ++d) {
                    const uint32_t sX = smem_u + p.ring_off + d * stage_bytes + kStageW;
                    ptx::tma_load_2d(sX, &tmX, &full[d], def_kb[d] * (BK / ESZ), def_tb[d] * p.BN);
                }
            };
            bool ok = true;
            // test hook: before its first load, CTA 0 waits on a barrier that nothing
            // completes, so the bounded wait runs out and the CTA takes its abort path
            if (p.inject_stall && cta == 0)
                ok = wait_bounded(stall, 0, abort_flag, p.status, 0x400u, p.timeout_ns);
            for (long long u = u_begin; u < u_end && ok;) {
                const Seg sg = seg_at(u, u_end, KB);
                u += sg.kb1 - sg.kb0;
                const int nb = sg.tile / p.n_tb, tb = sg.tile - nb * p.n_tb;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!waited && n_def == p.stages) flush_deferred();
                    if (!wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 0x1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sW = smem_u + p.ring_off + stage * stage_bytes;
                    const uint32_t sX = sW + kStageW;
                    if constexpr (kW4 == kWcMxfp4) {
                        // packed codes (128 rows x 32 bytes) and the k-block's two scale blocks
                        const uint32_t sP = sX + (uint32_t)(p.BN * BK);
                        ptx::mbar_arrive_expect_tx(&full[stage], (uint32_t)(4096 + 256 + p.BN * BK));
                        ptx::bulk_g2s(sP, p.Wpk + ((size_t)nb * (p.K / 64) + kb) * 4096, 4096, &full[stage]);
                        ptx::bulk_g2s(sP + 4096, p.wsc + ((size_t)nb * (p.K / 32) + kb * 2) * kBlockM, 256,
                                      &full[stage]);
                    } else if constexpr (kW4 == kWcE4m3) {
                        // E4M3 codes: 128 rows x 64 bytes
                        const uint32_t sP = sX + (uint32_t)(p.BN * BK);
                        ptx::mbar_arrive_expect_tx(&full[stage], (uint32_t)(kCodeStage + p.BN * BK));
                        ptx::tma_load_2d_hint(sP, &tmW, &full[stage], kb * 64, nb * kBlockM, w_policy);
                    } else {
                        ptx::mbar_arrive_expect_tx(&full[stage], (uint32_t)stage_bytes);
                        ptx::tma_load_2d_hint(sW, &tmW, &full[stage], kb * (BK / ESZ), nb * kBlockM, w_policy);
                    }
                    if (waited) {
                        ptx::tma_load_2d(sX, &tmX, &full[stage], kb * (BK / ESZ), tb * p.BN);
                    } else {  // first ring pass: stage == n_def
                        def_kb[n_def] = kb;
                        def_tb[n_def] = tb;
                        ++n_def;
                    }
                    issued[stage] = true;
                    issued_phase[stage] = phase;
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!waited) flush_deferred();
            if (!ok)  // let every load this CTA issued land before it exits
                for (int s = 0; s < p.stages; ++s)
                    if (issued[s]) drain_wait(&full[s], issued_phase[s]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            const uint32_t idesc = ESZ == 1 ? make_idesc(p.BN) : make_idesc_bf16(p.BN);
            bool ok = true, any = false;
            int i = 0, lj = 0;
            const uint32_t slots_u = smem_u + p.slots_off, vq_u = smem_u + p.v_off;
            const int kgq = p.r16 >> 3;
            // The up-projection of a y-segment (one that ends in an epilogue) comes in
            // phases of at most n_slots adapters: the epilogue warps build a phase's
            // operands and signal lready, this thread adds them to the segment's
            // accumulator between its own k-blocks (after the segment's first k-block,
            // which starts the accumulator) and commits bempty, which frees the slots
            // for the next phase. tfull follows the last k-block and the last phase.
            // At most two y-segments wait for phases (the two TMEM buffers), in order.
            int fq_buf[2] = {0, 0}, fq_ph[2] = {0, 0};
            bool fq_base_done[2] = {false, false};
            int fq_n = 0;
            auto issue_phase = [&]() {
                ++lj;
                ptx::tc_fence_after();
                const int pbuf = fq_buf[0];
                const uint32_t dp = tmem_base + (uint32_t)(pbuf * p.BN);
                const int nact = s_nact;
                const int e0 = fq_ph[0] * p.n_slots, e1 = min(nact, e0 + p.n_slots);
                for (int e = e0; e < e1; ++e) {
                    // D[n][t] += (B_a[j][n] / sw[n]) * (s_a v[t][j] / sx[t]) over adapter a's tokens
                    const int4 lq = s_lq[e];
                    const int c0 = lq.x & ~15, w = ((lq.y + 15) & ~15) - c0;
                    const uint32_t idl = make_idesc_bf16(w);
                    const uint32_t sb = slots_u + (uint32_t)((e - e0) * p.r16 * 256);
                    for (int ks = 0; ks < (p.r16 >> 4); ++ks)
                        ptx::tc_mma_f16(dp + (uint32_t)c0, make_desc_kmajor(sb + (uint32_t)(ks * 256), kgq),
                                        make_desc_kmajor(vq_u + (uint32_t)(lq.z + ks * 256), kgq), idl, 1u);
                }
                ptx::tc_commit(bempty);  // the slots may be refilled once these MMAs are done
                ++fq_ph[0];
                if (e1 >= nact) {  // that was the segment's last phase
                    if (fq_base_done[0]) ptx::tc_commit(&tfull[pbuf]);
                    else fq_ph[0] = -1;  // tfull goes with the segment's last k-block
                    if (fq_base_done[0]) {
                        fq_buf[0] = fq_buf[1];
                        fq_ph[0] = fq_ph[1];
                        fq_base_done[0] = fq_base_done[1];
                        --fq_n;
                    }
                }
            };
            // issue the next phase of the oldest waiting segment if its operands are ready
            // (block: wait for them, bounded)
            auto lora_step = [&](bool block) -> bool {
                if (fq_n == 0 || fq_ph[0] < 0) return true;
                if (block) {
                    if (!wait_bounded(lready, (uint32_t)(lj & 1), abort_flag, p.status, 0x200u, p.timeout_ns)) return false;
                } else if (!ptx::mbar_test_wait(lready, (uint32_t)(lj & 1))) {  // no suspend
                    return true;
                }
                issue_phase();
                return true;
            };
            // every phase of the waiting segment that uses TMEM buffer b
            auto lora_flush = [&](int b) -> bool {
                while (fq_n > 0 && (b < 0 || fq_buf[0] == b || (fq_n > 1 && fq_buf[1] == b))) {
                    if (fq_ph[0] < 0) return true;  // its k-blocks are not all issued yet
                    if (!lora_step(true)) return false;
                }
                return true;
            };
            for (long long u = u_begin; u < u_end && ok; ++i) {
                const Seg sg = seg_at(u, u_end, KB);
                u += sg.kb1 - sg.kb0;
                const int buf = i & 1;
                const uint32_t bphase = (uint32_t)((i >> 1) & 1);
                const bool yseg = p.lora && sg.kb0 == 0;
                if (!lora_flush(buf)) {  // that buffer's epilogue comes first
                    ok = false;
                    break;
                }
                if (!wait_bounded(&tempty[buf], bphase ^ 1, abort_flag, p.status, 0x2u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * p.BN);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!lora_step(false) ||
                        !wait_bounded(kW4 != kWcNone ? &conv[stage] : &full[stage], phase, abort_flag, p.status, 0x4u,
                                      p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sW = smem_u + p.ring_off + stage * stage_bytes;
                    const uint32_t sX = sW + kStageW;
                    // 32 bytes of K per instruction: 32 E4M3 or 16 bf16 elements
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        if constexpr (ESZ == 1)
                            ptx::tc_mma_f8(d, make_desc<BK>(sW + kk * 32), make_desc<BK>(sX + kk * 32), idesc,
                                           (kb > sg.kb0 || kk != 0) ? 1u : 0u);
                        else
                            ptx::tc_mma_f16(d, make_desc<BK>(sW + kk * 32), make_desc<BK>(sX + kk * 32), idesc,
                                            (kb > sg.kb0 || kk != 0) ? 1u : 0u);
                    }
                    any = true;
                    ptx::tc_commit(&empty[stage]);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                    if (yseg && kb == sg.kb0) {  // the accumulator is started: phases may follow
                        fq_buf[fq_n] = buf;
                        fq_ph[fq_n] = 0;
                        fq_base_done[fq_n] = false;
                        ++fq_n;
                    }
                }
                if (!ok) break;
                if (yseg) {
                    const int q = fq_n - 1;  // this segment's entry (the newest)
                    fq_base_done[q] = true;
                    if (fq_ph[q] < 0) {  // its phases were all issued already
                        ptx::tc_commit(&tfull[buf]);
                        --fq_n;  // it is the only entry: an older one would be ahead of it
                    }
                } else {
                    ptx::tc_commit(&tfull[buf]);
                }
            }
            if (ok && !lora_flush(-1)) ok = false;
            if (!ok && any) {  // wait for the MMAs in flight before TMEM is freed
                ptx::tc_commit(drain);
                drain_wait(drain, 0);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ B stager
        // for every segment that ends in an epilogue (kb0 == 0): the B slices of the
        // adapters of its token block, in phases of at most n_slots adapters; a phase
        // waits for bempty (the MMAs of the previous phase are done)
        if (lane == 0 && p.lora) {
            ptx::tma_prefetch_desc(&tmB);
            const int n_valid = p.counts[0];
            const int n_active = p.counts[1];
            int j = 0, slots_tb = -1, nact = 0;
            bool pending = false;
            uint32_t pending_phase = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok;) {
                const Seg sg = seg_at(u, u_end, KB);
                u += sg.kb1 - sg.kb0;
                if (sg.kb0 != 0) continue;  // partial accumulators only: no epilogue here
                const int nb = sg.tile / p.n_tb, tb = sg.tile - nb * p.n_tb;
                for (int ph = 0;; ++ph) {
                    if (!(ok = wait_bounded(bempty, (uint32_t)((j & 1) ^ 1), abort_flag, p.status, 0x8u, p.timeout_ns))) break;
                    if (ph == 0 && tb != slots_tb) {
                        // the adapters of this token block (kept while the block does not change)
                        slots_tb = tb;
                        const int p0 = tb * p.BN;
                        const int p1 = min(min(p.M, p0 + p.BN), n_valid);
                        int lo = 0, hi = n_active;  // first active segment that ends after p0
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (p.indptr[p.active[mid] + 1] > p0) hi = mid; else lo = mid + 1;
                        }
                        nact = 0;
                        for (int s2 = lo; s2 < n_active && nact < p.v_adapters; ++s2) {
                            const int a = p.active[s2];
                            if (p.indptr[a] >= p1) break;
                            int r = p.ranks ? p.ranks[a] : p.r_max;
                            r = max(1, min(r, p.r_max));
                            s_slot_rank[nact] = r;
                            s_lq[nact] = make_int4(max(p.indptr[a], p0) - p0, min(p.indptr[a + 1], p1) - p0, 0, 0);
                            s_slot_adapter[nact++] = a;
                        }
                        s_nact = nact;
                    }
                    const int e0 = ph * p.n_slots, e1 = min(nact, e0 + p.n_slots);
                    uint32_t bytes = 0;
                    for (int e = e0; e < e1; ++e) bytes += (uint32_t)(((s_slot_rank[e] + 7) >> 3) * 2048);
                    if (bytes) ptx::mbar_arrive_expect_tx(bfull, bytes);
                    for (int e = e0; e < e1; ++e) {
                        const int a = s_slot_adapter[e];
                        const uint32_t dst = smem_u + p.slots_off + (uint32_t)((e - e0) * p.r16 * 256);
                        for (int rb = 0; rb < ((s_slot_rank[e] + 7) >> 3); ++rb)
                            ptx::tma_load_2d(dst + rb * 2048, &tmB, bfull, nb * kBlockM, a * p.r_max + rb * 8);
                    }
                    if (!bytes) ptx::mbar_arrive(bfull);
                    pending = true;
                    pending_phase = (uint32_t)(j & 1);
                    ++j;
                    if (e1 >= nact) break;  // the segment's last phase
                }
            }
            if (*abort_flag && pending) drain_wait(bfull, pending_phase);
        }
    } else if (kW4 == kWcNone || warp < 3 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue warps
        const int ew = warp - 3;
        const int quarter = warp & 3;         // TMEM lane quarter this warp may access
        const int grp = ew >> 2;              // which half of the token chunks
        const int etid = ew * 32 + lane;      // 0..255
        const int n_local = quarter * 32 + lane;
        int* s_m = reinterpret_cast<int*>(smem + p.meta_off);
        int* s_a = s_m + p.BN;
        int* s_r = s_a + p.BN;  // rank of the token's adapter
        int* s_q = s_r + p.BN;  // B slot of the token's adapter (-1: none, -2: not staged)
        float* s_sx = reinterpret_cast<float*>(s_q + p.BN);
        uint8_t* vq = smem + p.v_off;     // V' tiles of the staged adapters (K-major bf16)
        uint8_t* slots = smem + p.slots_off;  // B of the staged adapters, then B' in place
        const int kgq = p.r16 >> 3;
        // barrier among the epilogue warps, bounded like every other wait
        uint32_t epi_phase = 0;
        auto epi_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(epibar);
            const bool ok = wait_bounded(epibar, epi_phase, abort_flag, p.status, 0x40u, p.timeout_ns);
            epi_phase ^= 1;
            return ok;
        };
        ptx::pdl_wait();  // xq, sx and the zeroed v / flags / count come from the quantiser
        bool ok = true;

        // ---- down-projection: work item = 64 columns of K (q) for a block of up to 64
        // tokens (so that a large M spreads over every CTA)
        const int n_chunks = (p.K + kShrinkCols - 1) / kShrinkCols;
        const int n_tblk = (p.M + kShrinkTok - 1) / kShrinkTok;
        const int n_dp = n_chunks * n_tblk;
        if (p.lora) {
            const int ng = p.r_max >> 3;  // groups of 8 rank columns (a power of two)
            const int lg = __ffs(ng) - 1;
            for (int it = cta; it < n_dp && ok; it += G) {
                const int q = it % n_chunks, tblk = it / n_chunks;
                const int t_base = tblk * kShrinkTok;
                const int Mtb = min(kShrinkTok, p.M - t_base);
                // with few (token, group) pairs, split the 64 columns over up to 4 threads
                int ls = 0;
                while (ls < 2 && (Mtb << (lg + ls + 1)) <= kEpiThreads) ++ls;
                const int kspan = kShrinkCols >> ls;  // 64, 32 or 16 columns per thread
                const int total = Mtb << (lg + ls);
                float* vcopy = p.v + (size_t)(q & (p.v_rep - 1)) * p.M * p.r_max;
                // work items w: (token, group of 8 ranks, K sub-range); the 2^ls sub-ranges of
                // one (token, group) sit in consecutive lanes, the loop is uniform per warp
                for (int wb = ew * 32; wb < total; wb += kEpiThreads) {
                    const int w = wb + lane;
                    const int pg = w >> ls, sub = w & ((1 << ls) - 1);
                    const int pp = t_base + (pg >> lg), g = pg & (ng - 1);
                    const int k0 = q * kShrinkCols + sub * kspan;
                    int kw = min(kspan, p.K - k0);  // a multiple of 16 (or <= 0)
                    int r = 0, m = 0, a = -1;
                    if (w < total && kw > 0) {
                        m = p.perm[pp];
                        a = p.tok_adapter[m];
                        if (a >= 0) {
                            r = p.ranks ? p.ranks[a] : p.r_max;
                            r = max(1, min(r, p.r_max));
                        }
                    }
                    const bool live = a >= 0 && 8 * g < r;
                    if (!live) kw = 0;
                    const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)m * p.K + k0);
                    const uint16_t* ar = p.A + ((size_t)max(a, 0) * p.K + k0) * p.r_max + 8 * g;
                    float acc[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
                    for (int kk = 0; kk < kw; kk += 16) {
                        // 16 columns: all 18 loads in flight before the first FMA
                        const uint4 xv0 = __ldg(xr + (kk >> 3)), xv1 = __ldg(xr + (kk >> 3) + 1);
                        uint4 av[16];
#pragma unroll
                        for (int h = 0; h < 16; ++h)
                            av[h] = __ldg(reinterpret_cast<const uint4*>(ar + (size_t)(kk + h) * p.r_max));
                        const uint32_t xw[8] = {xv0.x, xv0.y, xv0.z, xv0.w, xv1.x, xv1.y, xv1.z, xv1.w};
#pragma unroll
                        for (int h = 0; h < 16; ++h) {
                            const float xf = __uint_as_float((h & 1) ? (xw[h >> 1] & 0xffff0000u) : (xw[h >> 1] << 16));
                            const uint32_t aw[4] = {av[h].x, av[h].y, av[h].z, av[h].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                acc[2 * e] = fmaf(xf, __uint_as_float(aw[e] << 16), acc[2 * e]);
                                acc[2 * e + 1] = fmaf(xf, __uint_as_float(aw[e] & 0xffff0000u), acc[2 * e + 1]);
                            }
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (8 * g + e >= r) acc[e] = 0.f;  // the pool's padding past the rank
                    // the sub-ranges' sums meet in their first lane: one pair of atomics per item
                    for (int o = 1; o < (1 << ls); o <<= 1) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
                    }
                    if (live && sub == 0 && w < total) {
                        float* vd = vcopy + (size_t)pp * p.r_max + 8 * g;
                        atomicAdd(reinterpret_cast<float4*>(vd), make_float4(acc[0], acc[1], acc[2], acc[3]));
                        atomicAdd(reinterpret_cast<float4*>(vd + 4), make_float4(acc[4], acc[5], acc[6], acc[7]));
                    }
                }
                __threadfence();
                ok = epi_sync();
                if (ok && etid == 0) atomicAdd(p.v_done, 1);
            }
        }

        // ---- epilogues of this CTA's segments
        int i = 0, jf = 0, staged_tb = -1, slotted_tb = -1;
        bool v_ready = !p.lora;
        for (long long u = u_begin; u < u_end && ok; ++i) {
            const Seg sg = seg_at(u, u_end, KB);
            u += sg.kb1 - sg.kb0;
            const int nb = sg.tile / p.n_tb, tb = sg.tile - nb * p.n_tb;
            const int buf = i & 1;
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * p.BN);
            if (sg.kb0 > 0) {
                // later k-blocks of a tile another CTA finishes: fp32 partials to the workspace
                if (!wait_bounded(&tfull[buf], (uint32_t)((i >> 1) & 1), abort_flag, p.status, 0x10u, p.timeout_ns)) break;
                ptx::tc_fence_after();
                // per 16-column chunk four planes [128 rows][4 columns]: each store of a
                // warp covers 512 contiguous bytes
                for (int c0 = grp * 16; c0 < p.BN; c0 += 32) {
                    float acc[16];
                    ptx::tmem_ld16(taddr + (uint32_t)c0, acc);
                    float4* dst = reinterpret_cast<float4*>(p.partials + ((size_t)cta * (p.BN >> 4) + (c0 >> 4)) * 2048) + n_local;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        __stcg(dst + q * kBlockM, make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]));
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
                __threadfence();
                if (!(ok = epi_sync())) break;
                if (etid == 0) atomicExch(p.flags + cta, 1);
                continue;
            }
            if (staged_tb != tb) {
                if (!v_ready) {  // every CTA's share of the down-projection is in v
                    if (etid == 0) ok = wait_count(p.v_done, n_dp, abort_flag, p.status, 0x80u, p.timeout_ns);
                    if (!(ok = epi_sync() && ok)) break;
                    v_ready = true;
                }
                // this token block's metadata and s_a * v in shared memory
                if (staged_tb >= 0 && !(ok = epi_sync())) break;
                for (int pl = etid; pl < p.BN; pl += kEpiThreads) {
                    const int pp = tb * p.BN + pl;
                    int m = 0, a = -1;
                    float sxp = 0.f;
                    if (pp < p.M) {
                        m = p.perm ? p.perm[pp] : pp;
                        sxp = p.sx[pp];
                        if (p.lora) a = p.tok_adapter[m];
                    }
                    s_m[pl] = m;
                    s_a[pl] = a;
                    s_sx[pl] = sxp;
                    s_r[pl] = 0;
                    if (p.lora) {
                        int r = 0;
                        float sc = 0.f;
                        if (a >= 0) {
                            r = p.ranks ? p.ranks[a] : p.r_max;
                            r = max(0, min(r, p.r_max));
                            sc = p.scales ? p.scales[a] : 1.f;
                        }
                        s_r[pl] = r;
                        (void)sc;
                    }
                }
                if (!(ok = epi_sync())) break;
                staged_tb = tb;
            }
            // the LoRA operands of this segment, phase by phase: the MMA warp adds each
            // phase to the accumulator (between its k-blocks) and signals tfull after the last
            for (int ph = 0; p.lora && ok; ++ph) {
                if (!(ok = wait_bounded(bfull, (uint32_t)(jf & 1), abort_flag, p.status, 0x20u, p.timeout_ns))) break;
                ++jf;
                const int nact = s_nact;
                const int e0 = ph * p.n_slots, e1 = min(nact, e0 + p.n_slots);
                if (ph == 0 && slotted_tb != tb) {
                    // per token: its entry in the block's adapter list (-2: past the list, done on
                    // CUDA cores below); per entry e: V'_e[t][j] = s_a v[t][j] / sx[t] for its
                    // tokens t (zero for the other tokens of its 16-aligned column range), K-major
                    // bf16, for every phase of every segment of this token block. Each token's
                    // v row is loaded first, so the build waits for one round trip to memory
                    // lane (token pl, lane cp of the token's 2^lg_lanes): the lane loads copies
                    // cp, cp + lanes, ... of the token's v row and adds them, then the token's
                    // lanes sum by shuffles (BN * lanes <= 256)
                    const int lanes = 1 << p.lg_lanes, cpl = p.v_rep >> p.lg_lanes;
                    const int pl = etid >> p.lg_lanes, cp = etid & (lanes - 1);
                    const size_t cstride = (size_t)lanes * p.M * p.r_max / 4;  // float4s between a lane's copies
                    int q_own = -1;
                    float4 vr[4];  // v[token][0..16) (a larger rank loads the rest later)
#pragma unroll
                    for (int h = 0; h < 4; ++h) vr[h] = make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4* vg = reinterpret_cast<const float4*>(
                        p.v + ((size_t)cp * p.M + tb * p.BN + min(pl, p.BN - 1)) * p.r_max);
                    auto add4 = [](float4& a4, const float4 b4) {
                        a4.x += b4.x;
                        a4.y += b4.y;
                        a4.z += b4.z;
                        a4.w += b4.w;
                    };
                    if (pl < p.BN) {
                        const int a = s_a[pl];
                        if (a >= 0) {
                            q_own = -2;
                            for (int t = 0; t < nact; ++t)
                                if (s_slot_adapter[t] == a) { q_own = t; break; }
                        }
                        if (cp == 0) s_q[pl] = q_own;
                        if (q_own >= 0) {
                            for (int i = 0; i < cpl; ++i)
#pragma unroll
                                for (int h = 0; h < 4; ++h)
                                    if (4 * h < p.r_max) add4(vr[h], __ldcg(vg + i * cstride + h));
                        }
                    }
                    // zero every slot's tile and publish its byte offset
                    int off = 0;
                    for (int q = 0; q < nact; ++q) {
                        const int4 lq = s_lq[q];
                        const int w = ((lq.y + 15) & ~15) - (lq.x & ~15);
                        if (etid == 0) s_lq[q].z = off;
                        for (int i = etid; i < w * kgq; i += kEpiThreads)
                            *reinterpret_cast<uint4*>(vq + off + i * 16) = make_uint4(0u, 0u, 0u, 0u);
                        off += w * kgq * 16;
                    }
                    if (!(ok = epi_sync())) break;
                    auto sum_copies = [&](float4& f) {
                        for (int o = 1; o < lanes; o <<= 1) {
                            f.x += __shfl_xor_sync(0xffffffffu, f.x, o);
                            f.y += __shfl_xor_sync(0xffffffffu, f.y, o);
                            f.z += __shfl_xor_sync(0xffffffffu, f.z, o);
                            f.w += __shfl_xor_sync(0xffffffffu, f.w, o);
                        }
                    };
#pragma unroll
                    for (int h = 0; h < 4; ++h) sum_copies(vr[h]);
                    {  // this token's row of its slot's tile (lane cp == 0 writes it)
                        const int4 lq = s_lq[max(q_own, 0)];
                        const int rr = pl - (lq.x & ~15);
                        const int r = q_own >= 0 ? s_slot_rank[q_own] : 0;
                        const float f = q_own >= 0 ? (p.scales ? p.scales[s_slot_adapter[q_own]] : 1.f) / s_sx[pl] : 0.f;
#pragma unroll
                        for (int kg = 0; kg < MAXR / 8; ++kg) {
                            if (kg >= kgq) break;
                            float vv[8];
                            const bool in_row = q_own >= 0 && 8 * kg < p.r_max;  // r_max: a multiple of 8
                            float4 f0 = make_float4(0.f, 0.f, 0.f, 0.f), f1 = f0;
                            if (kg < 2) {
                                f0 = vr[2 * kg];
                                f1 = vr[2 * kg + 1];
                            } else {
                                if (in_row)
                                    for (int i = 0; i < cpl; ++i) {
                                        add4(f0, __ldcg(vg + i * cstride + 2 * kg));
                                        add4(f1, __ldcg(vg + i * cstride + 2 * kg + 1));
                                    }
                                sum_copies(f0);
                                sum_copies(f1);
                            }
                            if (q_own < 0 || cp != 0) continue;
                            vv[0] = f0.x; vv[1] = f0.y; vv[2] = f0.z; vv[3] = f0.w;
                            vv[4] = f1.x; vv[5] = f1.y; vv[6] = f1.z; vv[7] = f1.w;
                            uint32_t wv[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const int j = kg * 8 + 2 * h;
                                const float v0 = j < r ? f * vv[2 * h] : 0.f;
                                const float v1 = j + 1 < r ? f * vv[2 * h + 1] : 0.f;
                                __nv_bfloat162 hv = __floats2bfloat162_rn(v0, v1);
                                wv[h] = *reinterpret_cast<uint32_t*>(&hv);
                            }
                            *reinterpret_cast<uint4*>(vq + lq.z + kmajor_off(rr, kg, kgq)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        }
                    }
                    slotted_tb = tb;
                }
                // B'[n][j] = B_a[j][n] / sw[n] in place, K-major, for the phase's slots: each
                // thread reads its row n of kSpt slots, then (after a barrier) writes them
                const int nn = etid & 127, half = etid >> 7;
                const float inv_sw2 = (nb * kBlockM + nn < p.N) ? 1.f / ((p.sw ? p.sw[nb * kBlockM + nn] : 1.f) * kWShift) : 0.f;
                const int nbuf = e1 - e0;
                constexpr int kSpt = MAXR <= 16 ? 4 : (MAXR <= 32 ? 2 : 1);
                for (int b0 = 0; b0 < nbuf && ok; b0 += 2 * kSpt) {
                    uint32_t colw[kSpt][MAXR / 2];
#pragma unroll
                    for (int t = 0; t < kSpt; ++t) {
                        const int b = b0 + 2 * t + half;
                        const int r = b < nbuf ? s_slot_rank[e0 + b] : 0;
                        const uint16_t* raw = reinterpret_cast<const uint16_t*>(slots + (size_t)(b < nbuf ? b : 0) * p.r16 * 256) + nn;
#pragma unroll
                        for (int j = 0; j < MAXR; j += 2) {
                            const float c0 = j < r ? __uint_as_float((uint32_t)raw[j * 128] << 16) * inv_sw2 : 0.f;
                            const float c1 = j + 1 < r ? __uint_as_float((uint32_t)raw[(j + 1) * 128] << 16) * inv_sw2 : 0.f;
                            __nv_bfloat162 hv = __floats2bfloat162_rn(c0, c1);
                            colw[t][j >> 1] = *reinterpret_cast<uint32_t*>(&hv);
                        }
                    }
                    if (!(ok = epi_sync())) break;
#pragma unroll
                    for (int t = 0; t < kSpt; ++t) {
                        const int b = b0 + 2 * t + half;
                        if (b >= nbuf) continue;
                        uint8_t* dst = slots + (size_t)b * p.r16 * 256;
#pragma unroll
                        for (int kg = 0; kg < MAXR / 8; ++kg) {
                            if (kg >= kgq) break;
                            *reinterpret_cast<uint4*>(dst + kmajor_off(nn, kg, kgq)) =
                                make_uint4(colw[t][4 * kg], colw[t][4 * kg + 1], colw[t][4 * kg + 2], colw[t][4 * kg + 3]);
                        }
                    }
                    // the next round reads other slots: no barrier before it
                }
                if (!ok) break;
                ptx::fence_proxy_async_smem();  // generic writes, read by the tensor core (async proxy)
                if (!(ok = epi_sync())) break;
                if (etid == 0) ptx::mbar_arrive(lready);
                if (e1 >= nact) break;  // the segment's last phase
            }
            if (!ok) break;
            if (!(ok = wait_bounded(&tfull[buf], (uint32_t)((i >> 1) & 1), abort_flag, p.status, 0x10u, p.timeout_ns))) break;
            ptx::tc_fence_after();
            // the CTAs after this one that hold later k-blocks of this tile
            int c_hi = cta + 1;
            if (sg.kb1 < KB) {
                const long long tile_end = (long long)(sg.tile + 1) * KB;
                while (c_hi < G && unit_begin(p.units, c_hi, G) < tile_end) ++c_hi;
                if (etid == 0)
                    for (int cc = cta + 1; cc < c_hi && ok; ++cc)
                        ok = wait_count(p.flags + cc, 1, abort_flag, p.status, 0x100u, p.timeout_ns);
                if (!(ok = epi_sync() && ok)) break;
            }

            const int n = nb * kBlockM + n_local;
            const float swn = n < p.N ? (p.sw ? p.sw[n] : 1.f) * kWShift : 0.f;

            // partial sums of the later k-blocks for 16 columns (zero when nobody else has any);
            // the next chunk's are loaded while this one is processed
            const bool fixup = c_hi > cta + 1;
            // the partial sums of the next CTA (the usual single contributor) are loaded two
            // chunks ahead of their use, as raw registers; those of any further CTA are added
            // when their chunk is processed
            auto part_src = [&](int cc, int c) {
                return reinterpret_cast<const float4*>(p.partials + ((size_t)cc * (p.BN >> 4) + (c >> 4)) * 2048) + n_local;
            };
            auto part_issue = [&](int c, float4 (&dst)[4]) {
                if (fixup && c < p.BN && tb * p.BN + c < p.M) {
                    const float4* src = part_src(cta + 1, c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[q] = __ldcg(src + q * kBlockM);
                }
            };
            float4 pa[4], pb[4];  // chunk c0 and chunk c0 + 32 of this warp
            part_issue(grp * 16, pa);
            part_issue(grp * 16 + 32, pb);
            // 16 tokens per chunk, fully unrolled so the accumulator stays in registers
            for (int c0 = grp * 16; c0 < p.BN; c0 += 32) {
                const int valid_n = min(16, p.M - (tb * p.BN + c0));  // tokens of this chunk
                if (valid_n <= 0) break;
                float acc[16];
                ptx::tmem_ld16(taddr + (uint32_t)c0, acc);
                if (fixup) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[4 * q] += pa[q].x;
                        acc[4 * q + 1] += pa[q].y;
                        acc[4 * q + 2] += pa[q].z;
                        acc[4 * q + 3] += pa[q].w;
                        pa[q] = pb[q];
                    }
                    part_issue(c0 + 64, pb);
                    for (int cc = cta + 2; cc < c_hi; ++cc) {
                        const float4* src = part_src(cc, c0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 f = __ldcg(src + q * kBlockM);
                            acc[4 * q] += f.x;
                            acc[4 * q + 1] += f.y;
                            acc[4 * q + 2] += f.z;
                            acc[4 * q + 3] += f.w;
                        }
                    }
                }
                float lo[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) lo[e] = 0.f;
                if (p.lora) {
                    // adapters past the V' capacity of the token block: their term on CUDA cores, B
                    // and v from global memory (the staged ones are in the accumulator)
                    bool far = false;
#pragma unroll
                    for (int e = 0; e < 16; ++e) far = far || (e < valid_n && s_q[c0 + e] == -2);
                    if (far) {
                        for (int e = 0; e < valid_n; ++e) {
                            if (s_q[c0 + e] != -2) continue;
                            const int a = s_a[c0 + e], r = s_r[c0 + e];
                            const float sc = p.scales ? p.scales[a] : 1.f;
                            const uint16_t* gb = p.B + ((size_t)a * p.r_max) * p.N + n;
                            const float* vg = p.v + (size_t)(tb * p.BN + c0 + e) * p.r_max;
                            float l = 0.f;
                            for (int j = 0; j < r; ++j) {
                                float vj = 0.f;
                                for (int c = 0; c < p.v_rep; ++c) vj += __ldcg(vg + (size_t)c * p.M * p.r_max + j);
                                l = fmaf(vj, n < p.N ? __uint_as_float((uint32_t)gb[(size_t)j * p.N] << 16) : 0.f, l);
                            }
#pragma unroll
                            for (int e2 = 0; e2 < 16; ++e2)
                                if (e2 == e) lo[e2] = sc * l;
                        }
                    }
                }
                {
                    // y is 16-byte aligned and N % 8 == 0 (checked by the caller): after an 8x8
                    // transpose inside each group of 8 lanes, a lane holds two token rows of 8
                    // consecutive columns, so a chunk takes two 16-byte stores instead of 16
                    float sxv[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 f = reinterpret_cast<const float4*>(s_sx + c0)[q];
                        sxv[4 * q] = f.x;
                        sxv[4 * q + 1] = f.y;
                        sxv[4 * q + 2] = f.z;
                        sxv[4 * q + 3] = f.w;
                    }
                    uint32_t w[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float o0 = acc[2 * k] * sxv[2 * k] * swn + lo[2 * k];
                        const float o1 = acc[2 * k + 1] * sxv[2 * k + 1] * swn + lo[2 * k + 1];
                        __nv_bfloat162 h = __floats2bfloat162_rn(o0, o1);
                        w[k] = *reinterpret_cast<uint32_t*>(&h);
                    }
                    transpose8x8(w, lane);
                    const int j = lane & 7;                                 // token pair of this lane
                    const int ng = nb * kBlockM + quarter * 32 + (lane & ~7);  // its 8 columns
                    const int2 rows = reinterpret_cast<const int2*>(s_m + c0)[j];
                    if (ng < p.N) {                                         // N % 8 == 0: all 8 or none
                        if (2 * j < valid_n) {
                            const uint4 r0 = make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                                                        __byte_perm(w[4], w[5], 0x5410), __byte_perm(w[6], w[7], 0x5410));
                            *reinterpret_cast<uint4*>(p.y + (size_t)rows.x * p.N + ng) = r0;
                        }
                        if (2 * j + 1 < valid_n) {
                            const uint4 r1 = make_uint4(__byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632),
                                                        __byte_perm(w[4], w[5], 0x7632), __byte_perm(w[6], w[7], 0x7632));
                            *reinterpret_cast<uint4*>(p.y + (size_t)rows.y * p.N + ng) = r1;
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&tempty[buf]);
            }
        }
    }

    if constexpr (kW4 != kWcNone) {
        if (warp >= 3 + kEpiWarps) {
            // ------------------------------------------------------------ converter warps
            // thread = half of one W row of the tile: its 32 codes of the k-block (and, for
            // MX FP4, their block scale) become 32 bf16 values, four 16-byte chunks of the
            // 128-byte swizzled row the MMA descriptor expects
            constexpr int kCvtThreads = kCvtWarps * 32;
            static_assert(kCvtThreads == 128 || kCvtThreads == 256, "a thread converts one or two half rows");
            const int ct = (warp - 3 - kEpiWarps) * 32 + lane;
            const int row = ct & 127;
            const uint4* tab = reinterpret_cast<const uint4*>(smem + p.tab_off);
            if constexpr (kW4 == kWcMxfp4) {
                for (int e = ct; e < 256; e += kCvtThreads) {
                    uint32_t lo0, lo1, hi0, hi1;
                    e2m1_tables((uint32_t)e, lo0, lo1, hi0, hi1);
                    *reinterpret_cast<uint4*>(smem + p.tab_off + e * 16) = make_uint4(lo0, lo1, hi0, hi1);
                }
                ptx::named_sync(1, kCvtThreads);  // the table is complete
            }
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok;) {
                const Seg sg = seg_at(u, u_end, KB);
                u += sg.kb1 - sg.kb0;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    bool got = true;
                    if (lane == 0) got = wait_bounded(&full[stage], phase, abort_flag, p.status, 0x800u, p.timeout_ns);
                    got = __shfl_sync(0xffffffffu, got, 0);
                    if (!got) {
                        ok = false;
                        break;
                    }
                    if (lane != 0) drain_wait(&full[stage], phase);  // complete already: acquire
                    uint8_t* st_base = smem + p.ring_off + (size_t)stage * stage_bytes;
                    const uint8_t* pk = st_base + kStageW + p.BN * BK;
                    uint8_t* dst = st_base + row * 128;
                    const int sw = row & 7;
#pragma unroll
                    for (int half = ct >> 7; half < 2; half += kCvtThreads / 128) {
                        const int c0 = 4 * half;
                        if constexpr (kW4 == kWcE4m3) {
                            // 32 E4M3 codes -> bf16 times 2^-112 (exact)
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint4 q = *reinterpret_cast<const uint4*>(pk + row * 64 + half * 32 + h * 16);
                                const uint2 a = e4m3x4_to_bf16_shifted(q.x), b = e4m3x4_to_bf16_shifted(q.y);
                                const uint2 c = e4m3x4_to_bf16_shifted(q.z), d = e4m3x4_to_bf16_shifted(q.w);
                                *reinterpret_cast<uint4*>(dst + (((c0 + 2 * h) ^ sw) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
                                *reinterpret_cast<uint4*>(dst + (((c0 + 2 * h + 1) ^ sw) << 4)) = make_uint4(c.x, c.y, d.x, d.y);
                            }
                        } else {
                            const uint4 q = *reinterpret_cast<const uint4*>(pk + row * 32 + half * 16);
                            const uint4 t = tab[pk[4096 + half * 128 + row]];
                            *reinterpret_cast<uint4*>(dst + (((c0 + 0) ^ sw) << 4)) = e2m1x8_to_bf16(q.x, t.x, t.y, t.z, t.w);
                            *reinterpret_cast<uint4*>(dst + (((c0 + 1) ^ sw) << 4)) = e2m1x8_to_bf16(q.y, t.x, t.y, t.z, t.w);
                            *reinterpret_cast<uint4*>(dst + (((c0 + 2) ^ sw) << 4)) = e2m1x8_to_bf16(q.z, t.x, t.y, t.z, t.w);
                            *reinterpret_cast<uint4*>(dst + (((c0 + 3) ^ sw) << 4)) = e2m1x8_to_bf16(q.w, t.x, t.y, t.z, t.w);
                        }
                    }
                    ptx::fence_proxy_async_smem();  // generic writes, read by the tensor core
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&conv[stage]);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    }

    // the single-lane roles of warps 0-2 rejoin their warps before the aligned barrier
    // (otherwise a lane arriving late is not held by it)
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, ncols);
    }
}

// ---------------------------------------------------------------- host side

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base,
               uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz)
{
    return encode_tmap_2d(m, dt, base, inner, outer, inner * (uint64_t)elem_bytes, box_inner,
                          box_outer, swz);
}

template <int BK, int MAXR, int ESZ, int kW4 = kWcNone>
cudaError_t launch_t(const GemmParams& p, const CUtensorMap& tmW, const CUtensorMap& tmX,
                     const CUtensorMap& tmB, size_t smem, int grid, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(fp8_gemm_kernel<BK, MAXR, ESZ, kW4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kW4 != kWcNone ? kThreadsW4 : kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // a programmatic dependent of the quantiser: the first W loads overlap it
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fp8_gemm_kernel<BK, MAXR, ESZ, kW4>, tmW, tmX, tmB, p);
}

size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

}  // namespace

int device_sm_count()
{
    int dev = 0;
    cudaGetDevice(&dev);
    static int cached[64] = {0};
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

int fp8_gemm_tile_n(int M)
{
    const int n_tb = (M + 255) / 256;
    return (((M + n_tb - 1) / n_tb) + 15) / 16 * 16;
}

int fp8_gemm_v_copies(int M)
{
    // 8 copies: the adds of 128 K chunks into one 16-byte piece of v are spread 8 ways;
    // the V' build sums them (one lane per copy at few tokens, several copies a lane at more)
    (void)M;
    return 8;
}

size_t fp8_gemm_partial_bytes(int M)
{
    return (size_t)device_sm_count() * kBlockM * (size_t)fp8_gemm_tile_n(M) * 4;
}

cudaError_t launch_fp8_gemm(const Fp8GemmArgs& a, cudaStream_t stream)
{
    GemmParams p = {};
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.n_tb = (a.M + 255) / 256;
    p.BN = fp8_gemm_tile_n(a.M);
    p.n_nb = (a.N + kBlockM - 1) / kBlockM;
    p.num_tiles = p.n_nb * p.n_tb;
    p.sx = a.sx;
    p.sw = a.sw;
    p.wsc = a.wsc;
    p.Wpk = a.Wq;
    p.y = a.y;
    p.status = a.status;
    p.partials = a.partials;
    p.flags = a.flags;
    p.v_done = a.v_done;
    p.lora = a.lora ? 1 : 0;
    p.x = a.x;
    p.A = a.A;
    p.perm = a.perm;
    p.tok_adapter = a.tok_adapter;
    p.indptr = a.indptr;
    p.active = a.active;
    p.counts = a.counts;
    p.v = a.v;
    p.v_rep = fp8_gemm_v_copies(a.M);
    p.lg_rep = __builtin_ctz((unsigned)p.v_rep);
    p.lg_lanes = p.lg_rep;
    while ((p.BN << p.lg_lanes) > kEpiThreads) --p.lg_lanes;
    p.B = a.B;
    p.ranks = a.ranks;
    p.scales = a.scales;
    p.n_adapters = a.n_adapters;
    p.r_max = a.lora ? a.r_max : 0;
    p.r8 = a.lora ? (a.r_max + 7) / 8 * 8 : 0;
    p.r16 = a.lora ? (a.r_max + 15) / 16 * 16 : 0;

    // shared-memory plan: ring | B slots | v | meta | barriers, within the
    // opt-in per-block limit minus the kernel's static shared memory
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, fp8_gemm_kernel<128, 64, 1>) != cudaSuccess) return cudaErrorInvalidValue;
    const size_t kSmemMax = (size_t)(optin > 0 ? optin : 232448) - fa.sharedSizeBytes - 256;
    const size_t meta = align_up((size_t)p.BN * 20, 128);  // token, adapter, rank, slot, sx
    const size_t bars = 8 * (3 * kMaxStages + 10);
    // a slot holds one adapter's B[j][128 n] as loaded, then B'[128 n][r16] in place
    const size_t slot_bytes = (size_t)p.r16 * 256;
    // V' tiles of va adapters: their token ranges are disjoint and contiguous, so their
    // 16-aligned windows cover at most BN + 16 (va - 1) token rows of r16 bf16
    auto vq_bytes = [&](int va) -> size_t {
        return (a.lora && va > 0) ? align_up(((size_t)p.BN + 16 * (size_t)(va - 1)) * p.r16 * 2, 128) : 0;
    };
    const int wc = a.wsc != nullptr ? kWcMxfp4 : (a.esz == 2 && a.w_e4m3 ? kWcE4m3 : kWcNone);
    const bool w4 = wc != kWcNone;
    auto fit = [&](int bk, int va, int ns) -> int {
        if (w4 && bk != 128) return 0;  // the converter writes 128-byte rows
        const size_t stage_bytes = (size_t)kBlockM * bk + (size_t)p.BN * bk + wc_stage_bytes(wc);
        const size_t fixed = 1024 + meta + vq_bytes(va) + bars + (size_t)ns * slot_bytes +
                             (wc == kWcMxfp4 ? (size_t)kE2m1TabBytes + 16 : 0);
        if (fixed >= kSmemMax) return 0;
        const size_t st = (kSmemMax - fixed) / stage_bytes;
        return (int)(st > (size_t)kMaxStages ? kMaxStages : st);
    };
    // Every adapter of a token block gets a V' tile when they fit (va); their B slices
    // pass through ns slots, in phases of ns adapters. Preference: 128-byte k-blocks with
    // >= 4 stages, then with 3 (a tile of 256 tokens), then 64-byte k-blocks; within
    // each, as many slots as fit; fewer V' tiles only as a last resort.
    int want_va = a.lora ? (a.n_adapters < p.BN ? a.n_adapters : p.BN) : 0;
    if (want_va > 256) want_va = 256;
    int BK = 0, va = 0, ns = 0, stages = 0;
    if (!a.lora) {
        BK = 128;
        stages = fit(128, 0, 0);
    } else {
        // a phase costs a few microseconds of latency (load, transform, MMAs): keep at
        // least 4 slots (or one per adapter) so that a segment needs few phases
        const int tries[3][2] = {{128, 4}, {128, 3}, {64, 4}};
        for (int v = want_va; v >= 1 && !BK; v = v > 1 ? (v + 1) / 2 : 0) {
            for (int t = 0; t < 3 && !BK; ++t) {
                const int bk = tries[t][0], min_st = tries[t][1];
                int n = v;
                while (n >= 1 && fit(bk, v, n) < min_st) --n;
                if (n >= (v < 4 ? v : 4)) {
                    BK = bk;
                    va = v;
                    ns = n;
                    stages = fit(bk, v, n);
                }
            }
        }
        if (!BK) {  // no tensor-core slots at all: every adapter on CUDA cores
            BK = 64;
            stages = fit(64, 0, 0);
        }
    }
    // At a few tokens the weight stream is HBM-bound with fewer stages in flight as well;
    // a shallower queue of weight loads shortens the latency of the LoRA term's own loads
    // (down-projection, v, B): 6 stages rather than 8 measured ~1 us faster at M = 16
    if (a.lora && p.BN <= 32 && stages > 6) stages = 6;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    p.stages = stages;
    p.n_slots = ns;
    p.v_adapters = va;
    const int esz = a.esz == 2 ? 2 : 1;
    p.k_blocks = (a.K * esz + BK - 1) / BK;
    p.units = (long long)p.num_tiles * p.k_blocks;
    const size_t stage_bytes = (size_t)kBlockM * BK + (size_t)p.BN * BK + wc_stage_bytes(wc);
    p.ring_off = 0;
    p.slots_off = (uint32_t)align_up((size_t)stages * stage_bytes, 1024);
    p.v_off = (uint32_t)align_up(p.slots_off + (size_t)ns * slot_bytes, 128);
    p.meta_off = (uint32_t)(p.v_off + vq_bytes(va));
    p.bar_off = (uint32_t)align_up(p.meta_off + meta, 8);
    p.tab_off = (uint32_t)align_up(p.bar_off + bars, 16);
    const size_t smem = align_up(p.tab_off + (wc == kWcMxfp4 ? (size_t)kE2m1TabBytes : 0), 128) + 1024;  // + alignment slack

    CUtensorMap tmW, tmX, tmB;
    const CUtensorMapSwizzle swz = BK == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapDataType dt = esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if (!encode_2d(&tmX, dt, esz, a.xq, (uint64_t)a.K, (uint64_t)a.M, (uint32_t)(BK / esz), (uint32_t)p.BN, swz))
        return cudaErrorInvalidValue;
    if (wc == kWcMxfp4) {  // packed codes in 4096-byte tiles: 1-D bulk copies, no tensor map
        if (esz != 2 || BK != 128) return cudaErrorInvalidValue;
        tmW = tmX;  // a valid map the kernel never loads through
    } else if (wc == kWcE4m3) {  // E4M3 codes: [N][K] bytes, boxes of 128 rows x 64 bytes, not swizzled
        if (esz != 2 || BK != 128 ||
            !encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Wq, (uint64_t)a.K, (uint64_t)a.N, 64, kBlockM,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else if (!encode_2d(&tmW, dt, esz, a.Wq, (uint64_t)a.K, (uint64_t)a.N, (uint32_t)(BK / esz), kBlockM, swz)) {
        return cudaErrorInvalidValue;
    }
    if (a.lora) {
        if (!encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.B, (uint64_t)a.N,
                       (uint64_t)a.n_adapters * a.r_max, 128, 8, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else {
        tmB = tmW;  // unused
    }

    p.timeout_ns = debug_wait_limit_ns();
    p.inject_stall = debug_inject_stall();
    // One persistent CTA per SM (the partial buffers and flags are sized for that).
    // The CTAs wait on one another (the down-projection count, the stream-K flags), so
    // every CTA of the grid must be resident at once: the grid is at most the SMs times
    // the CTAs of this kernel that fit on one SM (one, by its shared memory). A context
    // limited to fewer SMs than the device has (an MPS share, a green context) cannot
    // hold that grid: its CTAs would wait until the bounded waits give up.
    const bool small_r = p.r8 <= 16;
    auto kern = wc == kWcMxfp4 ? (small_r ? fp8_gemm_kernel<128, 16, 2, kWcMxfp4> : fp8_gemm_kernel<128, 64, 2, kWcMxfp4>)
              : wc == kWcE4m3 ? (small_r ? fp8_gemm_kernel<128, 16, 2, kWcE4m3> : fp8_gemm_kernel<128, 64, 2, kWcE4m3>)
              : esz == 1 ? (BK == 128 ? (small_r ? fp8_gemm_kernel<128, 16, 1> : fp8_gemm_kernel<128, 64, 1>)
                                      : (small_r ? fp8_gemm_kernel<64, 16, 1> : fp8_gemm_kernel<64, 64, 1>))
                         : (BK == 128 ? (small_r ? fp8_gemm_kernel<128, 16, 2> : fp8_gemm_kernel<128, 64, 2>)
                                      : (small_r ? fp8_gemm_kernel<64, 16, 2> : fp8_gemm_kernel<64, 64, 2>));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, w4 ? kThreadsW4 : kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = device_sm_count();
    if (grid > p.units) grid = p.units;
    if (wc == kWcMxfp4)
        return small_r ? launch_t<128, 16, 2, kWcMxfp4>(p, tmW, tmX, tmB, smem, (int)grid, stream)
                       : launch_t<128, 64, 2, kWcMxfp4>(p, tmW, tmX, tmB, smem, (int)grid, stream);
    if (wc == kWcE4m3)
        return small_r ? launch_t<128, 16, 2, kWcE4m3>(p, tmW, tmX, tmB, smem, (int)grid, stream)
                       : launch_t<128, 64, 2, kWcE4m3>(p, tmW, tmX, tmB, smem, (int)grid, stream);
    if (esz == 2) {
        if (BK == 128)
            return small_r ? launch_t<128, 16, 2>(p, tmW, tmX, tmB, smem, (int)grid, stream)
                           : launch_t<128, 64, 2>(p, tmW, tmX, tmB, smem, (int)grid, stream);
        return small_r ? launch_t<64, 16, 2>(p, tmW, tmX, tmB, smem, (int)grid, stream)
                       : launch_t<64, 64, 2>(p, tmW, tmX, tmB, smem, (int)grid, stream);
    }
    if (BK == 128)
        return small_r ? launch_t<128, 16, 1>(p, tmW, tmX, tmB, smem, (int)grid, stream)
                       : launch_t<128, 64, 1>(p, tmW, tmX, tmB, smem, (int)grid, stream);
    return small_r ? launch_t<64, 16, 1>(p, tmW, tmX, tmB, smem, (int)grid, stream)
                   : launch_t<64, 64, 1>(p, tmW, tmX, tmB, smem, (int)grid, stream);
}

}  // namespace lora
