// api.cu -- the extern "C" entry points declared in include/lora.h.
// Host-side argument checks, workspace carving and stream-ordered launches;
// no allocation, no exceptions across the ABI.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "internal.h"
#include "lora.h"

using namespace lora;

namespace {

constexpr int kVersion = 1;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA; }

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// `parts` planes of fp32 v [n_slices][T][r_max] for lora_apply's two-launch path
size_t apply_v_bytes(int T, const lora_pool_t& pool, int parts)
{
    return (size_t)parts * pool.n_slices * T * pool.r_max * 4;
}

// Checks shared by every call that reads the pool.
int check_pool(const lora_pool_t* pool)
{
    if (!pool || !pool->A || !pool->B) return LORA_ERR_INVALID_ARG;
    if (pool->n_slices < 1 || pool->n_adapters < 1 || pool->h_in < 1 || pool->h_out < 1 ||
        pool->r_max < 1)
        return LORA_ERR_INVALID_ARG;
    if (pool->n_slices > 65535 || pool->n_adapters > LORA_MAX_ADAPTERS) return LORA_ERR_UNSUPPORTED;
    if (pool->r_max > LORA_MAX_RANK) return LORA_ERR_UNSUPPORTED;
    if (pool->h_in % 8 || pool->h_out % 8 || pool->r_max % 8) return LORA_ERR_INVALID_ARG;
    if (pool->r_max & (pool->r_max - 1)) return LORA_ERR_UNSUPPORTED;  // 8, 16, 32 or 64
    if (!aligned16(pool->A) || !aligned16(pool->B)) return LORA_ERR_INVALID_ARG;
    if ((long long)pool->n_slices * pool->n_adapters * pool->h_in >= (1ll << 31) ||
        (long long)pool->n_slices * pool->n_adapters * pool->r_max >= (1ll << 31))
        return LORA_ERR_UNSUPPORTED;
    return LORA_OK;
}

int check_segments(const lora_segments_t* seg, int n_adapters)
{
    if (!seg) return LORA_ERR_INVALID_ARG;
    if (seg->T < 0 || seg->n_adapters != n_adapters) return LORA_ERR_INVALID_ARG;
    if (!seg->indptr || !seg->active || !seg->tiles || !seg->counts) return LORA_ERR_INVALID_ARG;
    if (!aligned16(seg->tiles)) return LORA_ERR_INVALID_ARG;
    if (seg->T > 0 && (!seg->perm || !seg->tok_adapter)) return LORA_ERR_INVALID_ARG;
    return LORA_OK;
}

// GEMM workspace: status | xq (esz bytes per element) | sx | v (with a pool) |
// sync words | partials. [off_v, off_part) is zeroed by the quantiser on every call.
// Batches whose adapters are too many to fold into the GEMM's accumulator (more
// than kFuseMaxAdapters in the pool and in the batch), and batches of more than
// kFuseMaxTokens tokens (prefill: the down-projection of that many tokens on the
// epilogue warps costs more than the SGMV apply), run the base GEMM and then the SGMV
// apply instead (see gemm_lora_launch).
constexpr int kFuseMaxAdapters = 16;
constexpr int kFuseMaxTokens = 1024;
bool gemm_split(int M, const lora_pool_t* pool)
{
    return pool && ((pool->n_adapters > kFuseMaxAdapters && M > kFuseMaxAdapters) || M > kFuseMaxTokens);
}

size_t fp8_ws_layout(int M, int K, const lora_pool_t* pool, size_t* off_xq, size_t* off_sx,
                     size_t* off_v, size_t* off_sync, size_t* off_part, int esz = 1, size_t* off_order = nullptr)
{
    size_t off = 256;  // status word block
    *off_xq = off;
    off += align256((size_t)M * K * esz);
    *off_sx = off;
    off += align256((size_t)M * 4);
    *off_v = off;
    if (pool) off += align256((size_t)fp8_gemm_v_copies(M) * M * pool->r_max * 4);
    *off_sync = off;  // [0]: down-projection count, [16 ..]: one flag per SM
    off += align256((size_t)(16 + device_sm_count()) * 4);
    *off_part = off;
    off += align256(fp8_gemm_partial_bytes(M));
    if (off_order) *off_order = off;  // the split path's apply: tile rows in cost order, or
    if (gemm_split(M, pool)) {        // for long segments the tensor-core shrink's planes of v
        size_t o = sgmv_order_bytes(M, pool->n_adapters);
        if (sgmv_expand_tc_eligible(M, *pool)) {
            const size_t v = apply_v_bytes(M, *pool, sgmv_shrink_tc_parts(*pool));
            if (v > o) o = v;
        }
        off += align256(o);
    }
    return off;
}

// Backward workspace: the forward GEMM's workspace for (M, K' = N, the transposed
// pool) | A' = B^T [n_adapters][N][r_max] | B' = A^T [n_adapters][r_max][K] | u | v.
size_t bwd_ws_layout(int M, const lora_pool_t* pool, size_t* off_at, size_t* off_bt, size_t* off_u,
                     size_t* off_v)
{
    size_t a, b, c, d, e;
    size_t off = align256(fp8_ws_layout(M, pool->h_out, pool, &a, &b, &c, &d, &e));
    *off_at = off;
    off += align256((size_t)pool->n_adapters * pool->h_out * pool->r_max * 2);
    *off_bt = off;
    off += align256((size_t)pool->n_adapters * pool->r_max * pool->h_in * 2);
    *off_u = off;
    off += align256((size_t)M * pool->r_max * 4);
    *off_v = off;
    off += align256((size_t)M * pool->r_max * 4);
    return off;
}

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitNs};
std::atomic<int> g_inject_stall{0};

}  // namespace

namespace lora {

unsigned long long debug_wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
int debug_inject_stall() { return g_inject_stall.load(std::memory_order_relaxed); }

// Checks of fp8_gemm_lora_epilogue's arguments other than the workspace
// (shared with the entry point that allocates nothing, so both answer alike).
int fp8_gemm_check_args(const void* x, int M, int K, int N, const uint8_t* Wq, const float* w_scale,
                        const lora_pool_t* pool, const lora_segments_t* seg, const void* y)
{
    if (M < 1 || K < 16 || N < 8 || K % 16 || N % 8) return LORA_ERR_INVALID_ARG;
    if (!x || !Wq || !w_scale || !y) return LORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wq) || !aligned16(y)) return LORA_ERR_INVALID_ARG;
    if (M > (1 << 24)) return LORA_ERR_UNSUPPORTED;
    if (pool) {
        int st = check_pool(pool);
        if (st != LORA_OK) return st;
        if (pool->n_slices != 1 || pool->h_in != K || pool->h_out != N) return LORA_ERR_INVALID_ARG;
        if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
        if (seg->T != M) return LORA_ERR_INVALID_ARG;
    }
    return LORA_OK;
}

namespace {
// Both GEMM entry points after their argument checks. esz 1: E4M3 operands
// (x quantised per token); esz 2: bf16 operands (x copied in segment order).
int gemm_lora_launch(int esz, const void* x, int M, int K, int N, const uint8_t* Wq, const float* w_scale,
                     const lora_pool_t* pool, const lora_segments_t* seg, void* y, void* ws,
                     size_t ws_bytes, lora_stream_t stream, const uint8_t* wsc = nullptr, bool w_e4m3 = false)
{
    size_t off_xq, off_sx, off_v, off_sync, off_part, off_order;
    const size_t need =
        fp8_ws_layout(M, K, pool, &off_xq, &off_sx, &off_v, &off_sync, &off_part, esz, &off_order);
    if (!ws || ws_bytes < need || !aligned16(ws)) return LORA_ERR_WORKSPACE;
    const bool split = gemm_split(M, pool);
    const lora_pool_t* fused = split ? nullptr : pool;  // the adapters folded into the GEMM
    uint8_t* w = static_cast<uint8_t*>(ws);
    uint32_t* status = reinterpret_cast<uint32_t*>(w);
    uint8_t* xq = w + off_xq;
    float* sx = reinterpret_cast<float*>(w + off_sx);
    float* v = pool ? reinterpret_cast<float*>(w + off_v) : nullptr;
    int* sync = reinterpret_cast<int*>(w + off_sync);
    cudaStream_t s = (cudaStream_t)stream;

    // 1. activations -> E4M3 (or copied as bf16), rows in segment order when adapters
    //    are present; the same kernel zeroes v and the GEMM's synchronisation words
    cudaError_t e = launch_quantize_rows(x, fused ? seg->perm : nullptr, M, K, xq, sx, w + off_v,
                                         (off_part - off_v) / 4, s, esz == 2);
    if (e != cudaSuccess) return LORA_ERR_CUDA;
    // 2. the GEMM, a programmatic dependent of the quantiser: its weights start
    //    streaming at once, the down-projection runs in its epilogue warps meanwhile
    //    and the up-projection in its epilogue
    Fp8GemmArgs a = {};
    a.M = M;
    a.N = N;
    a.K = K;
    a.esz = esz;
    a.xq = xq;
    a.sx = sx;
    a.Wq = Wq;
    a.sw = w_scale;
    a.wsc = wsc;
    a.w_e4m3 = w_e4m3;
    a.y = static_cast<uint16_t*>(y);
    a.status = status;
    a.partials = reinterpret_cast<float*>(w + off_part);
    a.v_done = sync;
    a.flags = sync + 16;
    a.lora = fused != nullptr;
    if (fused) {
        a.perm = seg->perm;
        a.tok_adapter = seg->tok_adapter;
        a.indptr = seg->indptr;
        a.active = seg->active;
        a.counts = seg->counts;
        a.v = v;
        a.x = static_cast<const uint16_t*>(x);
        a.A = static_cast<const uint16_t*>(pool->A);
        a.B = static_cast<const uint16_t*>(pool->B);
        a.ranks = pool->ranks;
        a.scales = pool->scales;
        a.n_adapters = pool->n_adapters;
        a.r_max = pool->r_max;
    }
    e = launch_fp8_gemm(a, s);
    if (e != cudaSuccess || !split) return cuda_status(e);
    // 3. many adapters or tokens: their term added to the GEMM's bf16 output by the SGMV
    //    apply: for long segments the tensor-core shrink into planes of v (in the
    //    workspace) and the tensor-core expand, else the cluster kernel (a general batch's
    //    tile rows in cost order, in the workspace)
    if (sgmv_expand_tc_eligible(M, *pool)) {
        float* vp = reinterpret_cast<float*>(w + off_order);
        int planes = sgmv_shrink_tc_parts(*pool);
        e = launch_sgmv_shrink_tc(x, 0, *pool, *seg, vp, planes, s);
        if (e == cudaErrorInvalidValue) {  // the pool's tensor map was refused: the cluster shrink
            e = launch_sgmv(SGMV_SHRINK, x, 0, *pool, *seg, vp, nullptr, s, false);
            planes = 1;
        }
        if (e != cudaSuccess) return LORA_ERR_CUDA;
        return cuda_status(launch_sgmv_expand_tc(vp, planes, *pool, *seg, y, s));
    }
    void* order = tile_tokens_for(M, pool->n_adapters) > LORA_DECODE_TILE_TOKENS ? w + off_order : nullptr;
    return cuda_status(launch_sgmv(SGMV_APPLY, x, 0, *pool, *seg, nullptr, y, s, false, order));
}

}  // namespace

}  // namespace lora

extern "C" {

int lora_debug_set_wait_limit(uint64_t limit_ns, int inject_stall)
{
    if (limit_ns == 0) limit_ns = kDefaultWaitNs;
    if (limit_ns < 1000 || limit_ns > kDefaultWaitNs) return LORA_ERR_INVALID_ARG;
    if (inject_stall != 0 && inject_stall != 1) return LORA_ERR_INVALID_ARG;
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    g_inject_stall.store(inject_stall, std::memory_order_relaxed);
    return LORA_OK;
}

const char* lora_status_string(int s)
{
    switch (s) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARG: return "invalid argument";
    case LORA_ERR_UNSUPPORTED: return "unsupported shape";
    case LORA_ERR_BAD_ADAPTER_ID: return "adapter id outside [-1, n_adapters)";
    case LORA_ERR_CUDA: return "CUDA error";
    case LORA_ERR_WORKSPACE: return "workspace missing or too small";
    case LORA_ERR_TIMEOUT: return "a bounded device wait timed out";
    default: return "unknown status";
    }
}

int lora_version(void) { return kVersion; }

int lora_tile_tokens(void) { return LORA_TILE_TOKENS; }

int lora_tile_tokens_for(int T, int n_adapters)
{
    if (T < 0 || n_adapters < 1) return -1;
    return tile_tokens_for(T, n_adapters);
}

int lora_max_tiles(int T, int n_adapters)
{
    if (T < 0 || n_adapters < 1) return -1;
    return max_tiles_for(T, n_adapters);
}

int lora_segments_status(const lora_segments_t* seg, lora_stream_t stream, uint32_t* detail)
{
    if (!seg || !seg->counts) return LORA_ERR_INVALID_ARG;
    int32_t word = 0;
    int32_t* dev = seg->counts + kSegStatusSlot;
    cudaError_t e = cudaMemcpyAsync(&word, dev, sizeof(word), cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return LORA_ERR_CUDA;
    if (detail) *detail = (uint32_t)word;
    if (word) {
        e = cudaMemsetAsync(dev, 0, sizeof(int32_t), (cudaStream_t)stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
        if (e != cudaSuccess) return LORA_ERR_CUDA;
        return (word & kSegTooLarge) ? LORA_ERR_INVALID_ARG : LORA_ERR_TIMEOUT;
    }
    return LORA_OK;
}

size_t lora_workspace_size(int op, int T, int K, const lora_pool_t* pool)
{
    if (T < 0) return (size_t)-1;
    switch (op) {
    case LORA_OP_SHRINK:
    case LORA_OP_EXPAND: return 0;
    case LORA_OP_APPLY:
        // v stays on chip; a general batch's tile rows in cost order (optional workspace)
        if (!pool || check_pool(pool) != LORA_OK) return (size_t)-1;
        if (T == 0 || tile_tokens_for(T, pool->n_adapters) <= LORA_DECODE_TILE_TOKENS) return 0;
        // long segments: v through the workspace (shrink, then the tensor-core expand)
        if (sgmv_expand_tc_eligible(T, *pool)) {
            const size_t v = apply_v_bytes(T, *pool, sgmv_shrink_tc_parts(*pool));
            const size_t o = sgmv_order_bytes(T, pool->n_adapters);
            return align256(v > o ? v : o);
        }
        return align256(sgmv_order_bytes(T, pool->n_adapters));
    case LORA_OP_FP8_BACKWARD: {
        if (!pool || check_pool(pool) != LORA_OK || T < 1) return (size_t)-1;
        size_t a, b, c, d;
        return bwd_ws_layout(T, pool, &a, &b, &c, &d);
    }
    case LORA_OP_FP8_GEMM:
    case LORA_OP_BF16_GEMM:
    case LORA_OP_MXFP4_GEMM:
    case LORA_OP_W8A16_GEMM: {
        if (K <= 0) return (size_t)-1;
        if (pool && check_pool(pool) != LORA_OK) return (size_t)-1;
        if (T < 1) return (size_t)-1;
        size_t a, b, c, d, e;
        return fp8_ws_layout(T, K, pool, &a, &b, &c, &d, &e, op == LORA_OP_FP8_GEMM ? 1 : 2);
    }
    default: return (size_t)-1;
    }
}

int lora_workspace_init(void* ws, size_t ws_bytes, lora_stream_t stream)
{
    if (!ws || ws_bytes == 0) return LORA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

int lora_workspace_status(void* ws, size_t ws_bytes, lora_stream_t stream, uint32_t* detail)
{
    if (!ws || ws_bytes < 256) return LORA_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return LORA_ERR_CUDA;
    if (detail) *detail = word;
    if (word) {
        e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), (cudaStream_t)stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
        if (e != cudaSuccess) return LORA_ERR_CUDA;
        return LORA_ERR_TIMEOUT;
    }
    return LORA_OK;
}

int lora_build_segments(const int32_t* ids, int T, int n_adapters, const lora_segments_t* seg,
                        int sync_check, lora_stream_t stream)
{
    if (T < 0 || n_adapters < 1) return LORA_ERR_INVALID_ARG;
    if (n_adapters > LORA_MAX_ADAPTERS || T >= (1 << 30)) return LORA_ERR_UNSUPPORTED;
    if (T > 0 && !ids) return LORA_ERR_INVALID_ARG;
    int st = check_segments(seg, n_adapters);
    if (st != LORA_OK) return st;
    if (seg->T != T) return LORA_ERR_INVALID_ARG;
    cudaError_t e = launch_build_segments(ids, T, n_adapters, *seg, (cudaStream_t)stream);
    if (e != cudaSuccess) return LORA_ERR_CUDA;
    if (sync_check) {
        int32_t counts[4];
        e = cudaMemcpyAsync(counts, seg->counts, sizeof(counts), cudaMemcpyDeviceToHost,
                            (cudaStream_t)stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
        if (e != cudaSuccess) return LORA_ERR_CUDA;
        if (counts[2] != 0) return LORA_ERR_BAD_ADAPTER_ID;
    }
    return LORA_OK;
}

static int check_x(const void* x, int64_t x_slice_stride, const lora_pool_t* pool, int T)
{
    if (!x || !aligned16(x)) return LORA_ERR_INVALID_ARG;
    if (x_slice_stride < 0 || x_slice_stride % 8) return LORA_ERR_INVALID_ARG;
    if (x_slice_stride != 0 && x_slice_stride < (int64_t)T * pool->h_in) return LORA_ERR_INVALID_ARG;
    return LORA_OK;
}

int lora_shrink(const void* x, int64_t x_slice_stride, const lora_pool_t* pool,
                const lora_segments_t* seg, float* v, void* ws, size_t ws_bytes,
                lora_stream_t stream)
{
    (void)ws;
    (void)ws_bytes;
    int st = check_pool(pool);
    if (st != LORA_OK) return st;
    if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
    if (seg->T == 0) return LORA_OK;
    if ((st = check_x(x, x_slice_stride, pool, seg->T)) != LORA_OK) return st;
    if (!v || !aligned16(v)) return LORA_ERR_INVALID_ARG;
    return cuda_status(launch_sgmv(SGMV_SHRINK, x, x_slice_stride, *pool, *seg, v, nullptr,
                                   (cudaStream_t)stream, false));
}

int lora_expand(const float* v, const lora_pool_t* pool, const lora_segments_t* seg, void* y,
                void* ws, size_t ws_bytes, lora_stream_t stream)
{
    (void)ws;
    (void)ws_bytes;
    int st = check_pool(pool);
    if (st != LORA_OK) return st;
    if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
    if (seg->T == 0) return LORA_OK;
    if (!v || !aligned16(v) || !y || !aligned16(y)) return LORA_ERR_INVALID_ARG;
    if (sgmv_expand_tc_eligible(seg->T, *pool))  // long segments: the tensor-core expand
        return cuda_status(launch_sgmv_expand_tc(v, 1, *pool, *seg, y, (cudaStream_t)stream));
    return cuda_status(launch_sgmv(SGMV_EXPAND, nullptr, 0, *pool, *seg, const_cast<float*>(v), y,
                                   (cudaStream_t)stream, false));
}

int lora_apply(const void* x, int64_t x_slice_stride, const lora_pool_t* pool,
               const lora_segments_t* seg, void* y, void* ws, size_t ws_bytes,
               lora_stream_t stream)
{
    int st = check_pool(pool);
    if (st != LORA_OK) return st;
    if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
    if (seg->T == 0) return LORA_OK;
    if ((st = check_x(x, x_slice_stride, pool, seg->T)) != LORA_OK) return st;
    if (!y || !aligned16(y)) return LORA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    // one tile row per thread-block cluster, v exchanged on chip; with a workspace, a
    // general batch's tile rows run in descending cost (a small ordering kernel first)
    // long segments with room for v in the workspace: the shrink into planes of v (on the
    // tensor cores; with room for one plane only, or if the pool's tensor map is refused,
    // the cluster shrink), then the tensor-core expand as its programmatic dependent
    if (ws && sgmv_expand_tc_eligible(seg->T, *pool) && ws_bytes >= apply_v_bytes(seg->T, *pool, 1) &&
        aligned16(ws)) {
        float* v = static_cast<float*>(ws);
        const int parts = sgmv_shrink_tc_parts(*pool);
        int planes = 0;
        if (ws_bytes >= apply_v_bytes(seg->T, *pool, parts)) {
            const cudaError_t e = launch_sgmv_shrink_tc(x, x_slice_stride, *pool, *seg, v, parts, s);
            if (e == cudaSuccess) planes = parts;
            else if (e != cudaErrorInvalidValue) return cuda_status(e);
        }
        if (planes == 0) {
            const cudaError_t e = launch_sgmv(SGMV_SHRINK, x, x_slice_stride, *pool, *seg, v, nullptr, s, false);
            if (e != cudaSuccess) return cuda_status(e);
            planes = 1;
        }
        return cuda_status(launch_sgmv_expand_tc(v, planes, *pool, *seg, y, s));
    }
    void* order = nullptr;
    if (ws && tile_tokens_for(seg->T, pool->n_adapters) > LORA_DECODE_TILE_TOKENS) {
        if (ws_bytes < sgmv_order_bytes(seg->T, pool->n_adapters) || !aligned16(ws)) return LORA_ERR_WORKSPACE;
        order = ws;
    }
    return cuda_status(launch_sgmv(SGMV_APPLY, x, x_slice_stride, *pool, *seg, nullptr, y, s, false, order));
}

int fp8_quantize_rows(const void* x, int M, int K, uint8_t* xq, float* sx, lora_stream_t stream)
{
    if (M < 0 || K <= 0 || K % 16) return LORA_ERR_INVALID_ARG;
    if (M == 0) return LORA_OK;
    if (!x || !xq || !sx || !aligned16(x) || !aligned16(xq)) return LORA_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_rows(x, nullptr, M, K, xq, sx, nullptr, 0, (cudaStream_t)stream));
}

int fp8_gemm_lora_epilogue(const void* x, int M, int K, int N, const uint8_t* Wq,
                           const float* w_scale, const lora_pool_t* pool,
                           const lora_segments_t* seg, void* y, void* ws, size_t ws_bytes,
                           lora_stream_t stream)
{
    const int st = fp8_gemm_check_args(x, M, K, N, Wq, w_scale, pool, seg, y);
    if (st != LORA_OK) return st;
    return gemm_lora_launch(1, x, M, K, N, Wq, w_scale, pool, seg, y, ws, ws_bytes, stream);
}

int fp8_lora_backward(const void* x, const void* dY, int M, int K, int N, const uint8_t* WqT,
                      const float* swT, const lora_pool_t* pool, const lora_segments_t* seg, void* dX,
                      float* dA, float* dB, void* ws, size_t ws_bytes, lora_stream_t stream)
{
    int st = check_pool(pool);
    if (st != LORA_OK) return st;
    if (pool->n_slices != 1 || pool->h_in != K || pool->h_out != N) return LORA_ERR_INVALID_ARG;
    if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
    if (M < 1 || seg->T != M || K % 8 || N % 16 || K < 8 || N < 16) return LORA_ERR_INVALID_ARG;
    if (M > (1 << 24)) return LORA_ERR_UNSUPPORTED;
    if (!x || !dY || !WqT || !swT || !dX || !dA || !dB) return LORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dY) || !aligned16(WqT) || !aligned16(dX) || !aligned16(dA) ||
        !aligned16(dB))
        return LORA_ERR_INVALID_ARG;
    size_t off_at, off_bt, off_u, off_v;
    const size_t need = bwd_ws_layout(M, pool, &off_at, &off_bt, &off_u, &off_v);
    if (!ws || ws_bytes < need || !aligned16(ws)) return LORA_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t s = (cudaStream_t)stream;
    // the transposed pool: A' = B^T (h_in' = N), B' = A^T (h_out' = K)
    lora_pool_t pt = *pool;
    pt.A = w + off_at;
    pt.B = w + off_bt;
    pt.h_in = N;
    pt.h_out = K;
    float* u = reinterpret_cast<float*>(w + off_u);
    float* v = reinterpret_cast<float*>(w + off_v);
    const size_t na = (size_t)pool->n_adapters;
    // 1. the gradients of adapters without tokens are zero
    if (cudaMemsetAsync(dA, 0, na * K * pool->r_max * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dB, 0, na * pool->r_max * N * 4, s) != cudaSuccess)
        return LORA_ERR_CUDA;
    // 2. A' = B^T and B' = A^T of the active adapters
    if (launch_transpose_pool(*pool, *seg, const_cast<void*>(pt.A), const_cast<void*>(pt.B), s) != cudaSuccess)
        return LORA_ERR_CUDA;
    // 3. dX = dY.W + s (dY.B^T).A^T: the forward's fused 8-bit GEMM of dY with W^T
    //    (quantised per input channel) and the transposed pool; its workspace leads
    st = gemm_lora_launch(1, dY, M, N, K, WqT, swT, &pt, seg, dX, w, off_at, stream);
    if (st != LORA_OK) return st;
    // 4. u = dY.B^T per token: the GEMM's own down-projection when it folded the adapters
    //    into its accumulator (summed from its workspace copies), else a shrink of dY
    cudaError_t eu;
    if (!gemm_split(M, &pt)) {
        size_t g_xq, g_sx, g_v, g_sync, g_part;
        fp8_ws_layout(M, N, &pt, &g_xq, &g_sx, &g_v, &g_sync, &g_part, 1);
        eu = launch_gather_u(reinterpret_cast<const float*>(w + g_v), fp8_gemm_v_copies(M), *seg, M, pool->r_max, u, s);
    } else {
        eu = launch_sgmv(SGMV_SHRINK, dY, 0, pt, *seg, u, nullptr, s, false);
    }
    if (eu != cudaSuccess) return LORA_ERR_CUDA;
    // 5. v = x.A per token, then dA = s x^T u and dB = s v^T dY per adapter
    if (launch_sgmv(SGMV_SHRINK, x, 0, *pool, *seg, v, nullptr, s, false) != cudaSuccess ||
        launch_grad_outer(true, x, u, K, *pool, *seg, dA, s) != cudaSuccess ||
        launch_grad_outer(false, dY, v, N, *pool, *seg, dB, s) != cudaSuccess)
        return LORA_ERR_CUDA;
    return LORA_OK;
}

int lora_switch_merge(const void* W, int N, int K, const lora_pool_t* pool, const int32_t* sel,
                      const float* gates, int n_sel, void* W_out, lora_stream_t stream)
{
    int st = check_pool(pool);
    if (st != LORA_OK) return st;
    if (N < 8 || K < 8 || N % 8 || K % 8 || n_sel < 1) return LORA_ERR_INVALID_ARG;
    if (pool->n_slices != 1 || pool->h_in != K || pool->h_out != N) return LORA_ERR_INVALID_ARG;
    if (!W || !W_out || !sel || !gates || !aligned16(W) || !aligned16(W_out)) return LORA_ERR_INVALID_ARG;
    if (n_sel > LORA_SWITCH_MAX_SELECTED || n_sel * ((pool->r_max + 15) / 16 * 16) > LORA_SWITCH_MAX_RANK_SUM)
        return LORA_ERR_UNSUPPORTED;
    // in place or disjoint: a partly overlapping output would be read after it is written
    const uintptr_t a0 = (uintptr_t)W, b0 = (uintptr_t)W_out, len = (uintptr_t)N * K * 2;
    if (a0 != b0 && a0 < b0 + len && b0 < a0 + len) return LORA_ERR_INVALID_ARG;
    return cuda_status(launch_lora_switch_merge(W, N, K, *pool, sel, gates, n_sel, W_out, (cudaStream_t)stream));
}

int w8a16_gemm_lora_epilogue(const void* x, int M, int K, int N, const uint8_t* Wq, const float* w_scale,
                             const lora_pool_t* pool, const lora_segments_t* seg, void* y, void* ws,
                             size_t ws_bytes, lora_stream_t stream)
{
    if (M < 1 || K < 64 || N < 8 || K % 64 || N % 8) return LORA_ERR_INVALID_ARG;
    if (!x || !Wq || !w_scale || !y) return LORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wq) || !aligned16(y)) return LORA_ERR_INVALID_ARG;
    if (M > (1 << 24)) return LORA_ERR_UNSUPPORTED;
    if (pool) {
        int st = check_pool(pool);
        if (st != LORA_OK) return st;
        if (pool->n_slices != 1 || pool->h_in != K || pool->h_out != N) return LORA_ERR_INVALID_ARG;
        if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
        if (seg->T != M) return LORA_ERR_INVALID_ARG;
    }
    return gemm_lora_launch(2, x, M, K, N, Wq, w_scale, pool, seg, y, ws, ws_bytes, stream, nullptr, true);
}

int mxfp4_quantize_rows(const void* W, int N, int K, uint8_t* Wp, uint8_t* Wsc, lora_stream_t stream)
{
    if (N < 1 || K < 64 || K % 64) return LORA_ERR_INVALID_ARG;
    if (!W || !Wp || !Wsc || !aligned16(W) || !aligned16(Wp) || !aligned16(Wsc)) return LORA_ERR_INVALID_ARG;
    return cuda_status(launch_mxfp4_quantize(W, N, K, Wp, Wsc, (cudaStream_t)stream));
}

int mxfp4_gemm_lora_epilogue(const void* x, int M, int K, int N, const uint8_t* Wp, const uint8_t* Wsc,
                             const lora_pool_t* pool, const lora_segments_t* seg, void* y, void* ws,
                             size_t ws_bytes, lora_stream_t stream)
{
    if (M < 1 || K < 64 || N < 8 || K % 64 || N % 8) return LORA_ERR_INVALID_ARG;
    if (!x || !Wp || !Wsc || !y) return LORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wp) || !aligned16(Wsc) || !aligned16(y)) return LORA_ERR_INVALID_ARG;
    if (M > (1 << 24)) return LORA_ERR_UNSUPPORTED;
    if (pool) {
        int st = check_pool(pool);
        if (st != LORA_OK) return st;
        if (pool->n_slices != 1 || pool->h_in != K || pool->h_out != N) return LORA_ERR_INVALID_ARG;
        if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
        if (seg->T != M) return LORA_ERR_INVALID_ARG;
    }
    return gemm_lora_launch(2, x, M, K, N, Wp, nullptr, pool, seg, y, ws, ws_bytes, stream, Wsc);
}

int bf16_gemm_lora_epilogue(const void* x, int M, int K, int N, const void* W,
                            const lora_pool_t* pool, const lora_segments_t* seg, void* y,
                            void* ws, size_t ws_bytes, lora_stream_t stream)
{
    if (M < 1 || K < 8 || N < 8 || K % 8 || N % 8) return LORA_ERR_INVALID_ARG;
    if (!x || !W || !y) return LORA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W) || !aligned16(y)) return LORA_ERR_INVALID_ARG;
    if (M > (1 << 24)) return LORA_ERR_UNSUPPORTED;
    if (pool) {
        int st = check_pool(pool);
        if (st != LORA_OK) return st;
        if (pool->n_slices != 1 || pool->h_in != K || pool->h_out != N) return LORA_ERR_INVALID_ARG;
        if ((st = check_segments(seg, pool->n_adapters)) != LORA_OK) return st;
        if (seg->T != M) return LORA_ERR_INVALID_ARG;
    }
    return gemm_lora_launch(2, x, M, K, N, static_cast<const uint8_t*>(W), nullptr, pool, seg, y, ws,
                            ws_bytes, stream);
}

}  // extern "C"
