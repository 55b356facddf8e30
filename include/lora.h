/*
 * lora.h -- C ABI of liblora, the multi-tenant LoRA hot path on B200 (sm_100a).
 *
 * The problem (Punica README, section "How?"): a base weight W and, for n
 * adapters, LoRA matrices A_i [h_in, r_i] and B_i [r_i, h_out]. A batch X of
 * tokens maps token by token to adapters, and the output is
 *     Y = X.W + (x_1.A_1.B_1, ..., x_n.A_n.B_n),
 * here with a per-adapter scale s_i on the added term. Every token carries an
 * adapter id; -1 means "base model only" (EpiLoRA abstract, sentence 1: one
 * base copy serves the requests of many tenants, each with its own adapter).
 * The added term is computed as a shrink, v = x.A_i (rank r_i, fp32), and an
 * expand, y += s_i.v.B_i: SGMV for runs of tokens that share an adapter, BGMV
 * for one adapter per decode token (Punica README, "How?": Segmented Gather
 * Matrix-Vector multiplication). fp8_gemm_lora_epilogue() fuses the expand
 * into the epilogue of an 8-bit base GEMM whose down-projection is launched
 * first while the GEMM streams its weights (EpiLoRA abstract, sentences 3-4).
 *
 * Conventions for every call:
 *   - All array arguments are DEVICE pointers owned by the caller, unless a
 *     comment says "host". The library never allocates device memory; calls
 *     that need scratch space take a caller-owned workspace whose size comes
 *     from lora_workspace_size() (the Punica README's file listing records the
 *     same choice for SGMV: "use preallocated buffer").
 *   - bf16 arrays hold IEEE bfloat16 bit patterns; "e4m3" arrays hold OCP FP8
 *     E4M3 codes. Matrices are row-major with the last index contiguous.
 *   - Calls are ordered on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return once the work is enqueued. Errors that the host can
 *     see (NULL pointers, bad sizes, misalignment, unsupported shapes, launch
 *     failures) are returned before or instead of any launch; nothing is
 *     thrown across the ABI.
 *   - Pointers to bf16/e4m3/fp32 arrays must be 16-byte aligned, and every row
 *     length in bytes a multiple of 16 (so h_in, h_out, r_max, K must be
 *     multiples of 8 for bf16 rows, K a multiple of 16 for e4m3 rows).
 *   - Adapter ids outside [-1, n_adapters) are counted as bad and served as
 *     -1 (see lora_build_segments).
 */
#ifndef LORA_H_
#define LORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

struct CUstream_st;
typedef struct CUstream_st* lora_stream_t; /* same object as cudaStream_t */

typedef enum {
    LORA_OK = 0,
    LORA_ERR_INVALID_ARG = 1,    /* NULL pointer, size <= 0, misaligned pointer/stride */
    LORA_ERR_UNSUPPORTED = 2,    /* shape outside the implemented limits below */
    LORA_ERR_BAD_ADAPTER_ID = 3, /* sync_check found ids outside [-1, n_adapters) */
    LORA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
    LORA_ERR_WORKSPACE = 5,      /* workspace NULL or smaller than lora_workspace_size() */
    LORA_ERR_TIMEOUT = 6         /* a bounded device-side wait gave up (see lora_workspace_status) */
} lora_status_t;

/* Implemented limits. */
#define LORA_TILE_TOKENS 64    /* tokens per work tile of one adapter segment */
#define LORA_DECODE_TILE_TOKENS 4  /* the same in a decode-like batch (lora_tile_tokens_for) */
#define LORA_DECODE_MAX_TOKENS 64  /* largest batch that can count as decode-like */
#define LORA_MAX_RANK 64       /* largest r_max */
#define LORA_MAX_ADAPTERS 16384
#define LORA_SWITCH_MAX_SELECTED 8    /* adapters one lora_switch_merge may merge */
#define LORA_SWITCH_MAX_RANK_SUM 256  /* n_sel * round_up(r_max, 16) */

/*
 * Stacked adapter pool (the pages' per-adapter A_i, B_i, stacked; the
 * `n_slices` dimension holds several projections that share the token ids,
 * e.g. q/k/v/o of one layer, applied in one call).
 *   A      bf16 [n_slices][n_adapters][h_in][r_max]
 *   B      bf16 [n_slices][n_adapters][r_max][h_out]
 *   r_max  the padded rank of the pool: 8, 16, 32 or 64.
 *   ranks  int32 [n_adapters], each in 1..r_max; NULL = every adapter has rank r_max.
 *          Entries of A with column >= r_i and of B with row >= r_i are never read.
 *   scales fp32 [n_adapters] (s_i); NULL = 1.0.
 */
typedef struct {
    const void* A;
    const void* B;
    const int32_t* ranks;
    const float* scales;
    int32_t n_slices;
    int32_t n_adapters;
    int32_t h_in;
    int32_t h_out;
    int32_t r_max;
} lora_pool_t;

/*
 * Token grouping produced by lora_build_segments (device arrays, caller-owned,
 * filled by the call). For a batch of T tokens:
 *   perm        int32 [T]: token indices with a valid id, by ascending id and
 *               ascending token index within an id; then the tokens without an
 *               adapter, ascending.
 *   indptr      int32 [n_adapters+1]: adapter a owns perm[indptr[a] .. indptr[a+1]);
 *               indptr[n_adapters] = number of tokens with an adapter.
 *   active      int32 [n_adapters]: ids with >= 1 token, ascending; -1 after n_active.
 *   tiles       int32 [lora_max_tiles(T, n_adapters)][4]: every active segment
 *               cut, in order, into runs of at most
 *               lora_tile_tokens_for(T, n_adapters) tokens:
 *               {adapter, first position in perm, token count, segment index};
 *               the rows after the last run are {-1, 0, 0, -1}. One row is one
 *               unit of work of the SGMV kernels.
 *   tok_adapter int32 [T]: the id each token is served with (-1: none or bad id).
 *   counts      int32 [8]: n_valid, n_active, n_bad_ids, n_tiles, then a device
 *               status word (0 = ok; set by a kernel using these segments whose
 *               bounded wait gave up, see lora_segments_status) and 3 reserved.
 * T and n_adapters are host values describing the arrays.
 */
typedef struct {
    int32_t* perm;
    int32_t* indptr;
    int32_t* active;
    int32_t* tiles;
    int32_t* tok_adapter;
    int32_t* counts;
    int32_t T;
    int32_t n_adapters;
} lora_segments_t;

/*
 * Read and clear the status word of a segments object (counts[4]):
 * synchronises `stream`; LORA_OK, or LORA_ERR_TIMEOUT if an SGMV kernel that
 * used these segments gave up on a bounded wait, or LORA_ERR_INVALID_ARG if a
 * tile held more tokens than lora_tile_tokens_for(T, n_adapters) allows (the
 * tiles were not built by lora_build_segments for these sizes); the output is
 * then undefined. *detail (host, may be NULL) receives the raw word. The word
 * is also cleared by every lora_build_segments on the same object.
 */
LORA_API int lora_segments_status(const lora_segments_t* seg, lora_stream_t stream, uint32_t* detail);

/* Operation codes for lora_workspace_size. */
#define LORA_OP_SHRINK 0
#define LORA_OP_EXPAND 1
#define LORA_OP_APPLY 2
#define LORA_OP_FP8_GEMM 3
#define LORA_OP_BF16_GEMM 4
#define LORA_OP_FP8_BACKWARD 5
#define LORA_OP_MXFP4_GEMM 6
#define LORA_OP_W8A16_GEMM 7

/*
 * Bytes of workspace an operation needs (0 if it needs none), or (size_t)-1
 * for invalid arguments. For LORA_OP_FP8_GEMM, T is the
 * token count M and `K` the GEMM's reduction size; `pool` may be NULL (no
 * LoRA). LORA_OP_APPLY needs a valid pool. It returns:
 *   0 for a decode-like batch (lora_tile_tokens_for);
 *   for a batch of long segments (T >= 32 * n_adapters, h_out >= 128), the bytes of
 *   P = min(8, ceil(h_in / 64)) planes of fp32 v (P * n_slices * T * r_max * 4,
 *   at least the tile-order bytes, rounded up to 256; see lora_apply);
 *   otherwise the bytes of the tile rows in cost order (16 per row of
 *   lora_max_tiles). The other operations ignore K.
 * A workspace must be zeroed once after allocation (lora_workspace_init);
 * afterwards the library keeps it in a reusable state.
 */
LORA_API size_t lora_workspace_size(int op, int T, int K, const lora_pool_t* pool);

/* Zero a freshly allocated workspace (stream-ordered memset). */
LORA_API int lora_workspace_init(void* ws, size_t ws_bytes, lora_stream_t stream);

/*
 * Read and clear the device status word of a workspace: synchronises
 * `stream`, returns LORA_OK, or LORA_ERR_TIMEOUT if a kernel that used this
 * workspace gave up on a bounded wait since the last query (its output is
 * then undefined). *detail (host, may be NULL) receives the raw status word.
 */
LORA_API int lora_workspace_status(void* ws, size_t ws_bytes, lora_stream_t stream, uint32_t* detail);

/*
 * Group the tokens of one batch by adapter (the segments of SGMV; Punica
 * README, "How?"). ids int32 [T] (device). Fills every array of *seg, whose
 * T and n_adapters must equal the arguments. One single-CTA kernel: a stable
 * counting sort, bit-exact and deterministic. Built once per batch and shared
 * by every layer and projection of that batch.
 * sync_check != 0: synchronise the stream and return LORA_ERR_BAD_ADAPTER_ID if
 * any id was outside [-1, n_adapters). Without it, bad ids are only counted
 * (counts[2]) and served as -1.
 * T may be 0 (every output describes an empty batch). Limits: n_adapters <=
 * LORA_MAX_ADAPTERS, T < 2^30.
 */
LORA_API int lora_build_segments(const int32_t* ids, int T, int n_adapters, const lora_segments_t* seg,
                        int sync_check, lora_stream_t stream);

/*
 * Shrink (down-projection; the x_i.A_i half of the added term in the Punica
 * README, "How?"), for every slice s and token t with adapter a:
 *   v[s][t][j] = sum_k x[s][t][k] * A[s][a][k][j]   for j < r_a  (fp32 accumulate)
 *   v[s][t][j] = 0                                    for r_a <= j < r_max.
 * Rows of tokens without an adapter are not written.
 *   x  bf16 [n_slices][T][h_in], slice s at x + s * x_slice_stride elements
 *      (x_slice_stride = 0 lets all slices share one x; otherwise >= T*h_in and
 *      a multiple of 8).
 *   v  fp32 [n_slices][T][r_max].
 * Needs no workspace (ws may be NULL, ws_bytes 0). One kernel launch.
 */
LORA_API int lora_shrink(const void* x, int64_t x_slice_stride, const lora_pool_t* pool,
                const lora_segments_t* seg, float* v, void* ws, size_t ws_bytes,
                lora_stream_t stream);

/*
 * Expand (up-projection; the (x_i.A_i).B_i half of the added term in the
 * Punica README, "How?", added to the base output), in place on y, for every
 * slice s and token t with adapter a:
 *   y[s][t][n] = bf16( fp32(y[s][t][n]) + s_a * sum_{j < r_a} v[s][t][j] * B[s][a][j][n] )
 * (one rounding, to nearest even); rows of tokens without an adapter are untouched.
 *   v  fp32 [n_slices][T][r_max];  y bf16 [n_slices][T][h_out] (in/out).
 * Needs no workspace. One kernel launch: for a batch of long segments (not
 * decode-like, T >= 32 * n_adapters, h_out >= 128) the tcgen05 expand (the
 * 128-column blocks of every tile row as MMAs with B_a read in place by TMA
 * and v split into bf16 halves hi + lo, so ~16 bits of v; the grid's CTAs
 * take equal runs of (tile row, slice, block)), else the cluster SGMV kernel.
 */
LORA_API int lora_expand(const float* v, const lora_pool_t* pool, const lora_segments_t* seg, void* y,
                void* ws, size_t ws_bytes, lora_stream_t stream);

/*
 * Shrink then expand (y += s_a * (x.A_a).B_a; the whole added term of the
 * Punica README, "How?", for a batch of many adapters), v in fp32. Arguments
 * as lora_shrink / lora_expand, plus an optional workspace of
 * lora_workspace_size(LORA_OP_APPLY, T, 0, pool) bytes. The SGMV kernel: each
 * thread-block cluster takes one tile row (lora_tile_tokens_for) and keeps its
 * v on chip, the partial v of its CTAs exchanged through distributed shared
 * memory. With a workspace (ws != NULL, ws_bytes at least that size, 16-byte
 * aligned, else LORA_ERR_WORKSPACE), a batch that is not decode-like and whose
 * tile rows times slices exceed two per SM first runs a one-CTA kernel that writes
 * its tile rows into ws in descending cost (rows of more than four tokens, then
 * by descending rank), so that the long rows start first; the results are the
 * same either way. ws NULL: one launch, table order.
 * A batch of long segments (as for lora_expand's tensor-core path) with a
 * workspace of lora_workspace_size(LORA_OP_APPLY, ...) bytes instead runs two
 * launches. First the tcgen05 shrink writes P = min(8, ceil(h_in / 64)) planes
 * of fp32 v [n_slices][T][r_max] into the workspace, each the sum over one
 * part of h_in. Then the tcgen05 expand, as its programmatic dependent, adds
 * the planes in plane order (deterministic) and applies the term. The results
 * equal the one-launch path's up to fp32 rounding order.
 * With a workspace of one plane (n_slices * T * r_max * 4 bytes), the cluster
 * shrink writes v and the tensor-core expand follows. With a smaller workspace
 * (at least the tile-order bytes), such a batch takes the cluster kernel.
 */
LORA_API int lora_apply(const void* x, int64_t x_slice_stride, const lora_pool_t* pool,
               const lora_segments_t* seg, void* y, void* ws, size_t ws_bytes,
               lora_stream_t stream);

/*
 * Per-row FP8 quantisation (the activation step of the 8-bit GEMM; also used
 * offline for weights with one scale per output channel):
 *   sx[m] = fl32(amax_k |x[m][k]| / 448), or 1 if the row is all zero;
 *   xq[m][k] = E4M3(fl32(x[m][k] / sx[m])), round to nearest even, saturating.
 *   x bf16 [M][K]; xq e4m3 [M][K]; sx fp32 [M]. One kernel launch.
 */
LORA_API int fp8_quantize_rows(const void* x, int M, int K, uint8_t* xq, float* sx, lora_stream_t stream);

/*
 * 8-bit base GEMM with the LoRA expand fused into its epilogue (EpiLoRA
 * abstract, sentences 3-4):
 *   y[m][n] = bf16( sx[m] * w_scale[n] * sum_k xq[m][k] * Wq[n][k]
 *                   + s_a * sum_{j < r_a} v[m][j] * B[0][a][j][n] ),
 *   a = seg->tok_adapter[m]; the LoRA term is absent when a == -1 or pool == NULL;
 *   xq, sx: x quantised per token as in fp8_quantize_rows;
 *   v = x.A_a in fp32 from the unquantised bf16 x (as lora_shrink).
 * Two launches: the activation quantiser, then the GEMM as its programmatic
 * dependent. The GEMM's mainloop starts streaming Wq at once. Its epilogue
 * warps compute the down-projection v meanwhile; the page runs it first as a
 * separate shrink. Each CTA waits for the whole v only before its first
 * epilogue.
 *   x bf16 [M][K]; Wq e4m3 [N][K]; w_scale fp32 [N]; y bf16 [M][N] (out).
 *   pool: NULL for the base GEMM alone; else n_slices == 1, h_in == K, h_out == N.
 *   seg: required when pool != NULL (built for these M tokens); may be NULL otherwise.
 *   ws: lora_workspace_size(LORA_OP_FP8_GEMM, M, K, pool) bytes.
 * Limits: K % 16 == 0, N % 8 == 0, M >= 1.
 * Many adapters or tokens: when the pool holds more than 16 adapters and
 * M > 16, or M > 1024, the adapters' term is not folded into the GEMM's
 * accumulator; the call runs the base GEMM and then the SGMV apply of
 * lora_apply on its output, so y = bf16(bf16(base) + term). That is three or
 * four launches: the workspace holds the apply's tile order, or, for a batch
 * of long segments (M >= 32 * n_adapters), the tensor-core shrink's planes of
 * v, followed by the tensor-core expand.
 * The GEMM is a persistent grid of one CTA per SM whose CTAs wait on one
 * another (the down-projection count, stream-K partials), so all of them must
 * be resident at once: the context needs every SM of the device. Where fewer
 * are available (an MPS share, a green context, another kernel holding SMs
 * for long), the waits give up after 2 s and lora_workspace_status reports
 * LORA_ERR_TIMEOUT.
 */
LORA_API int fp8_gemm_lora_epilogue(const void* x, int M, int K, int N, const uint8_t* Wq,
                           const float* w_scale, const lora_pool_t* pool,
                           const lora_segments_t* seg, void* y, void* ws, size_t ws_bytes,
                           lora_stream_t stream);

/*
 * 16-bit base GEMM with the same fused LoRA term (the EpiLoRA abstract,
 * sentences 3-4, for the engine that keeps activations and weights in 16
 * bits, sentence 6):
 *   y[m][n] = bf16( sum_k x[m][k] * W[n][k]
 *                   + s_a * sum_{j < r_a} v[m][j] * B[0][a][j][n] ),
 *   v = x.A_a in fp32, a = seg->tok_adapter[m] (no term for -1 or pool == NULL).
 * The same kernel as fp8_gemm_lora_epilogue with bf16 tensor-core operands
 * (tcgen05 kind::f16, fp32 accumulation in TMEM) and no scales: a copy kernel
 * puts x's rows in segment order, then the GEMM runs as its programmatic
 * dependent with the down-projection on its epilogue warps.
 *   x bf16 [M][K]; W bf16 [N][K]; y bf16 [M][N] (out).
 *   pool / seg as for fp8_gemm_lora_epilogue.
 *   ws: lora_workspace_size(LORA_OP_BF16_GEMM, M, K, pool) bytes.
 * Limits: K % 8 == 0, N % 8 == 0, M >= 1. The residency note of
 * fp8_gemm_lora_epilogue applies.
 */
LORA_API int bf16_gemm_lora_epilogue(const void* x, int M, int K, int N, const void* W,
                                     const lora_pool_t* pool, const lora_segments_t* seg, void* y,
                                     void* ws, size_t ws_bytes, lora_stream_t stream);

/*
 * The 8-bit weights with the activations kept in 16 bits (W8A16: the EpiLoRA
 * abstract's 8-bit base, sentence 2, under its 16-bit activation engine,
 * sentence 6) and the fused LoRA term:
 *   y[m][n] = bf16( w_scale[n] * sum_k x[m][k] * E4M3(Wq[n][k])
 *                   + s_a * sum_{j < r_a} v[m][j] * B[0][a][j][n] ),  v = x.A_a.
 * The same weights as fp8_gemm_lora_epilogue (fp8_quantize_rows of W), but x is
 * not quantised: the kernel of bf16_gemm_lora_epilogue, whose weight tiles
 * arrive as E4M3 codes and are turned on chip by eight converter warps into
 * bf16 tiles holding the codes' values times 2^-112 (exact: each pair goes
 * through f16) before the tcgen05 kind::f16 MMAs; the epilogue applies
 * w_scale * 2^112 (in fp32), as the 8-bit path applies w_scale.
 *   x bf16 [M][K]; Wq e4m3 [N][K]; w_scale fp32 [N]; y bf16 [M][N] (out).
 *   pool / seg as for fp8_gemm_lora_epilogue (including its many-adapter path).
 *   ws: lora_workspace_size(LORA_OP_W8A16_GEMM, M, K, pool) bytes.
 * Limits: K % 64 == 0, N % 8 == 0, M >= 1.
 */
LORA_API int w8a16_gemm_lora_epilogue(const void* x, int M, int K, int N, const uint8_t* Wq, const float* w_scale,
                                      const lora_pool_t* pool, const lora_segments_t* seg, void* y, void* ws,
                                      size_t ws_bytes, lora_stream_t stream);

/*
 * OCP MX FP4 quantisation of base weights (the 4-bit base of the EpiLoRA
 * abstract, sentence 2, read as the MX format): each block of 32 consecutive
 * values of a row shares the E8M0 scale X = 2^(floor(log2(amax)) - 2)
 * (exponent clamped to 0..254; 0 for an all-zero block) and each value
 * becomes the E2M1 code nearest to v / X (ties to the even fraction bit,
 * saturating at +-6). Finite weights only.
 *   W bf16 [N][K] (K % 64 == 0);
 *   Wp uint8, ceil(N / 128) * 128 * K / 2 bytes: two codes per byte (element 2i
 *   in the low nibble) in tiles of 128 rows x 64 values, tile (n / 128, k / 64)
 *   at byte ((n / 128) * (K / 64) + k / 64) * 4096, row n % 128 at 32-byte
 *   pitch (one k-block of 128 rows is one contiguous 4 KB copy for the GEMM);
 *   Wsc uint8 [ceil(N / 128)][K / 32][128]: the E8M0 scale of block b of row n
 *   at [n / 128][b][n % 128] (one k-block's scales of 128 rows are contiguous).
 *   The padding rows of the last 128-row group are not written.
 * One kernel launch.
 */
LORA_API int mxfp4_quantize_rows(const void* W, int N, int K, uint8_t* Wp, uint8_t* Wsc, lora_stream_t stream);

/*
 * 4-bit base GEMM with the fused LoRA term: the weights in OCP MX FP4
 * (mxfp4_quantize_rows), the activations in bf16 (the EpiLoRA abstract's
 * 4-bit base, sentence 2, and its 16-bit activation engine, sentence 6):
 *   y[m][n] = bf16( sum_k x[m][k] * E2M1(Wp[n][k]) * 2^(Wsc[n][k / 32] - 127)
 *                   + s_a * sum_{j < r_a} v[m][j] * B[0][a][j][n] ),  v = x.A_a.
 * The kernel of bf16_gemm_lora_epilogue, whose weight tiles arrive as packed
 * codes and scales (half the bytes of an 8-bit weight) and are turned into
 * bf16 on chip by eight converter warps before the tcgen05 kind::f16 MMAs.
 *   x bf16 [M][K]; Wp / Wsc as mxfp4_quantize_rows; y bf16 [M][N] (out).
 *   pool / seg as for fp8_gemm_lora_epilogue (including its many-adapter path).
 *   ws: lora_workspace_size(LORA_OP_MXFP4_GEMM, M, K, pool) bytes.
 * Limits: K % 64 == 0, N % 8 == 0, M >= 1.
 */
LORA_API int mxfp4_gemm_lora_epilogue(const void* x, int M, int K, int N, const uint8_t* Wp, const uint8_t* Wsc,
                                      const lora_pool_t* pool, const lora_segments_t* seg, void* y, void* ws,
                                      size_t ws_bytes, lora_stream_t stream);

/*
 * Gradients of the LoRA layer for training the adapters on a frozen 8-bit
 * base (EpiLoRA abstract, sentence 6: a trainer that keeps the base weights
 * in FP8; the chain rule of y = x.W^T + s_a (x.A_a).B_a of the Punica
 * README's "How?"). For the upstream gradient dY, per token m with adapter a:
 *   dX[m][k]   = bf16( sd[m] swT[k] sum_n dYq[m][n] WqT[k][n]
 *                      + s_a sum_j u[m][j] A_a[k][j] ),  u = dY.B_a^T (fp32)
 *   dA_a[k][j] = s_a sum_{m with adapter a} x[m][k] u[m][j]    (fp32)
 *   dB_a[j][n] = s_a sum_{m with adapter a} v[m][j] dY[m][n],  v = x.A_a (fp32)
 * The base term is the backward's 8-bit GEMM: dY quantised per token as
 * fp8_quantize_rows does (sd, dYq), and W^T quantised per input channel once
 * by the caller (WqT = E4M3 [K][N], swT [K], e.g. fp8_quantize_rows of W^T).
 * Launches: two memsets (dA, dB: adapters without tokens get zero), a
 * transpose of the active adapters' A and B into the workspace, the fused
 * GEMM of fp8_gemm_lora_epilogue on (dY, W^T, the transposed pool) for dX,
 * two shrinks (u, v), and one segmented outer-product kernel each for dA, dB.
 *   x bf16 [M][K]; dY bf16 [M][N]; dX bf16 [M][K] (out);
 *   dA fp32 [n_adapters][K][r_max], dB fp32 [n_adapters][r_max][N] (out; the
 *   padding past each rank is written as zero);
 *   pool: n_slices == 1, h_in == K, h_out == N; seg built for these M tokens;
 *   ws: lora_workspace_size(LORA_OP_FP8_BACKWARD, M, K, pool) bytes.
 * Limits: K % 8 == 0, N % 16 == 0. The residency note of
 * fp8_gemm_lora_epilogue applies to its GEMM.
 */
LORA_API int fp8_lora_backward(const void* x, const void* dY, int M, int K, int N, const uint8_t* WqT,
                               const float* swT, const lora_pool_t* pool, const lora_segments_t* seg,
                               void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                               lora_stream_t stream);

/*
 * Token-wise merge of router-selected adapters into the backbone (LoRA-Switch
 * abstract, shd-paper.top page: for each token a router switches the LoRA
 * adapters and their weights and merges them into the backbone, all selected
 * adapters in one fused kernel):
 *   W_out[n][k] = bf16( W[n][k] + sum_e gates[e] * s_a
 *                                * sum_{j < r_a} A[0][a][k][j] * B[0][a][j][n] ),
 *   a = sel[e]; entries with a outside [0, n_adapters) (-1: none) add nothing.
 * The gate and scale multiply the fp32 product, so the merged weight is
 * rounded once, to bf16. The token is then decoded with the merged weight
 * (e.g. bf16_gemm_lora_epilogue with pool = NULL); W itself stays unchanged
 * unless W_out == W.
 *   W bf16 [N][K] (y = x.W^T); W_out bf16 [N][K], W itself or a disjoint buffer.
 *   pool: n_slices == 1, h_in == K, h_out == N.
 *   sel int32 [n_sel], gates fp32 [n_sel]: DEVICE arrays (the router's output;
 *   the kernel waits for the previous kernel in the stream before reading them).
 * One kernel launch. Limits: N % 8 == 0, K % 8 == 0,
 * n_sel <= LORA_SWITCH_MAX_SELECTED and n_sel * round_up(r_max, 16) <=
 * LORA_SWITCH_MAX_RANK_SUM (else LORA_ERR_UNSUPPORTED).
 */
LORA_API int lora_switch_merge(const void* W, int N, int K, const lora_pool_t* pool, const int32_t* sel,
                               const float* gates, int n_sel, void* W_out, lora_stream_t stream);

/*
 * fp8_gemm_lora_epilogue for callers that cannot allocate device memory
 * (the pages have no counterpart of this call): for example a plugin inside
 * a serving engine that plans all device memory itself and only hands over
 * inputs and outputs, or a hot path that must not call cudaMalloc, which can
 * synchronise the device. Same arguments, checks and results as
 * fp8_gemm_lora_epilogue, minus the workspace: the scratch space lives in a
 * fixed array of lora_noalloc_scratch_bytes() (8 MiB) inside the library's
 * own device memory, held by every GPU that loads the library until the
 * process exits. Calls whose workspace would exceed it return
 * LORA_ERR_WORKSPACE (after the other argument checks). The call allocates
 * nothing (no cudaMalloc or cudaFree).
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * Every call shares the one array: calls that may overlap on the GPU (other
 * streams, other threads) race on it and must be ordered by the caller.
 * The array's status word is zero when the library loads and only
 * lora_noalloc_status clears it: a bounded-wait timeout of any call since the
 * last query stays visible until it is read.
 */
LORA_API int fp8_gemm_lora_epilogue_noalloc(const void* x, int M, int K, int N, const uint8_t* Wq,
                                            const float* w_scale, const lora_pool_t* pool,
                                            const lora_segments_t* seg, void* y, lora_stream_t stream);

/*
 * Read and clear the status word of the built-in scratch array on the current
 * device (fp8_gemm_lora_epilogue_noalloc's counterpart of
 * lora_workspace_status): synchronises `stream`; LORA_OK, or LORA_ERR_TIMEOUT
 * if a call since the last query gave up on a bounded wait (its output is
 * then undefined). *detail (host, may be NULL) receives the raw word.
 */
LORA_API int lora_noalloc_status(lora_stream_t stream, uint32_t* detail);

/* Bytes of the built-in scratch array used by fp8_gemm_lora_epilogue_noalloc. */
LORA_API size_t lora_noalloc_scratch_bytes(void);

/*
 * Test hook for the failure path (not for production use): limit_ns sets the
 * limit of every bounded device-side wait of later launches (1 us .. 2 s;
 * 0 restores the default of 2 s); inject_stall = 1 makes one CTA of each
 * later SGMV (non-decode tiles) and FP8 GEMM launch first wait on a barrier
 * that nothing completes, so that wait runs out, the kernel takes its abort
 * path, returns, and the status calls report LORA_ERR_TIMEOUT. Process-wide;
 * LORA_ERR_INVALID_ARG for values outside those ranges.
 */
LORA_API int lora_debug_set_wait_limit(uint64_t limit_ns, int inject_stall);

/* Static string for a status code. */
LORA_API const char* lora_status_string(int status);

/* Library version, and the largest tile size (LORA_TILE_TOKENS). */
LORA_API int lora_version(void);
LORA_API int lora_tile_tokens(void);

/* Tokens per row of lora_segments_t.tiles for a batch of T tokens over
 * n_adapters: LORA_DECODE_TILE_TOKENS when the batch is decode-like
 * (T <= LORA_DECODE_MAX_TOKENS and T <= 2 * n_adapters, so most adapters hold
 * one or two tokens; the SGMV kernels then run a variant built for tiles that
 * small), else LORA_TILE_TOKENS. -1 for invalid arguments (T < 0,
 * n_adapters < 1). */
LORA_API int lora_tile_tokens_for(int T, int n_adapters);

/* Rows of lora_segments_t.tiles for a batch of T tokens over n_adapters:
 * floor((T + (t - 1) * min(n_adapters, T)) / t) with
 * t = lora_tile_tokens_for(T, n_adapters) (an adapter with c tokens takes
 * ceil(c / t) <= (c + t - 1) / t rows); -1 for invalid arguments. */
LORA_API int lora_max_tiles(int T, int n_adapters);

#ifdef __cplusplus
}
#endif

#endif /* LORA_H_ */
