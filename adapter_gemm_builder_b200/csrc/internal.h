// internal.h -- launchers shared between the C-ABI layer (api.cu) and the
// kernel files. Every launcher enqueues on `stream` and returns the CUDA
// error of the launch (cudaSuccess when nothing was launched).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora.h"

namespace lora {

// Kernel files expose these; arguments are validated by api.cu.
cudaError_t launch_build_segments(const int32_t* ids, int T, int n_adapters,
                                  const lora_segments_t& seg, cudaStream_t stream);

enum SgmvMode { SGMV_SHRINK = 0, SGMV_EXPAND = 1, SGMV_APPLY = 2 };

// x, v, y may be NULL where the mode does not use them. order: NULL, or
// sgmv_order_bytes(T, n_adapters) bytes of device memory (16-byte aligned) into which
// a small kernel first writes the tile rows in descending cost, which the SGMV
// kernel then walks (long rows first, no tail of a few long CTAs).
cudaError_t launch_sgmv(int mode, const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                        const lora_segments_t& seg, float* v, void* y, cudaStream_t stream,
                        bool pdl_trigger, void* order = nullptr);
size_t sgmv_order_bytes(int T, int n_adapters);
// The expand on the tcgen05 tensor cores (sgmv_tc.cu) for batches of long segments:
// whether a batch qualifies, and the launch (v fp32 [n_slices][T][r_max], y in place).
// v may come as v_parts planes of [n_slices][T][r_max] (the shrink below) that the
// expand sums in plane order.
bool sgmv_expand_tc_eligible(int T, const lora_pool_t& pool);
cudaError_t launch_sgmv_expand_tc(const float* v, int v_parts, const lora_pool_t& pool, const lora_segments_t& seg,
                                  void* y, cudaStream_t stream);
// The shrink on the tensor cores for the same batches, into `parts` planes of v (at most
// sgmv_shrink_tc_parts(pool)); cudaErrorInvalidValue if the pool's tensor map is refused.
int sgmv_shrink_tc_parts(const lora_pool_t& pool);
cudaError_t launch_sgmv_shrink_tc(const void* x, int64_t x_slice_stride, const lora_pool_t& pool,
                                  const lora_segments_t& seg, float* v, int parts, cudaStream_t stream);

// Token-wise merge of the selected adapters into the backbone (merge.cu).
cudaError_t launch_lora_switch_merge(const void* W, int N, int K, const lora_pool_t& pool, const int32_t* sel,
                                     const float* gates, int n_sel, void* W_out, cudaStream_t stream);

// Adapter gradients (grad.cu): the transposed pool (A'_a = B_a^T [N][r_max],
// B'_a = A_a^T [r_max][K]) of the active adapters, and the segmented outer
// products dA_a = s_a x_a^T u_a ([K][r_max], row_major_long) or
// dB_a = s_a v_a^T dY_a ([r_max][N]) of the active adapters.
cudaError_t launch_transpose_pool(const lora_pool_t& pool, const lora_segments_t& seg, void* At, void* Bt,
                                  cudaStream_t stream);
// u[perm[pos]][j] = sum over the v_rep copies of vg[c][pos][j] (the fused GEMM's
// down-projection, segment order) for every position with an adapter (grad.cu).
cudaError_t launch_gather_u(const float* vg, int v_rep, const lora_segments_t& seg, int M, int r_max, float* u,
                            cudaStream_t stream);
cudaError_t launch_grad_outer(bool row_major_long, const void* lng, const float* shrt, int L,
                              const lora_pool_t& pool, const lora_segments_t& seg, float* out, cudaStream_t stream);

// Per-row E4M3 quantisation; row p of the output is row perm[p] of x
// (perm == NULL: identity). The kernel also zeroes zero_words 32-bit words at
// `zero` (may be NULL) and lets a programmatic dependent launch start early.
// copy_bf16: the rows are copied as bf16 instead (xq holds M * K bf16) and sx = 1.
cudaError_t launch_quantize_rows(const void* x, const int32_t* perm, int M, int K, uint8_t* xq,
                                 float* sx, void* zero, size_t zero_words, cudaStream_t stream,
                                 bool copy_bf16 = false);

// OCP MX FP4 quantisation of W bf16 [N][K] (K % 64 == 0): Wp [N][K / 2] packed
// E2M1 codes (element 2i in the low nibble), Wsc E8M0 [ceil(N / 128)][K / 32][128].
cudaError_t launch_mxfp4_quantize(const void* W, int N, int K, uint8_t* Wp, uint8_t* Wsc, cudaStream_t stream);

struct Fp8GemmArgs {
    int M, N, K;
    int esz;             // operand element bytes: 1 = E4M3 (kind::f8f6f4), 2 = bf16 (kind::f16)
    const uint8_t* xq;   // e4m3 (or bf16) [M][K], rows in perm order
    const float* sx;     // [M], perm order (1 for bf16 operands)
    const uint8_t* Wq;   // e4m3 (or bf16) [N][K]
    const float* sw;     // [N]; NULL = 1 (bf16 weights carry no scale)
    const uint8_t* wsc;  // MX FP4 weights (esz 2): Wq holds the packed E2M1 codes
                         // [N][K / 2] and wsc the E8M0 scales [ceil(N / 128)][K / 32][128]
    bool w_e4m3;         // esz 2 with E4M3 weight codes (W8A16): converted to bf16 on chip
    uint16_t* y;         // bf16 [M][N]
    uint32_t* status;    // device status word
    float* partials;     // fp32 [SMs][128][fp8_gemm_tile_n(M)] stream-K partials
    int* flags;          // [SMs], zero on entry
    int* v_done;         // zero on entry
    // LoRA epilogue (lora == false: base only)
    bool lora;
    const uint16_t* x;          // bf16 [M][K], by token index (the down-projection's input)
    const uint16_t* A;          // bf16 [n_adapters][K][r_max]
    const int32_t* perm;        // [M]
    const int32_t* tok_adapter; // [M]
    const int32_t* indptr;      // [n_adapters+1]
    const int32_t* active;      // [n_adapters]
    const int32_t* counts;      // [4]
    float* v;                   // fp32 [M][r_max], segment order, zero on entry
    const uint16_t* B;          // bf16 [n_adapters][r_max][N]
    const int32_t* ranks;
    const float* scales;
    int n_adapters, r_max;
};
// Launched as a programmatic dependent of the previous kernel (the quantiser).
cudaError_t launch_fp8_gemm(const Fp8GemmArgs& a, cudaStream_t stream);
// Token columns of a GEMM tile for M tokens, and the bytes of partial sums.
int fp8_gemm_tile_n(int M);
size_t fp8_gemm_partial_bytes(int M);
// copies of the down-projection v the fused GEMM spreads its atomics over (a power of two)
int fp8_gemm_v_copies(int M);

int device_sm_count();

// Limit of the kernels' bounded waits (2 s unless a test lowered it with
// lora_debug_set_wait_limit) and the test hook that makes one CTA wait on a
// barrier that nothing completes.
unsigned long long debug_wait_limit_ns();
int debug_inject_stall();

// Rows of lora_segments_t.tiles for T tokens over n_adapters.
int max_tiles_for(int T, int n_adapters);
// tokens per tile for a batch (LORA_DECODE_TILE_TOKENS for decode-like batches)
int tile_tokens_for(int T, int n_adapters);

// 2-D tiled tensor map (inner dimension contiguous); false on failure.
bool encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_outer, CUtensorMapSwizzle swz);

// 3-D tiled tensor map: dims innermost first, strides (bytes) of dims 1 and 2;
// out-of-range box elements are filled with zeros. false on failure.
bool encode_tmap_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, const uint64_t dims[3],
                    const uint64_t strides_bytes[2], const uint32_t box[3], CUtensorMapSwizzle swz);

// fp8_gemm_lora_epilogue's argument checks, workspace aside (a lora_status_t).
int fp8_gemm_check_args(const void* x, int M, int K, int N, const uint8_t* Wq, const float* w_scale,
                        const lora_pool_t* pool, const lora_segments_t* seg, const void* y);

// Slot of the device status word in lora_segments_t.counts.
constexpr int kSegStatusSlot = 4;
// status bit: a tile held more tokens than the segments' tile size allows
constexpr int kSegTooLarge = 0x1000;

}  // namespace lora
