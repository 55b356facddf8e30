// sgmv_common.cuh -- pieces of the cluster SGMV kernel (sgmv.cu: one tile per
// thread-block cluster with the split-K exchange of v in distributed shared
// memory): launch constants, the pools' tensor maps, the shared-memory tile
// layouts and the bounded waits.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "internal.h"
#include "ptx.cuh"

namespace lora {
namespace {

constexpr int kComputeWarps = 8;
constexpr int kCompute = kComputeWarps * 32;
constexpr int kThreads = kCompute + 32;  // + one producer warp
constexpr int kStages = 3;
constexpr int kTT = LORA_TILE_TOKENS;    // 64
constexpr int kSmallTile = 4;            // tiles of <= 4 tokens use CUDA-core FMAs
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // drains after an abort

// Tensor maps of the pools. a[i]: A viewed as {r_max, h_in, n_slices *
// n_adapters}, box {8 << i, 64, 1} (swizzle = the box row width);
// b[i]: B viewed as {h_out, r_max, n_slices * n_adapters}, box
// {64, min(16 (i + 1), r_max), 1}, 128-byte swizzle.
// bs[i]: B as b[i], box {128, min(16 (i + 1), r_max), 1}, not swizzled (small tiles:
// 256 contiguous bytes of each rank row per request).
// x: {h_in, T, slices of x}, y: {h_out, T, n_slices}, box {64, 16, 1}, 128-byte swizzle.
constexpr int kSmallBoxCols = 128;
struct AMaps {
    CUtensorMap m[4];
    CUtensorMap b[4];
    CUtensorMap bs[4];
    CUtensorMap x, y;
};

__device__ __forceinline__ int round_up(int a, int b) { return (a + b - 1) / b * b; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Byte offset of 16-byte chunk c of A row k in a stage: rows are `pitch` bytes;
// a swizzled tensor-map box XORs the chunk index with bits 7.. of the row's
// offset (mask `swz`: 7, 3, 1 for 128-, 64-, 32-byte rows; 0 unswizzled).
__device__ __forceinline__ uint32_t a_chunk(int k, int c, int pitch, int swz)
{
    const uint32_t off = (uint32_t)(k * pitch);
    return off + (uint32_t)((c ^ (int)((off >> 7) & (uint32_t)swz)) << 4);
}

// Byte offset of 16-byte chunk c (8 columns) of row `row` in a block-swizzled
// tile: blocks of 64 columns, each `rows` rows of 128 bytes, 128-byte swizzle.
__device__ __forceinline__ uint32_t blk_chunk(int row, int c, int rows)
{
    return (uint32_t)((c >> 3) * rows * 128 + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Gather `nt` rows of `cpr` 16-byte chunks with cp.async from all 32 lanes:
// row i of the tile is global row tok[i] (src + tok[i] * row_elems), written
// block-swizzled at dst.
__device__ __forceinline__ void gather_rows(uint32_t dst, const uint16_t* src, size_t row_elems,
                                            const int* tok, int nt, int cpr, int rows, int lane)
{
    if (cpr <= 32 && (cpr & (cpr - 1)) == 0) {  // whole blocks: no division
        const int lg = __ffs(cpr) - 1, c = lane & (cpr - 1);
        for (int row = lane >> lg; row < nt; row += 32 >> lg)
            ptx::cp_async16(dst + blk_chunk(row, c, rows), src + (size_t)tok[row] * row_elems + c * 8, 16);
    } else {
        for (int i = lane; i < nt * cpr; i += 32) {
            const int row = i / cpr, c = i - row * cpr;
            ptx::cp_async16(dst + blk_chunk(row, c, rows), src + (size_t)tok[row] * row_elems + c * 8, 16);
        }
    }
}

// Bounded wait by ONE thread; on expiry raises the CTA abort flag and the
// status word. The clock and the abort flag are read every 256 probes only.
// kHonorAbort = false: the wait does not end early when another role of the
// CTA aborted (used for the v exchange: the peers always send their bytes, and
// a CTA may not leave while their stores into its shared memory are in flight).
template <bool kClusterScope, bool kHonorAbort = true>
__device__ bool wait_one(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                         int code, unsigned long long limit)
{
    auto probe = [&]() {
        return kClusterScope ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
    };
    if (probe()) return true;
    const unsigned long long t0 = ptx::globaltimer();
    for (unsigned n = 1;; ++n) {
        if (probe()) return true;
        if ((n & 255) == 0) {
            if (kHonorAbort && *abort_flag) return false;
            if (ptx::globaltimer() - t0 > limit) {
                *abort_flag = 1;
                atomicOr(status, code);
                return false;
            }
        }
    }
}

// Bounded wait by a WHOLE warp (all 32 lanes must call it): lane 0 polls,
// the others then observe the completed phase themselves (acquire).
template <bool kClusterScope, bool kHonorAbort = true>
__device__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                         int code, unsigned long long limit)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0)
        ok = wait_one<kClusterScope, kHonorAbort>(bar, parity, abort_flag, status, code, limit);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && (threadIdx.x & 31) != 0)
        kClusterScope ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
    return ok;
}

// Tensor maps of the pools (see AMaps) for the shrink (A) and / or the expand (B).
inline bool build_pool_maps(AMaps& am, const lora_pool_t& pool, bool shrink, bool expand)
{
    memset(&am, 0, sizeof(am));
    if (shrink) {
        const uint64_t dims[3] = {(uint64_t)pool.r_max, (uint64_t)pool.h_in,
                                  (uint64_t)pool.n_slices * (uint64_t)pool.n_adapters};
        const uint64_t strides[2] = {(uint64_t)pool.r_max * 2, (uint64_t)pool.h_in * pool.r_max * 2};
        for (int i = 0; i < 4; ++i) {
            const int r8 = 8 << i;
            if (r8 > pool.r_max) break;
            const uint32_t box[3] = {(uint32_t)r8, 64, 1};
            const CUtensorMapSwizzle swz = r8 == 8 ? CU_TENSOR_MAP_SWIZZLE_NONE
                                         : r8 == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                         : r8 == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_128B;
            if (!encode_tmap_3d(&am.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pool.A, dims, strides, box, swz))
                return false;
        }
    }
    if (expand) {
        const uint64_t dims[3] = {(uint64_t)pool.h_out, (uint64_t)pool.r_max,
                                  (uint64_t)pool.n_slices * (uint64_t)pool.n_adapters};
        const uint64_t strides[2] = {(uint64_t)pool.h_out * 2, (uint64_t)pool.r_max * pool.h_out * 2};
        for (int i = 0; i < 4; ++i) {
            if (16 * i >= pool.r_max) break;
            const int rows = 16 * (i + 1) < pool.r_max ? 16 * (i + 1) : pool.r_max;
            const uint32_t box[3] = {64, (uint32_t)rows, 1};
            if (!encode_tmap_3d(&am.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pool.B, dims, strides, box,
                                CU_TENSOR_MAP_SWIZZLE_128B))
                return false;
            const uint32_t box_s[3] = {(uint32_t)kSmallBoxCols, (uint32_t)rows, 1};
            if (!encode_tmap_3d(&am.bs[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, pool.B, dims, strides, box_s,
                                CU_TENSOR_MAP_SWIZZLE_NONE))
                return false;
        }
    }
    return true;
}

// x and y as {columns, T, slices}, box {64, 16, 1}: for tiles of consecutive tokens.
// False (no maps) when the sizes do not allow them.
inline bool build_xy_maps(AMaps& am, const lora_pool_t& pool, int T, const void* x, int64_t x_slice_stride,
                          const void* y, bool shrink, bool expand)
{
    if (pool.h_in < 64 || pool.h_out < 64 || T < 16) return false;
    bool ok = true;
    const uint32_t box[3] = {64, 16, 1};
    if (shrink) {
        const uint64_t xs = x_slice_stride ? (uint64_t)x_slice_stride * 2 : (uint64_t)T * pool.h_in * 2;
        const uint64_t dims[3] = {(uint64_t)pool.h_in, (uint64_t)T, x_slice_stride ? (uint64_t)pool.n_slices : 1u};
        const uint64_t strides[2] = {(uint64_t)pool.h_in * 2, xs};
        ok = ok && encode_tmap_3d(&am.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, x, dims, strides, box,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (expand) {
        const uint64_t dims[3] = {(uint64_t)pool.h_out, (uint64_t)T, (uint64_t)pool.n_slices};
        const uint64_t strides[2] = {(uint64_t)pool.h_out * 2, (uint64_t)T * pool.h_out * 2};
        ok = ok && encode_tmap_3d(&am.y, CU_TENSOR_MAP_DATA_TYPE_UINT16, y, dims, strides, box,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    }
    return ok;
}

// Dynamic shared memory one CTA may take so that two fit on an SM, given the
// kernel's static shared memory (per device).
inline size_t smem_two_per_sm(size_t static_bytes)
{
    int dev = 0;
    cudaGetDevice(&dev);
    int per_sm = 0, reserved = 0;
    cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (per_sm <= 0) per_sm = 233472;
    return (size_t)per_sm / 2 - (size_t)reserved - static_bytes;
}

}  // namespace
}  // namespace lora
