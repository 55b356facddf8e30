// noalloc.cu -- fp8_gemm_lora_epilogue for callers that cannot allocate
// device memory.
//
// Some callers own no allocator: a plugin inside a serving engine that
// plans all device memory itself and hands a kernel only its inputs and
// outputs, or a hot path that must never call cudaMalloc (an allocation can
// synchronise the device). They cannot provide the workspace that
// fp8_gemm_lora_epilogue needs. This entry point keeps that scratch space in
// a fixed array in the library's own device memory instead.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library is loaded holds it (kNoAllocScratchBytes) until the process exits.
// Host code cannot use the array's name as a device address, so the address
// is looked up once per device with cudaGetSymbolAddress, while that device
// is current, on the first call made on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "lora.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per GPU
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first
// use); NULL if the look-up fails.
void* scratch_on_current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t lora_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int fp8_gemm_lora_epilogue_noalloc(const void* x, int M, int K, int N, const uint8_t* Wq,
                                   const float* w_scale, const lora_pool_t* pool,
                                   const lora_segments_t* seg, void* y, lora_stream_t stream)
{
    // the same argument checks, and status codes, as the workspace entry point
    const int st = lora::fp8_gemm_check_args(x, M, K, N, Wq, w_scale, pool, seg, y);
    if (st != LORA_OK) return st;
    const size_t need = lora_workspace_size(LORA_OP_FP8_GEMM, M, K, pool);
    if (need == (size_t)-1) return LORA_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return LORA_ERR_WORKSPACE;  // beyond the built-in scratch
    void* ws = scratch_on_current_device();
    if (!ws) return LORA_ERR_CUDA;
    // The status word (the first 256 bytes) starts at zero when the library is loaded
    // and is cleared only by lora_noalloc_status, so a bounded-wait timeout of any call
    // stays visible until it is read. Everything else the kernels read is rewritten by
    // each call before it is read (the quantiser zeroes v and the sync words).
    return fp8_gemm_lora_epilogue(x, M, K, N, Wq, w_scale, pool, seg, y, ws, need, stream);
}

int lora_noalloc_status(lora_stream_t stream, uint32_t* detail)
{
    void* ws = scratch_on_current_device();
    if (!ws) return LORA_ERR_CUDA;
    return lora_workspace_status(ws, 256, stream, detail);
}

}  // extern "C"
