// hq_noalloc.cu -- hq_encode_noalloc: the weight encoder for callers that cannot allocate GPU
// memory (see include/hq.h).  The encoder's scratch -- the status word, the work counter and one
// look-back slot per block of tiles -- lives in a fixed array in this library's device image
// instead of a caller-provided workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hq.h"
#include "hq_launch.h"

namespace {

// 128 KiB on every GPU that loads the library, held until the process exits.
constexpr size_t kNoallocScratchBytes = (size_t)HQ_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on `dev` (the current device), looked up once per device.
// In host code the array's name is only a stand-in for the device symbol, so it is never passed
// to a kernel directly.
void* scratch_address(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" hq_status_t hq_encode_noalloc(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols,
                                         const hq_params_t* p, hq_code_t* out, uint32_t* status_out, void* stream)
{
    if (!p || !x) return HQ_ERR_ARG;
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    // the scratch holds a 64-byte header and 8 bytes per block of tiles of this weight encoder
    const size_t need = hq::encode_workspace_bytes(rows, cols, p->tile, dtype == HQ_BF16 ? 0 : 1);
    if (need == 0) return HQ_ERR_ARG;
    if (need > kNoallocScratchBytes) return HQ_ERR_RANGE;
    // make the device that holds x current, then find the scratch on that device
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, x) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return HQ_ERR_ARG;
    }
    if (cudaSetDevice(attr.device) != cudaSuccess) return HQ_ERR_CUDA;
    void* ws = scratch_address(attr.device);
    if (!ws) return HQ_ERR_CUDA;
    // the regular encoder clears the header and look-back slots it uses before its kernel runs
    const hq_status_t st = hq_encode(x, dtype, rows, cols, p, out, ws, kNoallocScratchBytes, stream);
    if (st != HQ_OK) return st;
    if (status_out &&
        cudaMemcpyAsync(status_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)) !=
            cudaSuccess)
        return HQ_ERR_CUDA;
    return HQ_OK;
}
