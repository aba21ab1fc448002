// hq_noalloc.cu -- hq_encode_noalloc: the weight encoder for callers that cannot allocate GPU
// memory (see include/hq.h).  The encoder's scratch -- the status word, the work counter and one
// look-back slot per block of tiles -- lives in a fixed array in this library's device image
// instead of a caller-provided workspace.
#include <cuda.h>
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
struct Resolved {
    unsigned long long ctx_id;  // the context the address belongs to (unique within the process)
    void* addr;
};
Resolved g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// driver functions, found once (the library links the CUDA runtime statically)
void* driver_fn(const char* name)
{
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return p;
}

// Device address of the scratch array on `dev` (the current device).  It is looked up with
// cudaGetSymbolAddress the first time a device is used, and again whenever that device's primary
// context has changed since (a cudaDeviceReset destroys the context and the array with it).  In
// host code the array's name is only a stand-in for the device symbol, so it is never passed to a
// kernel directly.
void* scratch_address(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    if (cudaSetDevice(dev) != cudaSuccess) return nullptr;  // binds the device's primary context to this thread
    static const CtxGetCurrentFn get_current = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
    static const CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    Resolved& r = g_scratch[dev];
    if (!r.addr || r.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        r.addr = p;
        r.ctx_id = id;
    }
    return r.addr;
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
    // make the device that holds x current (device or managed memory, as for hq_encode), then find
    // the scratch on that device
    if (!hq::device_of(x)) return HQ_ERR_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
    void* ws = scratch_address(dev);
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
