// no_alloc.cu -- ssd_fwd for callers that cannot allocate device memory.
//
// Some callers only ever hold the input and output buffers their host
// application hands them: plugins and runtime extensions that have no access
// to an allocator, or latency-critical code that must not pay the device-wide
// synchronisation a cudaMalloc can cause.  ssd_fwd needs scratch (the
// per-chunk decays and states), which it normally takes from the caller; this
// variant takes it from a fixed buffer compiled into the library instead.
//
// The buffer is a file-scope __device__ array of SSD_NO_ALLOC_SCRATCH_BYTES.
// It is reserved on a device when the library's device code is loaded there:
// under CUDA's lazy module loading (the default since 12.2) that is the first
// call on the device, not library load, and it can fail for lack of memory.
// Host code cannot use the array's name as a device address, so the first
// call on each device looks up the address with cudaGetSymbolAddress (that
// device current) and caches it.  The status word of the kernels that ran on
// the buffer is its first 4 bytes, read by ssd_fwd_no_alloc_check_status.
#include <mutex>

#include "internal.cuh"

namespace {

constexpr size_t kScratchBytes = SSD_NO_ALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// The scratch's device address on the current device (looked up once per
// device); nullptr on failure.
void* scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_addr[dev] = p;
    }
    return g_addr[dev];
}

}  // namespace

extern "C" ssd_status ssd_fwd_no_alloc(const ssd_fwd_args* args, void* stream) {
    if (!args) return SSD_ERR_INVALID_ARG;
    const size_t need = ssd_fwd_workspace_size(args);
    if (need == 0) return ssd_fwd(args, stream);  // invalid sizes: ssd_fwd reports why
    if (need > kScratchBytes) return SSD_ERR_UNSUPPORTED;
    void* scratch = scratch_address();
    if (!scratch) return SSD_ERR_CUDA;
    ssd_fwd_args a = *args;
    a.workspace = scratch;
    a.workspace_bytes = kScratchBytes;
    return ssd_fwd(&a, stream);
}

extern "C" size_t ssd_fwd_no_alloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" ssd_status ssd_fwd_no_alloc_check_status(const ssd_fwd_args* args, void* stream) {
    if (!args) return SSD_ERR_INVALID_ARG;
    const size_t need = ssd_fwd_workspace_size(args);
    if (need == 0) return SSD_ERR_INVALID_ARG;
    if (need > kScratchBytes) return SSD_ERR_UNSUPPORTED;
    void* scratch = scratch_address();
    if (!scratch) return SSD_ERR_CUDA;
    ssd_fwd_args a = *args;
    a.workspace = scratch;
    a.workspace_bytes = kScratchBytes;
    return ssd_fwd_check_status(&a, stream);
}
