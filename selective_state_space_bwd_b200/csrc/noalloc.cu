// ssm_scan_fwd_noalloc: the forward scan for callers that cannot allocate device memory.
//
// Some callers cannot hand this library a workspace: code that runs where device allocation is
// not allowed or not owned by the caller (a plugin inside a framework whose allocator owns every
// byte of device memory, a latency-critical loop that must never call cudaMalloc, embedded
// runtimes with a fixed memory plan).  For them the forward's scratch lives in a file-scope
// device array of fixed size that the library itself carries; the caller still passes every
// input and output buffer.
#include "../../include/ssm_scan.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

// Scratch of the forward scan: the status word plus, for problems split into time segments,
// the per-segment summaries and entering states.  Every GPU that loads the library holds this
// array until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
// Device address of g_fwd_scratch per device; null until set up.  Kept for the life of the
// process (a cudaDeviceReset would reload the module and may move the array: the header tells
// callers not to use this entry point on a device after resetting it).
void* g_scratch_addr[kMaxDevices];

// In host code `g_fwd_scratch` names a host-side stand-in, not device memory, so the kernels get
// the address the runtime reports for the current device (looked up once per device).
int scratch_of_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return SSM_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SSM_OK;
}

}  // namespace

extern "C" int ssm_scan_fwd_noalloc(const ssm_shape* shape, const void* x, const void* delta_raw,
                                    const float* A_log, const void* Bm, const void* Cm,
                                    const float* Dskip, void* y, float* ckpt,
                                    ssm_stream_t stream) {
    const size_t need = ssm_scan_workspace_bytes(shape, 0);
    if (need == 0)  // invalid shape: let the regular entry point report which check failed
        return ssm_scan_fwd(shape, x, delta_raw, A_log, Bm, Cm, Dskip, y, ckpt, nullptr, 0, stream);
    if (need > kNoAllocScratchBytes) return SSM_ERR_WORKSPACE_TOO_SMALL;
    void* ws = nullptr;
    const int st = scratch_of_current_device(&ws);
    if (st != SSM_OK) return st;
    // The regular forward clears the status word at its start and uses the rest as scratch.
    return ssm_scan_fwd(shape, x, delta_raw, A_log, Bm, Cm, Dskip, y, ckpt, ws,
                        kNoAllocScratchBytes, stream);
}
