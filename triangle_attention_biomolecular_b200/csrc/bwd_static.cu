// Backward pass on a fixed scratch area held in the library's own static
// device memory, for callers that must not allocate device memory.
//
// tri_attn_bwd takes a caller-supplied workspace: per-row softmax vectors
// (D, log-sum-exp, mask in base-2 units, tile flags), dQ staging slots and,
// for small batches, dBias partial sums.  Some callers cannot provide one on
// the path where the backward runs: an application whose own allocator owns
// all device memory and forbids stray cudaMalloc, or a latency-critical loop
// in which cudaMalloc / cudaFree (which may synchronise the device) are not
// allowed.  tri_attn_bwd_static_scratch serves them: it runs exactly the
// kernels of tri_attn_bwd, with the workspace placed in the file-scope array
// below instead of in caller memory.  Nothing here allocates; the array is
// reserved by the CUDA runtime when this module is loaded onto a device.
//
// The array sits in its own translation unit (its own module), so a program
// that never calls this entry point does not load the module and does not
// reserve the memory on devices where modules load lazily.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "../../include/tri_attn.h"

// The scratch: TRI_ATTN_STATIC_SCRATCH_BYTES per device, 256-byte aligned as
// the backward's workspace requires.  Nothing in it has to start at zero:
// every word the kernels read is written earlier in the same call.
static __device__ __align__(256) unsigned char g_bwd_static_scratch[TRI_ATTN_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};  // device address of the array, per device ordinal

// Device address of the scratch array on the current device.  The first call
// on a device looks it up (which loads this module there); later calls reuse
// the stored address.
tri_attn_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TRI_ATTN_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return TRI_ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_bwd_static_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return TRI_ATTN_ERR_CUDA;
        }
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return TRI_ATTN_OK;
}

}  // namespace

extern "C" tri_attn_status tri_attn_bwd_static_scratch(const tri_attn_bwd_args* a, tri_attn_stream_t stream) {
    if (!a) return TRI_ATTN_ERR_NULL;
    tri_attn_bwd_args c = *a;
    const size_t need = tri_attn_bwd_workspace_bytes(a->f.B, a->f.N, a->f.H, a->f.d);
    if (need == 0) {
        // invalid sizes: let the regular entry point name the argument error
        c.workspace = nullptr;
        c.workspace_bytes = 0;
        return tri_attn_bwd(&c, stream);
    }
    if (need > static_cast<size_t>(TRI_ATTN_STATIC_SCRATCH_BYTES)) return TRI_ATTN_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    const tri_attn_status st = scratch_on_current_device(&scratch);
    if (st != TRI_ATTN_OK) return st;
    c.workspace = scratch;
    c.workspace_bytes = static_cast<size_t>(TRI_ATTN_STATIC_SCRATCH_BYTES);
    return tri_attn_bwd(&c, stream);
}
