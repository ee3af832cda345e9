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
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "../../include/tri_attn.h"

namespace tri {
// the host-side argument checks of tri_attn_bwd (csrc/api.cu); no CUDA call
tri_attn_status bwd_validate(const tri_attn_bwd_args* a);
}  // namespace tri

// The scratch: TRI_ATTN_STATIC_SCRATCH_BYTES per device, 256-byte aligned as
// the backward's workspace requires.  Nothing in it has to start at zero:
// every word the kernels read is written earlier in the same call.
static __device__ __align__(256) unsigned char g_bwd_static_scratch[TRI_ATTN_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;

// Device address of the array, per device ordinal, with the id of the CUDA
// context it was looked up in.  A device reset destroys that context and
// unloads the module; the next call then sees a new context id and looks the
// address up again instead of using a stale one.
struct ScratchSlot {
    unsigned long long ctx_id;
    void* addr;
};
ScratchSlot g_slot[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// id of the current context (0 if it cannot be told, and then the address is
// looked up again on every call)
unsigned long long current_context_id() {
    static std::once_flag once;
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device.  The first call
// in a device's context looks it up (which loads this module there); later
// calls in the same context reuse it.
tri_attn_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TRI_ATTN_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return TRI_ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    // cudaGetSymbolAddress makes the device's primary context current if needed,
    // so the context id is read after it
    void* ptr = g_slot[dev].addr;
    unsigned long long id = ptr ? current_context_id() : 0;
    if (!ptr || id == 0 || id != g_slot[dev].ctx_id) {
        ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_bwd_static_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            g_slot[dev] = ScratchSlot{0, nullptr};
            return TRI_ATTN_ERR_CUDA;
        }
        g_slot[dev] = ScratchSlot{current_context_id(), ptr};
    }
    *out = ptr;
    return TRI_ATTN_OK;
}

}  // namespace

extern "C" tri_attn_status tri_attn_bwd_static_scratch(const tri_attn_bwd_args* a, tri_attn_stream_t stream) {
    // every argument error is reported first, before any CUDA call
    tri_attn_status st = tri::bwd_validate(a);
    if (st) return st;
    const size_t need = tri_attn_bwd_workspace_bytes(a->f.B, a->f.N, a->f.H, a->f.d);
    if (need == 0) return TRI_ATTN_ERR_SHAPE;  // not reached: the sizes passed the checks above
    if (need > static_cast<size_t>(TRI_ATTN_STATIC_SCRATCH_BYTES)) return TRI_ATTN_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if ((st = scratch_on_current_device(&scratch))) return st;
    tri_attn_bwd_args c = *a;
    c.workspace = scratch;
    c.workspace_bytes = static_cast<size_t>(TRI_ATTN_STATIC_SCRATCH_BYTES);
    return tri_attn_bwd(&c, stream);
}
