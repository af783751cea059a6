// lb_linear_forward_noalloc: the layer forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside another
// framework's allocator (which owns every device allocation and forbids
// outside ones), plugins loaded into a process that already holds the whole
// device pool, and real-time paths where an allocation could block or fail.
// This entry point serves them: the caller still passes x, y and the weights,
// but the scratch that lb_linear_forward takes as a `workspace` argument lives
// in a fixed array in this library's own device memory instead.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes.  Every
// GPU that loads the library holds it until the process exits.  In host code
// its name is only a host-side stand-in, so the first call on each device looks
// up its device address with cudaGetSymbolAddress (with that device current)
// and keeps it; that first call should therefore come before any stream
// capture.  All calls share the one array and it keeps the last call's
// contents: every call clears the part that must start at zero, and calls
// whose kernels overlap on the GPU (different streams without ordering) race
// on it.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "lb_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 256 * 1024;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::once_flag g_scratch_once[kMaxDevices];
void* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

void lookup_scratch(int dev) {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_scratch_ptr[dev] = (g_scratch_err[dev] == cudaSuccess) ? p : nullptr;
}

}  // namespace

extern "C" size_t lb_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" lb_status lb_linear_forward_noalloc(const void* x, lb_dtype x_dtype, int64_t M,
                                               int64_t in, int64_t out, int64_t r,
                                               const lb_branch* br, int n_branches, float* y,
                                               void* stream) {
    if (M <= 0 || r <= 0 || n_branches < 1 || n_branches > 2) return LB_ERR_INVALID_ARG;
    const size_t need = lb_linear_workspace_size(M, in, out, r, n_branches);
    if (need == 0) return LB_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return LB_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LB_ERR_CUDA;
    std::call_once(g_scratch_once[dev], lookup_scratch, dev);
    if (g_scratch_err[dev] != cudaSuccess || g_scratch_ptr[dev] == nullptr) return LB_ERR_CUDA;
    // lb_linear_forward clears the header and the accumulators it needs zeroed.
    return lb_linear_forward(x, x_dtype, M, in, out, r, br, n_branches, y, g_scratch_ptr[dev],
                             kNoAllocScratchBytes, stream);
}
