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
// its name is only a host-side stand-in, so a call on a device looks up its
// device address with cudaGetSymbolAddress (with that device current) until a
// lookup succeeds, and keeps the address from then on; the first call on each
// device should therefore come before any stream capture.  All calls share the
// one array and it keeps the last call's contents: every call clears the part
// that must start at zero, and calls whose kernels overlap on the GPU
// (different streams without ordering) race on it.  Nothing here calls
// cudaMalloc, cudaFree or any allocating routine.
//
// Which kernels run: the ones lb_linear_forward would run, as far as their
// scratch fits the array.  The tensor-core path runs without its stage-1
// K split (whose partial sums need tens of MB); when even that does not fit,
// the lookup-table kernels run instead.  Both give the layer's result within
// the same fp32 accuracy.
#include <atomic>
#include <mutex>

#include "lb_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 256 * 1024;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
std::atomic<void*> g_scratch_ptr[kMaxDevices];   // null until a lookup on the device succeeds

// Device address of the array on device `dev` (current), or nullptr if the
// lookup fails; a failed lookup is retried on the next call.
void* scratch_address(int dev) {
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            (void)cudaGetLastError();   // not sticky: clear it for the caller
            return nullptr;
        }
        g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" size_t lb_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" lb_status lb_linear_forward_noalloc(const void* x, lb_dtype x_dtype, int64_t M,
                                               int64_t in, int64_t out, int64_t r,
                                               const lb_branch* br, int n_branches, float* y,
                                               void* stream) {
    if (!br || M <= 0 || in <= 0 || out <= 0 || r <= 0 || n_branches < 1 || n_branches > 2)
        return LB_ERR_INVALID_ARG;
    if (lb_linear_workspace_size(M, in, out, r, n_branches) == 0) return LB_ERR_INVALID_ARG;
    lb::LinearRoute route = lb::default_route(M, in, out, r, br, n_branches);
    if (route == lb::kRoutePrefill) {
        route = lb::prefill_workspace_bytes(M, in, r, false) <= kNoAllocScratchBytes
                    ? lb::kRoutePrefillNoSplit
                    : lb::kRouteDecode;
    }
    if (route == lb::kRouteDecode &&
        lb::decode_workspace_bytes(M, r, n_branches) > kNoAllocScratchBytes)
        return LB_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LB_ERR_CUDA;
    void* scratch = scratch_address(dev);
    if (scratch == nullptr) return LB_ERR_CUDA;
    // the route clears the header and the accumulators it needs zeroed
    return lb::linear_forward_route(x, x_dtype, M, in, out, r, br, n_branches, y, scratch,
                                    kNoAllocScratchBytes, 0, static_cast<cudaStream_t>(stream),
                                    route);
}
