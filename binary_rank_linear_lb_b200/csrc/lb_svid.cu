// Dual-SVID initialisation of a factorised layer on the GPU.
//
// "Samsung LittleBit: A 13B LLM Under 1 GB ...", section "How it works", item
// 3: the layer starts from a truncated SVD of the real weight, whose signs and
// magnitudes are mapped onto the binary factors and the scales; a second,
// residual branch is fitted to what the first one missed.  Per branch, on the
// residual R (W for the first branch):
//   R ~ U S V^T (rank r)                 cuSOLVER's randomized truncated SVD
//   U' = U S^(1/2), V' = V S^(1/2)       the singular values split evenly
//   sign(U'), sign(V')                   packed by this library's packer
//   |U'| ~ h l_u^T, |V'| ~ g l_v^T       rank-1 fits (power iteration)
//   h, g scaled to mean 1, l = l_u l_v, all rounded to fp16
//   R <- R - diag(h) sign(U') diag(l) sign(V')^T diag(g)
// The last step rebuilds the branch from exactly what is stored (fp16 scales,
// packed signs) and subtracts it with one cuBLAS GEMM.
//
// Storage: the weight and the residual are row-major out x in fp32, which is
// in x out in the column-major convention of cuSOLVER and cuBLAS.  U and V
// are kept column-major (out x r, in x r): their transposes are row-major
// r x out and r x in, which the packer reads along axis 0 (each output row
// along r) and axis 1 (each latent row along in).
#include <cublas_v2.h>
#include <cusolverDn.h>

#include <cstdlib>
#include <vector>

#include "lb_internal.cuh"

namespace lb {
namespace {

constexpr int kSvThreads = 256;
constexpr int kRank1Iters = 40;       // power iterations of each magnitude fit
constexpr int64_t kSvdIters = 4;      // power iterations inside the randomized SVD

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.0f;
    for (int w = 0; w < kSvThreads / 32; ++w) s += red[w];
    __syncthreads();
    return s;
}

// dst (n x k, column-major) = |src| * sqrt(S[col]).
__global__ void scaled_abs_kernel(const float* __restrict__ src, const float* __restrict__ S,
                                  int64_t n, int k, float* __restrict__ dst) {
    const int64_t total = n * k;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = fabsf(src[i]) * sqrtf(fmaxf(S[i / n], 0.0f));
}

// out[0] = v . v (one block).
__global__ void __launch_bounds__(kSvThreads) self_dot_kernel(const float* __restrict__ v, int64_t n,
                                                              float* __restrict__ out) {
    __shared__ float red[kSvThreads / 32];
    float s = 0.0f;
    for (int64_t i = threadIdx.x; i < n; i += kSvThreads) s += v[i] * v[i];
    s = block_sum(s, red);
    if (threadIdx.x == 0) out[0] = s;
}

// a[i] = sum_c A[c*n + i] b[c] / bb  (A: n x k column-major).
__global__ void col_matvec_kernel(const float* __restrict__ A, int64_t n, int k,
                                  const float* __restrict__ b, const float* __restrict__ bb,
                                  float* __restrict__ a) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float s = 0.0f;
    for (int c = 0; c < k; ++c) s += A[(int64_t)c * n + i] * b[c];
    const float d = bb[0];
    a[i] = d > 0.0f ? s / d : 0.0f;
}

// b[c] = sum_i A[c*n + i] a[i] / aa  (one block per column c).
__global__ void __launch_bounds__(kSvThreads) row_matvec_kernel(const float* __restrict__ A,
                                                                int64_t n,
                                                                const float* __restrict__ a,
                                                                const float* __restrict__ aa,
                                                                float* __restrict__ b) {
    __shared__ float red[kSvThreads / 32];
    const float* col = A + (int64_t)blockIdx.x * n;
    float s = 0.0f;
    for (int64_t i = threadIdx.x; i < n; i += kSvThreads) s += col[i] * a[i];
    s = block_sum(s, red);
    if (threadIdx.x == 0) {
        const float d = aa[0];
        b[blockIdx.x] = d > 0.0f ? s / d : 0.0f;
    }
}

__global__ void fill_kernel(float* __restrict__ v, int64_t n, float x) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        v[i] = x;
}

// Scale a (length n) to mean 1 and move the factor into b (length k): a /= m,
// b *= m with m = mean(a) (nothing if m = 0); fp16 copies of the results.
// One block.
__global__ void __launch_bounds__(kSvThreads) normalise_kernel(float* __restrict__ a, int64_t n,
                                                               float* __restrict__ b, int k,
                                                               __half* __restrict__ a16) {
    __shared__ float red[kSvThreads / 32];
    float s = 0.0f;
    for (int64_t i = threadIdx.x; i < n; i += kSvThreads) s += a[i];
    const float m = block_sum(s, red) / (float)n;
    if (m > 0.0f) {
        for (int64_t i = threadIdx.x; i < n; i += kSvThreads) a[i] /= m;
        for (int i = threadIdx.x; i < k; i += kSvThreads) b[i] *= m;
    }
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += kSvThreads) a16[i] = __float2half_rn(a[i]);
}

// l = fp16(l_u * l_v).
__global__ void latent_scale_kernel(const float* __restrict__ lu, const float* __restrict__ lv,
                                    int k, __half* __restrict__ l16) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < k) l16[i] = __float2half_rn(lu[i] * lv[i]);
}

// dst (n x k, column-major) = row[i] * s(i, c) * (col ? col[c] : 1) with fp16
// scales and s the signs of a packed matrix in either layout: packed along k
// (n rows of k signs: s(i, c) = bit c of row i), or with `across` packed along
// n (k rows of n signs: s(i, c) = bit i of row c).
__global__ void expand_kernel(const uint32_t* __restrict__ P, int sliced, int across, int64_t n,
                              int k, const __half* __restrict__ row, const __half* __restrict__ col,
                              float* __restrict__ dst) {
    const int64_t total = n * (int64_t)k;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx % n, c = idx / n;
        // (packed row, element within it) and the packed matrix's shape
        const int64_t pr = across ? c : i, pe = across ? i : c;
        const int64_t prows = across ? k : n, nw = ((across ? n : k) + 31) / 32;
        const uint32_t w = sliced ? P[sliced_offset(prows, nw, pr, pe >> 5)] : P[pr * nw + (pe >> 5)];
        float v = __half2float(row[i]);
        if (col != nullptr) v *= __half2float(col[c]);
        dst[idx] = ((w >> (pe & 31)) & 1u) ? -v : v;
    }
}

// dst (cols x rows, column-major) = src (rows x cols, column-major) transposed.
__global__ void transpose_kernel(const float* __restrict__ src, int64_t rows, int64_t cols,
                                 float* __restrict__ dst) {
    __shared__ float tile[32][33];
    const int64_t r0 = (int64_t)blockIdx.x * 32, c0 = (int64_t)blockIdx.y * 32;
    for (int j = threadIdx.y; j < 32; j += blockDim.y) {
        const int64_t r = r0 + threadIdx.x, c = c0 + j;
        if (r < rows && c < cols) tile[j][threadIdx.x] = src[c * rows + r];
    }
    __syncthreads();
    for (int j = threadIdx.y; j < 32; j += blockDim.y) {
        const int64_t c = c0 + threadIdx.x, r = r0 + j;
        if (r < rows && c < cols) dst[r * cols + c] = tile[threadIdx.x][j];
    }
}

unsigned grid_for(int64_t n) {
    const int64_t b = (n + kSvThreads - 1) / kSvThreads;
    return (unsigned)(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

// Power iteration for A (n x k, column-major, >= 0) ~ a b^T.
void rank1_fit(const float* A, int64_t n, int k, float* a, float* b, float* scal,
               cudaStream_t s) {
    fill_kernel<<<grid_for(k), kSvThreads, 0, s>>>(b, k, 1.0f);
    for (int it = 0; it < kRank1Iters; ++it) {
        self_dot_kernel<<<1, kSvThreads, 0, s>>>(b, k, scal);
        col_matvec_kernel<<<(unsigned)((n + kSvThreads - 1) / kSvThreads), kSvThreads, 0, s>>>(
            A, n, k, b, scal, a);
        self_dot_kernel<<<1, kSvThreads, 0, s>>>(a, n, scal + 1);
        row_matvec_kernel<<<(unsigned)k, kSvThreads, 0, s>>>(A, n, a, scal + 1, b);
    }
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

struct SvidLayout {
    size_t R, A, U, V, S, mag, expU, expV, h, g, lu, lv, scal, info, solver, total;
};

SvidLayout svid_layout(int64_t out, int64_t in, int64_t r, size_t solver_bytes) {
    SvidLayout L;
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += up256(bytes); return at; };
    L.R = take(4 * (size_t)out * in);
    L.A = take(4 * (size_t)out * in);
    L.U = take(4 * (size_t)out * r);
    L.V = take(4 * (size_t)in * r);
    L.S = take(4 * (size_t)r);
    L.mag = take(4 * (size_t)std::max(out, in) * r);
    L.expU = take(4 * (size_t)out * r);
    L.expV = take(4 * (size_t)in * r);
    L.h = take(4 * (size_t)out);
    L.g = take(4 * (size_t)in);
    L.lu = take(4 * (size_t)r);
    L.lv = take(4 * (size_t)r);
    L.scal = take(4 * 4);
    L.info = take(4);
    L.solver = take(solver_bytes);
    L.total = o;
    return L;
}

int64_t oversampling(int64_t r, int64_t n_min) { return std::min<int64_t>(std::max<int64_t>(r / 4, 8), n_min - r); }

// cuSOLVER's workspace for the rank-r SVD of an m x n (m >= n) column-major matrix.
bool solver_bytes(cusolverDnHandle_t h, cusolverDnParams_t prm, int64_t m, int64_t n, int64_t r,
                  size_t& dev, size_t& host) {
    return cusolverDnXgesvdr_bufferSize(h, prm, 'S', 'S', m, n, r, oversampling(r, n), kSvdIters,
                                        CUDA_R_32F, nullptr, m, CUDA_R_32F, nullptr, CUDA_R_32F,
                                        nullptr, m, CUDA_R_32F, nullptr, n, CUDA_R_32F, &dev,
                                        &host) == CUSOLVER_STATUS_SUCCESS;
}

struct Handles {
    cusolverDnHandle_t sol = nullptr;
    cusolverDnParams_t prm = nullptr;
    cublasHandle_t blas = nullptr;
    ~Handles() {
        if (prm) cusolverDnDestroyParams(prm);
        if (sol) cusolverDnDestroy(sol);
        if (blas) cublasDestroy(blas);
    }
    bool make(cudaStream_t s) {
        return cusolverDnCreate(&sol) == CUSOLVER_STATUS_SUCCESS &&
               cusolverDnCreateParams(&prm) == CUSOLVER_STATUS_SUCCESS &&
               cusolverDnSetStream(sol, s) == CUSOLVER_STATUS_SUCCESS &&
               cublasCreate(&blas) == CUBLAS_STATUS_SUCCESS &&
               cublasSetStream(blas, s) == CUBLAS_STATUS_SUCCESS &&
               cublasSetMathMode(blas, CUBLAS_PEDANTIC_MATH) == CUBLAS_STATUS_SUCCESS;
    }
};

bool svid_args_ok(int64_t out, int64_t in, int64_t r, int nb) {
    return out > 0 && in > 0 && r > 0 && r <= std::min(out, in) && nb >= 1 && nb <= 2 &&
           out <= (1 << 20) && in <= (1 << 20) && out * in <= ((int64_t)1 << 31);
}

}  // namespace
}  // namespace lb

using namespace lb;

extern "C" size_t lb_dual_svid_workspace_size(int64_t out, int64_t in, int64_t r, int n_branches) {
    if (!svid_args_ok(out, in, r, n_branches)) return 0;
    Handles H;
    if (cusolverDnCreate(&H.sol) != CUSOLVER_STATUS_SUCCESS ||
        cusolverDnCreateParams(&H.prm) != CUSOLVER_STATUS_SUCCESS)
        return 0;
    size_t dev = 0, host = 0;
    if (!solver_bytes(H.sol, H.prm, std::max(out, in), std::min(out, in), r, dev, host)) return 0;
    return svid_layout(out, in, r, dev).total;
}

extern "C" lb_status lb_dual_svid(const float* W, int64_t out, int64_t in, int64_t r,
                                  int n_branches, int layout, uint32_t* const* Vp,
                                  uint32_t* const* Up, uint16_t* const* h, uint16_t* const* g,
                                  uint16_t* const* l, void* workspace, size_t ws_bytes,
                                  void* stream) {
    if (!W || !Vp || !Up || !h || !g || !l || !workspace) return LB_ERR_INVALID_ARG;
    if (!svid_args_ok(out, in, r, n_branches)) return LB_ERR_INVALID_ARG;
    if (layout != LB_LAYOUT_ROWS && layout != LB_LAYOUT_SLICES) return LB_ERR_INVALID_ARG;
    for (int b = 0; b < n_branches; ++b) {
        if (!Vp[b] || !Up[b] || !h[b] || !g[b] || !l[b]) return LB_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(Vp[b]) | reinterpret_cast<uintptr_t>(Up[b])) & 15)
            return LB_ERR_ALIGNMENT;
        if ((reinterpret_cast<uintptr_t>(h[b]) | reinterpret_cast<uintptr_t>(g[b]) |
             reinterpret_cast<uintptr_t>(l[b])) & 1)
            return LB_ERR_ALIGNMENT;
    }
    if ((reinterpret_cast<uintptr_t>(W) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return LB_ERR_ALIGNMENT;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return LB_ERR_CUDA;
    if (major != 10) return LB_ERR_UNSUPPORTED;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Handles H;
    if (!H.make(s)) return LB_ERR_CUDA;
    const bool wide = in >= out;                 // the SVD runs on an m x n matrix with m >= n
    const int64_t m = wide ? in : out, n = wide ? out : in;
    size_t dev_bytes = 0, host_bytes = 0;
    if (!solver_bytes(H.sol, H.prm, m, n, r, dev_bytes, host_bytes)) return LB_ERR_CUDA;
    const SvidLayout L = svid_layout(out, in, r, dev_bytes);
    if (ws_bytes < L.total) return LB_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    float* R = reinterpret_cast<float*>(ws + L.R);
    float* A = reinterpret_cast<float*>(ws + L.A);
    float* U = reinterpret_cast<float*>(ws + L.U);       // out x r, column-major
    float* V = reinterpret_cast<float*>(ws + L.V);       // in x r, column-major
    float* S = reinterpret_cast<float*>(ws + L.S);
    float* mag = reinterpret_cast<float*>(ws + L.mag);
    float* eU = reinterpret_cast<float*>(ws + L.expU);
    float* eV = reinterpret_cast<float*>(ws + L.expV);
    float* hv = reinterpret_cast<float*>(ws + L.h);
    float* gv = reinterpret_cast<float*>(ws + L.g);
    float* lu = reinterpret_cast<float*>(ws + L.lu);
    float* lv = reinterpret_cast<float*>(ws + L.lv);
    float* scal = reinterpret_cast<float*>(ws + L.scal);
    int* info = reinterpret_cast<int*>(ws + L.info);
    std::vector<unsigned char> host_buf(host_bytes > 0 ? host_bytes : 1);

    if (cudaMemcpyAsync(R, W, 4 * (size_t)out * in, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LB_ERR_CUDA;
    const bool sliced = layout == LB_LAYOUT_SLICES;
    for (int b = 0; b < n_branches; ++b) {
        // the SVD of R (R is in x out column-major; cuSOLVER overwrites its input)
        if (wide) {
            if (cudaMemcpyAsync(A, R, 4 * (size_t)out * in, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
                return LB_ERR_CUDA;
        } else {
            transpose_kernel<<<dim3((unsigned)((in + 31) / 32), (unsigned)((out + 31) / 32)),
                               dim3(32, 8), 0, s>>>(R, in, out, A);
        }
        float* Ucm = wide ? V : U;                         // m x r
        float* Vcm = wide ? U : V;                         // n x r
        if (cusolverDnXgesvdr(H.sol, H.prm, 'S', 'S', m, n, r, oversampling(r, n), kSvdIters,
                              CUDA_R_32F, A, m, CUDA_R_32F, S, CUDA_R_32F, Ucm, m, CUDA_R_32F, Vcm,
                              n, CUDA_R_32F, ws + L.solver, dev_bytes, host_buf.data(), host_bytes,
                              info) != CUSOLVER_STATUS_SUCCESS)
            return LB_ERR_CUDA;
        int hinfo = 0;
        if (cudaMemcpyAsync(&hinfo, info, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return LB_ERR_CUDA;
        if (hinfo != 0) return LB_ERR_CUDA;
        // signs: U^T is row-major r x out (axis 0: each output row along r), V^T is
        // row-major r x in (axis 1: each latent row along in); sqrt(S) > 0 keeps them
        if (launch_pack(U, r, out, out, 0, Up[b], (r + 31) / 32, sliced, s) != cudaSuccess ||
            launch_pack(V, r, in, in, 1, Vp[b], (in + 31) / 32, sliced, s) != cudaSuccess)
            return LB_ERR_CUDA;
        // magnitudes: |U'| ~ h l_u^T, |V'| ~ g l_v^T; h, g to mean 1; l = l_u l_v
        __half* h16 = reinterpret_cast<__half*>(h[b]);
        __half* g16 = reinterpret_cast<__half*>(g[b]);
        __half* l16 = reinterpret_cast<__half*>(l[b]);
        scaled_abs_kernel<<<grid_for(out * r), kSvThreads, 0, s>>>(U, S, out, (int)r, mag);
        rank1_fit(mag, out, (int)r, hv, lu, scal, s);
        normalise_kernel<<<1, kSvThreads, 0, s>>>(hv, out, lu, (int)r, h16);
        scaled_abs_kernel<<<grid_for(in * r), kSvThreads, 0, s>>>(V, S, in, (int)r, mag);
        rank1_fit(mag, in, (int)r, gv, lv, scal, s);
        normalise_kernel<<<1, kSvThreads, 0, s>>>(gv, in, lv, (int)r, g16);
        latent_scale_kernel<<<(unsigned)((r + kSvThreads - 1) / kSvThreads), kSvThreads, 0, s>>>(
            lu, lv, (int)r, l16);
        // R <- R - diag(h) S_U diag(l) S_V^T diag(g), from the stored branch:
        // in the column-major view R (in x out) -= E_V (in x r) E_U^T (r x out)
        expand_kernel<<<grid_for(out * r), kSvThreads, 0, s>>>(Up[b], sliced, 0, out, (int)r, h16,
                                                               l16, eU);
        expand_kernel<<<grid_for(in * r), kSvThreads, 0, s>>>(Vp[b], sliced, 1, in, (int)r, g16,
                                                              nullptr, eV);
        const float alpha = -1.0f, beta = 1.0f;
        if (cublasSgemm(H.blas, CUBLAS_OP_N, CUBLAS_OP_T, (int)in, (int)out, (int)r, &alpha, eV,
                        (int)in, eU, (int)out, &beta, R, (int)in) != CUBLAS_STATUS_SUCCESS)
            return LB_ERR_CUDA;
        if (cudaGetLastError() != cudaSuccess) return LB_ERR_CUDA;
    }
    return cudaStreamSynchronize(s) == cudaSuccess ? LB_OK : LB_ERR_CUDA;
}
