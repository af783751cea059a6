// Bit-serial variant of the layer: every product a sign times a sign, computed
// as XOR + popcount on 32-bit words.
//
// "Samsung LittleBit: A 13B LLM Under 1 GB ...", section "The XOR claim": when
// both operands are signs, a multiply becomes an XOR plus a popcount.  The
// activations of the layer are not signs, so each vector v (g o x for the first
// contraction, l o t for the second) is first quantised to B-bit fixed point in
// a code whose bit-planes are signs:
//   D = 2^e, the smallest (e >= -100) with max|v| <= (2^B - 1) D;
//   q_j = 2 floor(v_j / 2D) + 1, odd, |D q_j - v_j| <= D;
//   q_j = sum_p 2^p sigma_jp, sigma_jp = 2 bit_p((q_j + 2^B - 1) / 2) - 1.
// A plane is stored like the packed signs (bit 1 <=> -1), so for a packed row
// of signs s over n valid columns
//   sum_j s_j q_j = sum_p 2^p (n - 2 popc(s XOR plane_p))
// exactly, in integers.  The result is the layer applied to the quantised
// vectors: t'_k = l_k * (D1 T_k) in fp32, y_i = sum_b h_bi D2_b Z_bi.
//
// Kernels (one launch each, stream-ordered): quantise x -> planes; first
// contraction (a warp per row of V); quantise t' -> planes; second
// contraction (a warp per output row, both branches).  Code decisions use
// fp32 with explicitly rounded operations, so they do not depend on the
// compiler's contraction of multiplies and adds.
#include "lb_internal.cuh"

namespace lb {
namespace {

constexpr int kXorThreads = 256;

// D = 2^e for the largest magnitude A (see the header comment).
__device__ __forceinline__ float xor_scale(float A, int B) {
    const float top = (float)((1 << B) - 1);
    int e = -100;
    if (A > __fmul_rn(top, ldexpf(1.0f, e))) {
        int ea;
        frexpf(A, &ea);
        e = max(ea - B - 1, -100);
        while (A > __fmul_rn(top, ldexpf(1.0f, e))) ++e;
        while (e > -100 && A <= __fmul_rn(top, ldexpf(1.0f, e - 1))) --e;
    }
    return ldexpf(1.0f, e);
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float m = 0.0f;
    for (int w = 0; w < kXorThreads / 32; ++w) m = fmaxf(m, red[w]);
    return m;
}

// Element j of vector (m, b): g o x (kind: an lb_dtype of x) or t' (kind < 0).
__device__ __forceinline__ float xor_elem(const void* src, int kind, const __half* g, int64_t at,
                                          int j) {
    if (kind < 0) return reinterpret_cast<const float*>(src)[at + j];
    float xv;
    if (kind == LB_F16) xv = __half2float(reinterpret_cast<const __half*>(src)[at + j]);
    else if (kind == LB_BF16) xv = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[at + j]);
    else xv = reinterpret_cast<const float*>(src)[at + j];
    return __fmul_rn(__half2float(g[j]), xv);
}

// Quantise the n-element vectors (m, b) (one block each, blockIdx.x = m * nb + b)
// into B planes of nw words: planes[(m*nb + b)*B + p][w]; D to scale[m*nb + b].
__global__ void __launch_bounds__(kXorThreads) xor_quantise_kernel(
    const void* __restrict__ src, int kind, int64_t src_pitch, int64_t branch_pitch, int nb,
    const __half* __restrict__ g0, const __half* __restrict__ g1, int n, int B,
    uint32_t* __restrict__ planes, float* __restrict__ scale) {
    __shared__ float red[kXorThreads / 32];
    const int m = blockIdx.x / nb, b = blockIdx.x % nb;
    const __half* g = b == 0 ? g0 : g1;
    const int64_t at = (int64_t)m * src_pitch + (int64_t)b * branch_pitch;
    float A = 0.0f;
    for (int j = threadIdx.x; j < n; j += kXorThreads) A = fmaxf(A, fabsf(xor_elem(src, kind, g, at, j)));
    A = block_max(A, red);
    const float D = xor_scale(A, B);
    const float inv2d = __fdiv_rn(1.0f, __fmul_rn(2.0f, D));   // a power of two: exact
    const int nw = (n + 31) / 32;
    const int lane = threadIdx.x & 31;
    const int top = (1 << B) - 1;
    uint32_t* out = planes + (size_t)blockIdx.x * B * nw;
    for (int w = threadIdx.x >> 5; w < nw; w += kXorThreads / 32) {
        const int j = 32 * w + lane;
        const bool valid = j < n;
        int v = 0;
        if (valid) {
            const float q = __fmaf_rn(2.0f, floorf(__fmul_rn(xor_elem(src, kind, g, at, j), inv2d)), 1.0f);
            v = ((int)q + top) >> 1;       // in [0, 2^B - 1]
        }
        // plane p: bit set <=> sigma_p = -1 <=> bit p of v is 0 (valid columns only)
        uint32_t mine = 0u;
        for (int p = 0; p < B; ++p) {
            const uint32_t word = __ballot_sync(0xffffffffu, valid && !((v >> p) & 1));
            if (lane == p) mine = word;
        }
        if (lane < B) out[(size_t)lane * nw + w] = mine;
    }
    if (threadIdx.x == 0) scale[blockIdx.x] = D;
}

// Word w of packed row `row` of a matrix of n_rows rows of k signs (nw words).
__device__ __forceinline__ uint32_t sign_word(const uint32_t* P, int sliced, int64_t ld,
                                              int64_t n_rows, int64_t nw, int64_t row, int64_t w) {
    return sliced ? __ldg(P + sliced_offset(n_rows, nw, row, w)) : __ldg(P + row * ld + w);
}

// sum_j s_j q_j for one packed row against B planes, over n valid columns (nw
// words, the last one masked): the lane's share, to be summed over the warp.
__device__ __forceinline__ long long row_dot(const uint32_t* P, int sliced, int64_t ld,
                                             int64_t n_rows, int64_t row, const uint32_t* planes,
                                             int n, int B) {
    const int nw = (n + 31) / 32;
    const uint32_t last = (n & 31) ? ((1u << (n & 31)) - 1u) : 0xffffffffu;
    long long acc = 0;
    for (int w = threadIdx.x & 31; w < nw; w += 32) {
        const uint32_t s = sign_word(P, sliced, ld, n_rows, nw, row, w);
        const uint32_t mask = w == nw - 1 ? last : 0xffffffffu;
        long long d = 0;
        for (int p = B - 1; p >= 0; --p) d = 2 * d + __popc((s ^ planes[(size_t)p * nw + w]) & mask);
        acc += d;                    // sum_p 2^p popc_p
    }
    return acc;
}

__device__ __forceinline__ long long warp_sum(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

struct XorBranch {
    const uint32_t* P[2];
    int64_t ld[2];
    int sliced[2];
    const __half* s[2];      // stage 1: l; stage 2: h
};

// First contraction: a warp per (m, b, k): t'[m][b][k] = l_k * (D1 * T_k).
__global__ void __launch_bounds__(kXorThreads) xor_stage1_kernel(
    XorBranch V, int M, int nb, int in, int r, int B, const uint32_t* __restrict__ planes,
    const float* __restrict__ scale, float* __restrict__ tq) {
    const int64_t gw = ((int64_t)blockIdx.x * kXorThreads + threadIdx.x) >> 5;
    if (gw >= (int64_t)M * nb * r) return;
    const int k = (int)(gw % r);
    const int mb = (int)(gw / r);                   // m * nb + b
    const int b = mb % nb;
    const int nw = (in + 31) / 32;
    const long long pc = warp_sum(row_dot(V.P[b], V.sliced[b], V.ld[b], r, k,
                                          planes + (size_t)mb * B * nw, in, B));
    if ((threadIdx.x & 31) == 0) {
        const long long T = (long long)in * (long long)((1 << B) - 1) - 2 * pc;
        const float DT = __fmul_rn(scale[mb], __ll2float_rn(T));
        tq[(size_t)mb * r + k] = __fmul_rn(__half2float(V.s[b][k]), DT);
    }
}

// Second contraction: a warp per (m, i): y[m][i] = sum_b h_bi * D2_b * Z_bi.
__global__ void __launch_bounds__(kXorThreads) xor_stage2_kernel(
    XorBranch U, int M, int nb, int out, int r, int B, const uint32_t* __restrict__ planes,
    const float* __restrict__ scale, float* __restrict__ y) {
    const int64_t gw = ((int64_t)blockIdx.x * kXorThreads + threadIdx.x) >> 5;
    if (gw >= (int64_t)M * out) return;
    const int i = (int)(gw % out);
    const int m = (int)(gw / out);
    const int nw = (r + 31) / 32;
    float acc = 0.0f;
    for (int b = 0; b < nb; ++b) {
        const int mb = m * nb + b;
        const long long pc = warp_sum(row_dot(U.P[b], U.sliced[b], U.ld[b], out, i,
                                              planes + (size_t)mb * B * nw, r, B));
        const long long Z = (long long)r * (long long)((1 << B) - 1) - 2 * pc;
        acc = __fadd_rn(acc, __fmul_rn(__half2float(U.s[b][i]),
                                       __fmul_rn(scale[mb], __ll2float_rn(Z))));
    }
    if ((threadIdx.x & 31) == 0) y[(size_t)m * out + i] = acc;
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

struct XorLayout {
    size_t p1, s1, t, p2, s2, total;
};

XorLayout xor_layout(int64_t M, int64_t in, int64_t r, int nb, int B) {
    XorLayout L;
    const size_t mb = (size_t)M * nb;
    L.p1 = 0;
    L.s1 = L.p1 + up256(4 * mb * B * (size_t)((in + 31) / 32));
    L.t = L.s1 + up256(4 * mb);
    L.p2 = L.t + up256(4 * mb * (size_t)r);
    L.s2 = L.p2 + up256(4 * mb * B * (size_t)((r + 31) / 32));
    L.total = L.s2 + up256(4 * mb);
    return L;
}

bool xor_args_ok(int64_t M, int64_t in, int64_t out, int64_t r, int nb, int B) {
    // (grids of one warp per row: at most 2^33 rows of either contraction)
    return M > 0 && in > 0 && out > 0 && r > 0 && nb >= 1 && nb <= 2 && B >= 1 && B <= 24 &&
           in <= (1 << 24) && out <= (1 << 26) && r <= (1 << 24) && M <= (1 << 24) &&
           M * out <= ((int64_t)1 << 33) && M * nb * r <= ((int64_t)1 << 33);
}

}  // namespace
}  // namespace lb

using namespace lb;

extern "C" size_t lb_linear_xor_workspace_size(int64_t M, int64_t in, int64_t out, int64_t r,
                                               int n_branches, int bits) {
    if (!xor_args_ok(M, in, out, r, n_branches, bits)) return 0;
    return xor_layout(M, in, r, n_branches, bits).total;
}

extern "C" lb_status lb_linear_forward_xor(const void* x, lb_dtype x_dtype, int64_t M, int64_t in,
                                           int64_t out, int64_t r, const lb_branch* br,
                                           int n_branches, int bits, float* y, void* workspace,
                                           size_t ws_bytes, void* stream) {
    if (!x || !y || !br || !workspace) return LB_ERR_INVALID_ARG;
    if (!xor_args_ok(M, in, out, r, n_branches, bits)) return LB_ERR_INVALID_ARG;
    if (x_dtype != LB_F16 && x_dtype != LB_BF16 && x_dtype != LB_F32) return LB_ERR_INVALID_ARG;
    for (int b = 0; b < n_branches; ++b) {
        const lb_branch& B = br[b];
        if (!(B.Vp && B.Up && B.h && B.g && B.l && B.ld_v >= 0 && B.ld_u >= 0)) return LB_ERR_INVALID_ARG;
        if (B.layout != LB_LAYOUT_ROWS && B.layout != LB_LAYOUT_SLICES) return LB_ERR_INVALID_ARG;
        if (B.layout == LB_LAYOUT_SLICES && (B.ld_v || B.ld_u)) return LB_ERR_INVALID_ARG;
        if ((B.ld_v && B.ld_v < (in + 31) / 32) || (B.ld_u && B.ld_u < (r + 31) / 32))
            return LB_ERR_INVALID_ARG;
        const uintptr_t a = reinterpret_cast<uintptr_t>(B.Vp) | reinterpret_cast<uintptr_t>(B.Up);
        const uintptr_t s = reinterpret_cast<uintptr_t>(B.h) | reinterpret_cast<uintptr_t>(B.g) |
                            reinterpret_cast<uintptr_t>(B.l);
        if ((a & 3) || (s & 1)) return LB_ERR_ALIGNMENT;
    }
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y) |
         reinterpret_cast<uintptr_t>(workspace)) & 15)
        return LB_ERR_ALIGNMENT;
    const XorLayout L = xor_layout(M, in, r, n_branches, bits);
    if (ws_bytes < L.total) return LB_ERR_WORKSPACE;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return LB_ERR_CUDA;
    if (major != 10) return LB_ERR_UNSUPPORTED;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    uint32_t* p1 = reinterpret_cast<uint32_t*>(ws + L.p1);
    float* s1 = reinterpret_cast<float*>(ws + L.s1);
    float* tq = reinterpret_cast<float*>(ws + L.t);
    uint32_t* p2 = reinterpret_cast<uint32_t*>(ws + L.p2);
    float* s2 = reinterpret_cast<float*>(ws + L.s2);
    const int nb = n_branches;
    const lb_branch& b0 = br[0];
    const lb_branch& b1 = br[nb > 1 ? 1 : 0];
    XorBranch V, U;
    for (int b = 0; b < 2; ++b) {
        const lb_branch& B = b == 0 ? b0 : b1;
        V.P[b] = B.Vp; V.sliced[b] = B.layout == LB_LAYOUT_SLICES;
        V.ld[b] = B.ld_v ? B.ld_v : (in + 31) / 32;
        V.s[b] = reinterpret_cast<const __half*>(B.l);
        U.P[b] = B.Up; U.sliced[b] = B.layout == LB_LAYOUT_SLICES;
        U.ld[b] = B.ld_u ? B.ld_u : (r + 31) / 32;
        U.s[b] = reinterpret_cast<const __half*>(B.h);
    }
    const unsigned mbl = (unsigned)(M * nb);
    xor_quantise_kernel<<<mbl, kXorThreads, 0, s>>>(
        x, (int)x_dtype, in, 0, nb, reinterpret_cast<const __half*>(b0.g),
        reinterpret_cast<const __half*>(b1.g), (int)in, bits, p1, s1);
    const int64_t w1 = M * nb * r, w2 = M * out;
    const int wpb = kXorThreads / 32;
    xor_stage1_kernel<<<(unsigned)((w1 + wpb - 1) / wpb), kXorThreads, 0, s>>>(
        V, (int)M, nb, (int)in, (int)r, bits, p1, s1, tq);
    xor_quantise_kernel<<<mbl, kXorThreads, 0, s>>>(tq, -1, (int64_t)nb * r, r, nb, nullptr,
                                                    nullptr, (int)r, bits, p2, s2);
    xor_stage2_kernel<<<(unsigned)((w2 + wpb - 1) / wpb), kXorThreads, 0, s>>>(
        U, (int)M, nb, (int)out, (int)r, bits, p2, s2, y);
    return cudaGetLastError() == cudaSuccess ? LB_OK : LB_ERR_CUDA;
}
