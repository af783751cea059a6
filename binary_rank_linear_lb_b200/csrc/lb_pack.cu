// Sign packer: fp32 latent factor -> packed sign words (bit = latent < 0).
//
// "Samsung LittleBit: A 13B LLM Under 1 GB ..." (explainx.ai), "How it works",
// item 1: at inference only the signs of the latent factors are used, one bit
// per entry.  The packed layout is documented in include/lb.h.
//
// Both kernels read the latent exactly once with coalesced 128-byte warp loads,
// so they run at HBM speed; the packed output is 1/32 of the bytes read.  The
// output goes to the row-major layout (pitch ld_words) or to the sliced one
// (the packed matrix regrouped by 16-word slices, include/lb.h).
#include "lb_internal.cuh"

namespace lb {
namespace {

// axis = 1: one warp per (row, group of 32 output words).  Lane l reads column
// 32*w + l for w = 0..31 and a ballot forms word w; lane w keeps it.
// Word w of packed row `row` (n packed rows of nw words): where it goes.
__device__ __forceinline__ int64_t out_index(bool sliced, int64_t n, int64_t nw, int64_t ld_words,
                                             int64_t row, int64_t w) {
    return sliced ? sliced_offset(n, nw, row, w) : row * ld_words + w;
}

// Words written per packed row: the pitch (row-major), or the words of every
// slice including the last slice's padding (sliced).
__host__ __device__ __forceinline__ int64_t words_per_row(bool sliced, int64_t nw, int64_t ld_words) {
    const int64_t last = (nw - 1) >> 4;
    return sliced ? 16 * last + sliced_pitch(nw, last) : ld_words;
}

__global__ void __launch_bounds__(256) pack_rows_kernel(const float* __restrict__ latent,
                                                        int64_t rows, int64_t cols, int64_t ld,
                                                        uint32_t* __restrict__ packed,
                                                        int64_t ld_words, bool sliced) {
    const int64_t nw = (cols + 31) / 32;
    const int64_t W = words_per_row(sliced, nw, ld_words);
    const int lane = threadIdx.x & 31;
    const int64_t wg = blockIdx.x;                       // group of 32 words
    for (int64_t row = (int64_t)blockIdx.y * 8 + (threadIdx.x >> 5); row < rows;
         row += (int64_t)gridDim.y * 8) {
        const float* src = latent + row * ld;
        uint32_t mine = 0;
#pragma unroll 8
        for (int w = 0; w < 32; ++w) {
            const int64_t c = (wg * 32 + w) * 32 + lane;
            bool neg = false;
            if (c < cols) neg = __ldg(src + c) < 0.0f;
            const uint32_t word = __ballot_sync(0xffffffffu, neg);
            if (lane == w) mine = word;
        }
        const int64_t ow = wg * 32 + lane;
        if (ow < W) packed[out_index(sliced, rows, nw, ld_words, row, ow)] = mine;
    }
}

// axis = 0: one thread per (column, word).  Thread c reads rows 32*w .. 32*w+31
// of column c; neighbouring threads read neighbouring columns, so every warp
// load is one coalesced 128-byte line.
__global__ void __launch_bounds__(256) pack_cols_kernel(const float* __restrict__ latent,
                                                        int64_t rows, int64_t cols, int64_t ld,
                                                        uint32_t* __restrict__ packed,
                                                        int64_t ld_words, bool sliced) {
    const int64_t c = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (c >= cols) return;
    const int64_t nw = (rows + 31) / 32;
    const int64_t W = words_per_row(sliced, nw, ld_words);
    for (int64_t w = blockIdx.y; w < W; w += gridDim.y) {
        uint32_t word = 0;
        const int64_t r0 = w * 32;
        if (r0 + 32 <= rows) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                word |= (uint32_t)(__ldg(latent + (r0 + i) * ld + c) < 0.0f) << i;
        } else {
            for (int i = 0; i < 32 && r0 + i < rows; ++i)
                word |= (uint32_t)(__ldg(latent + (r0 + i) * ld + c) < 0.0f) << i;
        }
        packed[out_index(sliced, cols, nw, ld_words, c, w)] = word;
    }
}

}  // namespace

cudaError_t launch_pack(const float* latent, int64_t rows, int64_t cols, int64_t ld, int axis,
                        uint32_t* packed, int64_t ld_words, bool sliced, cudaStream_t s) {
    const int64_t W = words_per_row(sliced, ((axis == 1 ? cols : rows) + 31) / 32, ld_words);
    if (axis == 1) {
        const int64_t groups = (W + 31) / 32;
        const int64_t gy = (rows + 7) / 8;
        dim3 grid((unsigned)groups, (unsigned)(gy < 65535 ? gy : 65535));
        if (groups > 0x7fffffff) return cudaErrorInvalidValue;
        pack_rows_kernel<<<grid, 256, 0, s>>>(latent, rows, cols, ld, packed, ld_words, sliced);
    } else {
        const int64_t gx = (cols + 255) / 256;
        if (gx > 0x7fffffff) return cudaErrorInvalidValue;
        dim3 grid((unsigned)gx, (unsigned)(W < 65535 ? W : 65535));
        pack_cols_kernel<<<grid, 256, 0, s>>>(latent, rows, cols, ld, packed, ld_words, sliced);
    }
    return cudaGetLastError();
}

}  // namespace lb
