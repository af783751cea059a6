// Internal declarations shared by the CUDA sources of liblb.so.
//
// The decode path is a persistent "phase program": a list of phases, each a
// set of GEMV jobs out[row] (+)= oscale[row] * sum_col sign(P[row][col]) * v[col]
// over packed sign matrices P, separated by grid-wide waits.  One linear is two
// phases (the V contraction, then the U contraction); a decoder layer is eight.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/lb.h"

namespace lb {

// ---------------------------------------------------------------- constants
constexpr int kDecodeThreads = 512;          // 16 warps per CTA, one CTA per SM
constexpr int kDecodeWarps = kDecodeThreads / 32;
constexpr int kCtasPerSm = 1;
constexpr int kSliceElems = 512;             // columns covered by one lookup table
constexpr int kSliceWords = kSliceElems / 32;
constexpr int kRowBlock = 32;                // rows per warp work item (4 steps x 8 rows)
constexpr int kLutBytes = 64 * 1024;         // one table: 64 chunks x 256 entries x fp32
constexpr int kTables = 2;                   // tables resident at once (a batch of <= 2 tiles)
// Tables sit at shared-window addresses kTableAddr0 + t * 64 KB, so the table
// of a lookup is selected by bits 16-17 of the address (see lb_decode.cu).
constexpr uint32_t kTableAddr0 = 64u * 1024u;
constexpr int kVecPad = kSliceElems + kSliceElems / 16;   // staged slice, 4 floats of pad per 64
constexpr int kDepth = 2;                    // rowblocks each warp has in flight (registers)
constexpr int kRowBlockBytes = kRowBlock * kSliceWords * 4;   // 2 KB of signs
constexpr int kMaxLinearJobs = 16;           // per phase in a single-linear call
constexpr int kMaxPhaseJobs = 16;            // jobs of one phase (stack phases use <= 6)
constexpr int kMaxDecodeM = 8;               // rows of x the decode path takes at once
constexpr float kRmsEps = 1e-5f;

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
    unsigned int barrier;     // grid barrier arrival counter (zeroed per call)
    int error;                // 0 or LB_ERR_TIMEOUT (zeroed per call)
    unsigned int exit_count;
    int pad[61];
};
static_assert(sizeof(WsHeader) == 256, "header must be 256 bytes");

// Where a job's vector v[col] comes from.
enum VecKind : int {
    VK_X_F16 = 0,      // v = g[j] * x[j], x fp16
    VK_X_BF16 = 1,     // v = g[j] * x[j], x bf16
    VK_X_F32 = 2,      // v = g[j] * x[j], x fp32
    VK_T = 3,          // v = l[k] * t[k] * rs, rs = rsqrt(sumsq/n + eps) or 1
    VK_GQA = 4,        // v = g[j] * src[(j / (group*hd)) * hd + j % hd]
    VK_SILU_MUL = 5,   // v = g[j] * silu(src[j]) * src2[j]
};

struct alignas(64) LbJob {
    const uint32_t* P;        // packed rows [rows][ldw] (ldw = row pitch in words)
    const void* src;          // vector source
    const float* src2;        // second source (VK_SILU_MUL)
    const __half* vscale;     // g (first contraction) or l (second)
    const __half* oscale;     // h (second contraction) or nullptr
    float* out;               // fp32 accumulation target [rows], zeroed beforehand
    const float* norm_sumsq;  // VK_T: sum of squares of the normed input, or nullptr
    float* acc_sumsq;         // owner of a slice adds sum(src^2) of the slice here
    float* resid_init;        // owner of a slice writes float(src) of the slice here
    int rows, cols, ldw, kind;
    int n_slices, n_rowblocks, unit_begin, norm_n;
    int gqa_ghd, gqa_hd;
    int rg;                   // rowblocks per row group (units run group, slice, rowblock)
    int sliced;               // P is in the sliced layout (LB_LAYOUT_SLICES), ldw unused
};

struct alignas(16) LbPhase {
    int job_begin, n_jobs, n_units, zero_n;
    float* zero_ptr;          // if set, the CTAs zero zero_n floats here during the phase
    int split_off;            // offset of this phase's split_g+1 unit boundaries in the split table
    int split_g;              // CTAs the split was made for (-1 or another grid: even split)
    int next_job_begin;       // jobs of the following phase (0 / 0 for the last phase), so a
    int next_n_jobs;          // CTA can fetch that phase's plan without reading its header first
    int starts_g;             // CTAs the start table was made for (-1: no table, compute on device)
    int pad;
};
static_assert(sizeof(LbPhase) == 48, "LbPhase is copied in 16-byte pieces");

// A tile: the units of one slice of one job that a CTA runs in one go.
struct LbTile {
    int job, slice, rb0, nrb;
};

// A CTA's first batch of a phase (its unit range and the tiles of the range
// that the first batch takes), computed on the host when the plan is made so
// the CTA does not search for them between two phases.
struct alignas(16) LbStart {
    int u, u_end, j, nt, n_rb, pad[3];
    LbTile t[2];
};
static_assert(sizeof(LbStart) == 64, "LbStart is copied in 16-byte pieces");

__host__ __device__ __forceinline__ int find_job(const LbJob* jobs, int j, int j_end, int u) {
    while (j + 1 < j_end && jobs[j + 1].unit_begin <= u) ++j;
    return j;
}

// The tile of a unit range that starts at unit u (u < u_end).  A job's units
// run row group by row group, slice by slice inside a group, so the CTAs
// holding the slices of one group stream the same rows together and each DRAM
// page is read while it is open.
__host__ __device__ __forceinline__ LbTile next_tile(const LbJob* jobs, int n_jobs, int& j, int u,
                                                     int u_end) {
    j = find_job(jobs, j, n_jobs, u);
    const LbJob& J = jobs[j];
    const int local = u - J.unit_begin;
    const int per_group = J.rg * J.n_slices;
    const int g = local / per_group;
    const int off = local - g * per_group;
    const int left = J.n_rowblocks - g * J.rg;
    const int rows_g = J.rg < left ? J.rg : left;
    const int s = off / rows_g;
    const int rbi = off - s * rows_g;
    const int rest = u_end - u;
    return LbTile{j, s, g * J.rg + rbi, rows_g - rbi < rest ? rows_g - rbi : rest};
}

// Stack plans are prepared once and reused with different x / y buffers, so
// job pointers that mean "the call's x" or "the call's y" are stored as tags.
#define LB_TAG_X ((const void*)1)
#define LB_TAG_Y ((const void*)2)

// Dynamic shared memory: everything below the first table (staged vectors,
// reduction scratch, the phase plan) starts at the window's dynamic base
// (1 KB on sm_100) and must end below kTableAddr0; the size requested covers
// the tables for any base below that.
constexpr int kMiscBytes = 4 * kTables * kVecPad + 4 * 32 + 64 +
                           2 * (128 + kMaxPhaseJobs * (int)sizeof(LbJob));
constexpr int kDecodeSmem = (int)kTableAddr0 + kTables * kLutBytes;
static_assert(kDecodeSmem <= 227 * 1024, "decode kernel shared memory over the per-CTA limit");
static_assert(kMiscBytes + 1024 <= (int)kTableAddr0, "decode plan cache overlaps the tables");

// Plan of a single linear call, passed by value as a kernel parameter.
constexpr int kMaxGrid = 256;                // CTAs a split table has room for
// Costs of the host's work split, in 1/16 of a round of 16 rowblocks (one per rowblock).
constexpr int kBatchCost = 0;                // staging a batch's vectors
constexpr int kTileCost = 12;                // building a tile's table (and, with kBatchCost 0, its staging)

struct LinearPlan {
    LbJob jobs[2 * kMaxLinearJobs];
    LbPhase phases[2];
    int split[2 * (kMaxGrid + 1)];           // per-phase unit boundaries of the CTAs
};

// ------------------------------------------------------- sliced layout
// LB_LAYOUT_SLICES (include/lb.h): a packed matrix of n rows with nw words
// per row is stored slice by slice, slice s (words 16s .. 16s+15 of every row)
// as a block of n rows; full slices have a pitch of 16 words, the last one the
// words it holds rounded up to a multiple of 4.  Block s starts at word 16*n*s.
__host__ __device__ __forceinline__ int64_t sliced_pitch(int64_t nw, int64_t s) {
    const int64_t last = (nw - 1) >> 4;
    return s < last ? 16 : ((nw - 16 * last) + 3) & ~(int64_t)3;
}
__host__ __device__ __forceinline__ int64_t sliced_offset(int64_t n, int64_t nw, int64_t row,
                                                          int64_t w) {
    const int64_t s = w >> 4;
    return 16 * n * s + row * sliced_pitch(nw, s) + (w & 15);
}
__host__ __device__ __forceinline__ int64_t sliced_words(int64_t n, int64_t nw) {
    const int64_t last = (nw - 1) >> 4;
    return n * (16 * last + sliced_pitch(nw, last));
}

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint4 ld_stream_v4(const uint32_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" :: "l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ void red_add_v4_f32(float* p, float a, float b, float c, float d) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add_u32(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
// Shared-memory load / store at a 32-bit shared-window address plus a
// constant byte offset, which goes into the instruction instead of a register.
template <int kOff>
__device__ __forceinline__ float lds_f32_off(uint32_t saddr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(saddr), "n"(kOff));
    return v;
}
template <int kOff>
__device__ __forceinline__ void sts_f32_off(uint32_t saddr, float v) {
    asm volatile("st.shared.f32 [%0+%1], %2;" :: "r"(saddr), "n"(kOff), "f"(v) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :: "r"(dst), "l"(map), "r"(bar), "r"(x), "r"(y) : "memory");
}

// ------------------------------------------------------------ host helpers
int device_sm_count();               // SMs of the current device (cached per device)
bool device_is_sm100();
cudaError_t decode_configure();      // one-time kernel attribute setup per device

// Decode phase program launches (lb_decode.cu).
cudaError_t launch_linear_plan(const LinearPlan& plan, WsHeader* hdr, int n_phases,
                               cudaStream_t s);
cudaError_t launch_stack_plan(const LbPhase* phases, const LbJob* jobs, const int* splits,
                              const LbStart* starts, int n_phases, WsHeader* hdr, const void* x,
                              float* y, cudaStream_t s);
int decode_grid();                   // CTAs of a decode launch on the current device
// Row-group sizes of a phase's jobs for a grid of G CTAs (search: try scalings).
void plan_row_groups(LbJob* jobs, int n_jobs, int n_units, int G, bool search);
// Cost-balanced contiguous unit ranges for the G CTAs of a phase (out: G+1
// boundaries); returns the largest CTA cost of the split.
long long balanced_split(const LbJob* jobs, int n_jobs, int n_units, int G, int* out);
// The first batch of each CTA of each phase from the split table (G <= kMaxGrid);
// out holds n_phases * kMaxGrid records, phase q's at q * kMaxGrid.  Sets starts_g.
void plan_starts(LbPhase* phases, int n_phases, const LbJob* jobs, const int* split, int G,
                 LbStart* out);

// Tensor-core prefill path (lb_prefill.cu).
// lb_linear_forward uses the tensor cores from this many rows: measured on the
// 7B gate shape (4096 -> 11008), the two paths are level at 14-15 rows at 1.0
// bits/weight while the lookup-table kernels (two launches of 8 rows) stay ahead
// through 15 rows at 0.1; from 16 rows the tensor cores are ahead or within 5%.
constexpr int kPrefillMinM = 16;
cudaError_t prefill_configure();
// with_split: room for the stage-1 K split's partial sums (tens of MB when the
// split is possible); without it the launch never splits stage 1.
size_t prefill_workspace_bytes(int64_t M, int64_t in, int64_t r, bool with_split = true);
bool prefill_shape_ok(int64_t M, int64_t in, int64_t out, int64_t r);
cudaError_t launch_prefill(const void* x, int x_kind, int64_t M, int64_t in, int64_t out,
                           int64_t r, const lb_branch* br, int nb, float* y, void* workspace,
                           cudaStream_t s, bool allow_split = true);

// Which kernels a linear call runs (lb_api.cu).
enum LinearRoute { kRouteDecode = 0, kRoutePrefill = 1, kRoutePrefillNoSplit = 2 };
// The tensor-core path when lb_linear_forward would take it (shape and pointer
// alignment), else the decode path.
LinearRoute default_route(int64_t M, int64_t in, int64_t out, int64_t r, const lb_branch* br,
                          int n_branches);
// Workspace bytes of the decode path, and of any route.
size_t decode_workspace_bytes(int64_t M, int64_t r, int n_branches);
size_t route_workspace_bytes(LinearRoute route, int64_t M, int64_t in, int64_t r, int nb);
// lb_linear_forward on a given route, with its argument checks; the call is
// refused (LB_ERR_WORKSPACE) unless ws_bytes >= ws_need and >= what the route needs.
lb_status linear_forward_route(const void* x, lb_dtype x_dtype, int64_t M, int64_t in,
                               int64_t out, int64_t r, const lb_branch* br, int n_branches,
                               float* y, void* workspace, size_t ws_bytes, size_t ws_need,
                               cudaStream_t s, LinearRoute route);

// Packer (lb_pack.cu).  sliced: write the sliced layout (ld_words unused).
cudaError_t launch_pack(const float* latent, int64_t rows, int64_t cols, int64_t ld, int axis,
                        uint32_t* packed, int64_t ld_words, bool sliced, cudaStream_t s);

}  // namespace lb
