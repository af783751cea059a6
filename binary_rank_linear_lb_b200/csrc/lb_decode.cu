// Batch-1 / small-M decode path: a persistent phase program of lookup-table
// GEMVs over packed signs.
//
// The layer ("Samsung LittleBit: A 13B LLM Under 1 GB ...", "How it works",
// items 1-3) is two binary contractions with scales:
//   t = sign(V)^T (g o x),  y += h o (sign(U) (l o t))  for each branch.
// Each contraction is a GEMV whose matrix is a packed sign matrix P[rows][cols]
// and whose vector v is built on the fly (g o x, l o t, ...).
//
// Lookup tables.  For a slice of 1024 columns the CTA tabulates, for every
// chunk of 8 consecutive columns, all 256 signed sums  T_c[e] = sum_q (bit q of
// e ? -v_q : +v_q).  One byte of a packed row then costs one shared-memory load
// and one add instead of eight sign-selects and adds.  Table layout (bytes):
//   lut + (qb>>1)*64K + e*256 + (qb&1)*128 + w*4    chunk c = 4w + qb
// so the 32 lanes of a warp, which always look up 32 different words w, hit 32
// different banks.  A single PRMT assembles the address from the sign byte and
// a per-lane constant, so a lookup is PRMT + LDS + FADD.
//
// Work split.  A job (one matrix) is cut into units of 32 rows x one slice.
// The units of a phase are dealt to the CTAs in contiguous, equal ranges; a CTA
// rebuilds its table whenever its range enters a new (job, slice).  Partial
// row sums over a slice are added to the fp32 output with red.global.add, so the
// V-contraction result t never leaves L2 between the two phases.
//
// Phases are separated by a grid-wide wait (bounded spin); the kernel is
// launched cooperatively so that every CTA is resident.  While waiting, HBM is
// kept busy by L2 prefetches of the next phase's first sign rows.
#include "lb_internal.cuh"

namespace lb {
namespace {

constexpr long long kSpinLimitCycles = 4000000000LL;   // ~2 s at 2 GHz
constexpr int kPrefetchUnits = 8;                       // units prefetched per CTA ahead
constexpr int kPrefetchAhead = 2 * kDecodeWarps;        // rowblocks ahead within a tile
constexpr int kVecPad = kSliceElems + kSliceElems / 32; // padded staged vector

struct Smem {
    uint32_t lut;     // shared-window address of the table, a multiple of 64 KB
    float* vec;       // staged vector slice, index e + e/32
    float* red;       // 32 floats of reduction scratch
    int* flag;        // one int
};

__device__ __forceinline__ Smem smem_layout() {
    extern __shared__ __align__(16) unsigned char dsmem[];
    Smem s;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(dsmem);
    s.lut = (sbase + 65535u) & ~65535u;
    unsigned char* after = dsmem + (s.lut - sbase) + kLutBytes;
    s.vec = reinterpret_cast<float*>(after);
    s.red = s.vec + kVecPad;
    s.flag = reinterpret_cast<int*>(s.red + 32);
    return s;
}

__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }

// Grid-wide wait: every CTA adds one arrival, then waits until `target`
// arrivals are counted.  Gives up after kSpinLimitCycles and records
// LB_ERR_TIMEOUT; returns false if this CTA must stop.
__device__ bool grid_sync(WsHeader* hdr, unsigned target, int* flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        red_release_add_u32(&hdr->barrier, 1u);
        int ok = 1;
        const long long t0 = clock64();
        unsigned spins = 0;
        while (ld_acquire_u32(&hdr->barrier) < target) {
            if ((++spins & 63u) == 0) {
                if (*reinterpret_cast<volatile int*>(&hdr->error) != 0) { ok = 0; break; }
                if (clock64() - t0 > kSpinLimitCycles) {
                    atomicExch(&hdr->error, (int)LB_ERR_TIMEOUT);
                    ok = 0;
                    break;
                }
            }
        }
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

// First unit of CTA `cta` in a phase with n units over G CTAs.
__device__ __forceinline__ int unit_split(int n, int cta, int G) {
    return (int)(((long long)n * cta) / G);
}

// Stage v for slice s of job J into shared memory (zero past cols), do the
// slice owner's side duties, then build the 128 chunk tables.
__device__ void stage_and_build(const LbJob& J, int s, bool owner, const Smem& sm) {
    const int j0 = s * kSliceElems;
    float rs = 1.0f;
    if (J.kind == VK_T && J.norm_sumsq != nullptr)
        rs = rsqrtf(__ldcg(J.norm_sumsq) / (float)J.norm_n + kRmsEps);
    float sq = 0.0f;
    for (int e = threadIdx.x; e < kSliceElems; e += kDecodeThreads) {
        const int j = j0 + e;
        float v = 0.0f;
        if (j < J.cols) {
            float raw;
            switch (J.kind) {
                case VK_X_F16:
                    raw = __half2float(reinterpret_cast<const __half*>(J.src)[j]);
                    v = __half2float(__ldg(J.vscale + j)) * raw;
                    break;
                case VK_X_BF16:
                    raw = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(J.src)[j]);
                    v = __half2float(__ldg(J.vscale + j)) * raw;
                    break;
                case VK_X_F32:
                    raw = __ldcg(reinterpret_cast<const float*>(J.src) + j);
                    v = __half2float(__ldg(J.vscale + j)) * raw;
                    break;
                case VK_T:
                    raw = __ldcg(reinterpret_cast<const float*>(J.src) + j);
                    v = __half2float(__ldg(J.vscale + j)) * (raw * rs);
                    break;
                case VK_GQA: {
                    const int head = j / J.gqa_ghd;
                    raw = __ldcg(reinterpret_cast<const float*>(J.src) + head * J.gqa_hd +
                                 (j % J.gqa_hd));
                    v = __half2float(__ldg(J.vscale + j)) * raw;
                    break;
                }
                default: {  // VK_SILU_MUL
                    const float gt = __ldcg(reinterpret_cast<const float*>(J.src) + j);
                    raw = silu(gt) * __ldcg(J.src2 + j);
                    v = __half2float(__ldg(J.vscale + j)) * raw;
                    break;
                }
            }
            if (owner) {
                sq += raw * raw;
                if (J.resid_init != nullptr) J.resid_init[j] = raw;
            }
        }
        sm.vec[e + (e >> 5)] = v;
    }
    if (owner && J.acc_sumsq != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if ((threadIdx.x & 31) == 0) sm.red[threadIdx.x >> 5] = sq;
        __syncthreads();
        if (threadIdx.x == 0) {
            float tot = 0.0f;
            for (int w = 0; w < kDecodeWarps; ++w) tot += sm.red[w];
            atomicAdd(J.acc_sumsq, tot);
        }
    }
    __syncthreads();

    // Table build.  Warp wp fills byte position qb = wp/4 of every word and
    // the 4 high nibbles (wp%4)*4 .. +3; lane = word w of the slice.
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int qb = wp >> 2, hb = (wp & 3) * 4;
    const float* u = sm.vec + 32 * lane + 8 * qb + lane;   // padded index of element 32w+8qb
    const float u0 = u[0], u1 = u[1], u2 = u[2], u3 = u[3];
    const float u4 = u[4], u5 = u[5], u6 = u[6], u7 = u[7];
    // bit q of the entry index set <=> element q enters with sign -1
    const float p01[4] = {u0 + u1, u1 - u0, u0 - u1, -u0 - u1};
    const float p23[4] = {u2 + u3, u3 - u2, u2 - u3, -u2 - u3};
    const float q45[4] = {u4 + u5, u5 - u4, u4 - u5, -u4 - u5};
    const float q67[4] = {u6 + u7, u7 - u6, u6 - u7, -u6 - u7};
    float lo[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) lo[m] = p01[m & 3] + p23[m >> 2];
    const uint32_t base = sm.lut + (uint32_t)(qb >> 1) * 65536u + (uint32_t)(qb & 1) * 128u +
                          (uint32_t)lane * 4u;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int hn = hb + n;
        const float hi = q45[hn & 3] + q67[hn >> 2];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const uint32_t addr = base + (uint32_t)(hn * 16 + m) * 256u;
            asm volatile("st.shared.f32 [%0], %1;" :: "r"(addr), "f"(hi + lo[m]) : "memory");
        }
    }
    __syncthreads();
}

// Sign words [wbase, wbase+4) of `row`, zero outside the matrix.
__device__ __forceinline__ uint4 load_group(const LbJob& J, int row, int wbase, bool vec4) {
    uint4 d = make_uint4(0u, 0u, 0u, 0u);
    if (row < J.rows && wbase < J.ldw) {
        const uint32_t* p = J.P + (size_t)row * (size_t)J.ldw + wbase;
        if (vec4) {
            d = ld_stream_v4(p);
        } else {
            d.x = ld_stream_u32(p);
            if (wbase + 1 < J.ldw) d.y = ld_stream_u32(p + 1);
            if (wbase + 2 < J.ldw) d.z = ld_stream_u32(p + 2);
            if (wbase + 3 < J.ldw) d.w = ld_stream_u32(p + 3);
        }
    }
    return d;
}

__device__ __forceinline__ void prefetch_rowblock(const LbJob& J, int s, int rb, int lane) {
    const int row = rb * kRowBlock + lane;
    const int w0 = s * kSliceWords;
    if (row < J.rows && w0 < J.ldw) {
        const uint32_t* p = J.P + (size_t)row * (size_t)J.ldw + w0;
        const int nw = min(kSliceWords, J.ldw - w0);
        prefetch_l2(p);
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(p) >> 7;
        const uintptr_t a1 = reinterpret_cast<uintptr_t>(p + nw - 1) >> 7;
        if (a1 != a0) prefetch_l2(p + nw - 1);
    }
}

// Look up rowblocks [rb0, rb0+nrb) of slice s of job J against the table.
// Lane l = 8*rho + gam reads words 4*gam..4*gam+3 of row 4*i + rho of the
// rowblock (i = 0..7) and, in step jj, byte (jj + rho) % 4 of each word, so the
// 32 lanes of a warp always touch 32 different words.
__device__ void lookup_rowblocks(const LbJob& J, int s, int rb0, int nrb, const Smem& sm) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int rho = lane >> 3, gam = lane & 7;
    uint32_t B[4], S[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const uint32_t qbj = (uint32_t)((jj + rho) & 3);
        B[jj] = ((qbj & 1u) * 128u + 16u * (uint32_t)gam) |
                (((sm.lut >> 16) + (qbj >> 1)) << 16);
        S[jj] = 0x7604u | (qbj << 4);
    }
    const int wbase = s * kSliceWords + 4 * gam;
    const bool vec4 = (J.ldw & 3) == 0;
    const float hscale_default = 1.0f;
    for (int rb = rb0 + wp; rb < rb0 + nrb; rb += kDecodeWarps) {
        if (rb + kPrefetchAhead < rb0 + nrb) prefetch_rowblock(J, s, rb + kPrefetchAhead, lane);
        const int row0 = rb * kRowBlock;
        uint4 d[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = load_group(J, row0 + 4 * i + rho, wbase, vec4);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w4[4] = {d[i].x, d[i].y, d[i].z, d[i].w};
            float a = 0.0f;
#pragma unroll
            for (int reg = 0; reg < 4; ++reg) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    a += lds_f32(prmt(w4[reg], B[jj], S[jj]) + 4u * (uint32_t)reg);
            }
            acc[i] = a;
        }
        // Transpose-reduce over the 8 lanes of a rho group: afterwards lane gam
        // holds the full slice sum of row-step i = gam.
        const bool up4 = (gam & 4) != 0, up2 = (gam & 2) != 0, up1 = (gam & 1) != 0;
        float n4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float send = up4 ? acc[k] : acc[k + 4];
            const float keep = up4 ? acc[k + 4] : acc[k];
            n4[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
        float n2[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float send = up2 ? n4[k] : n4[k + 2];
            const float keep = up2 ? n4[k + 2] : n4[k];
            n2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        }
        const float send1 = up1 ? n2[0] : n2[1];
        const float keep1 = up1 ? n2[1] : n2[0];
        const float tot = keep1 + __shfl_xor_sync(0xffffffffu, send1, 1);
        const int row = row0 + 4 * gam + rho;
        if (row < J.rows) {
            const float hs = J.oscale ? __half2float(__ldg(J.oscale + row)) : hscale_default;
            red_add_f32(J.out + row, tot * hs);
        }
    }
}

__device__ __forceinline__ int find_job(const LbJob* jobs, int j, int j_end, int u) {
    while (j + 1 < j_end && jobs[j + 1].unit_begin <= u) ++j;
    return j;
}

struct CallArgs {
    const void* x;
    float* y;
};

template <typename T>
__device__ __forceinline__ T* resolve(T* p, const CallArgs& a) {
    if ((const void*)p == LB_TAG_X) return (T*)a.x;
    if ((const void*)p == LB_TAG_Y) return (T*)a.y;
    return p;
}

// Local copy of a job with the call's x / y substituted for their tags.
__device__ __forceinline__ LbJob fetch_job(const LbJob* jobs, int j, const CallArgs& a) {
    LbJob J = jobs[j];
    J.src = resolve(J.src, a);
    J.out = resolve(J.out, a);
    J.resid_init = resolve(J.resid_init, a);
    return J;
}

__device__ void run_phase(const LbPhase& ph, const LbJob* jobs, const Smem& sm,
                          const CallArgs& args) {
    const int G = gridDim.x, cta = blockIdx.x;
    float* zp = resolve(ph.zero_ptr, args);
    if (zp != nullptr) {
        for (int i = cta * kDecodeThreads + threadIdx.x; i < ph.zero_n; i += G * kDecodeThreads)
            zp[i] = 0.0f;
    }
    int u = unit_split(ph.n_units, cta, G);
    const int u_end = unit_split(ph.n_units, cta + 1, G);
    int j = ph.job_begin;
    const int j_end = ph.job_begin + ph.n_jobs;
    while (u < u_end) {
        j = find_job(jobs, j, j_end, u);
        const LbJob J = fetch_job(jobs, j, args);
        const int local = u - J.unit_begin;
        const int s = local / J.n_rowblocks;
        const int rb0 = local - s * J.n_rowblocks;
        const int nrb = min(J.n_rowblocks - rb0, u_end - u);
        stage_and_build(J, s, rb0 == 0, sm);
        lookup_rowblocks(J, s, rb0, nrb, sm);
        u += nrb;
        __syncthreads();
    }
}

// L2 prefetch of the first kPrefetchUnits units this CTA will take in phase ph.
__device__ void prefetch_phase(const LbPhase& ph, const LbJob* jobs) {
    const int G = gridDim.x, cta = blockIdx.x;
    const int u0 = unit_split(ph.n_units, cta, G);
    const int u1 = min(unit_split(ph.n_units, cta + 1, G), u0 + kPrefetchUnits);
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    for (int u = u0 + wp; u < u1; u += kDecodeWarps) {
        const int j = find_job(jobs, ph.job_begin, ph.job_begin + ph.n_jobs, u);
        const LbJob& J = jobs[j];
        const int local = u - J.unit_begin;
        const int s = local / J.n_rowblocks;
        prefetch_rowblock(J, s, local - s * J.n_rowblocks, lane);
    }
}

__device__ void run_program(const LbPhase* phases, int n_phases, const LbJob* jobs,
                            WsHeader* hdr, const CallArgs& args) {
    const Smem sm = smem_layout();
    const unsigned G = gridDim.x;
    for (int p = 0; p < n_phases; ++p) {
        if (p + 1 < n_phases) prefetch_phase(phases[p + 1], jobs);
        run_phase(phases[p], jobs, sm, args);
        if (p + 1 < n_phases) {
            if (!grid_sync(hdr, (unsigned)(p + 1) * G, sm.flag)) return;
        }
    }
}

__global__ void __launch_bounds__(kDecodeThreads, 1)
linear_program_kernel(const __grid_constant__ LinearPlan plan, int n_phases, WsHeader* hdr) {
    const CallArgs args = {nullptr, nullptr};
    run_program(plan.phases, n_phases, plan.jobs, hdr, args);
}

__global__ void __launch_bounds__(kDecodeThreads, 1)
stack_program_kernel(const LbPhase* __restrict__ phases, const LbJob* __restrict__ jobs,
                     int n_phases, WsHeader* hdr, const void* x, float* y) {
    const CallArgs args = {x, y};
    run_program(phases, n_phases, jobs, hdr, args);
}

cudaError_t launch_coop(const void* fn, void** args, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)device_sm_count());
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = kDecodeSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

cudaError_t decode_configure() {
    cudaError_t e = cudaFuncSetAttribute(linear_program_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kDecodeSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(stack_program_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDecodeSmem);
    if (e != cudaSuccess) return e;
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, linear_program_kernel, kDecodeThreads,
                                                      kDecodeSmem);
    if (e != cudaSuccess) return e;
    return nb >= 1 ? cudaSuccess : cudaErrorCooperativeLaunchTooLarge;
}

cudaError_t launch_linear_plan(const LinearPlan& plan, WsHeader* hdr, int n_phases,
                               cudaStream_t s) {
    void* args[] = {const_cast<LinearPlan*>(&plan), &n_phases, &hdr};
    return launch_coop(reinterpret_cast<const void*>(linear_program_kernel), args, s);
}

cudaError_t launch_stack_plan(const LbPhase* phases, const LbJob* jobs, int n_phases,
                              WsHeader* hdr, const void* x, float* y, cudaStream_t s) {
    void* args[] = {&phases, &jobs, &n_phases, &hdr, &x, &y};
    return launch_coop(reinterpret_cast<const void*>(stack_program_kernel), args, s);
}

}  // namespace lb
