// Batch-1 / small-M decode path: a persistent phase program of lookup-table
// GEMVs over packed signs.
//
// The layer ("Samsung LittleBit: A 13B LLM Under 1 GB ...", "How it works",
// items 1-3) is two binary contractions with scales:
//   t = sign(V)^T (g o x),  y += h o (sign(U) (l o t))  for each branch.
// Each contraction is a GEMV whose matrix is a packed sign matrix P[rows][cols]
// and whose vector v is built on the fly (g o x, l o t, ...).
//
// Lookup tables.  For a slice of 512 columns the CTA tabulates, for every
// chunk of 8 consecutive columns, all 256 signed sums  T_c[e] = sum_q (bit q of
// e ? -v_q : +v_q).  One byte of a packed row then costs one shared-memory load
// and one add.  With chunk c = 4w + qb (word w = 4*gam + reg of the slice, byte
// qb of the word) the entry lives at byte
//     e*256 + (reg&1)*128 + 4*(8*gam + 4*(reg>>1) + qb)
// of the 64 KB table, i.e. in bank 8*gam + 4*(reg>>1) + qb.  Two tables are
// resident, at shared-window addresses 64 KB and 128 KB, so bits 16-17 of a
// lookup address pick the table and a CTA can run the rowblocks of two tiles
// (two slices or two matrices) as one stream.
//
// Lane mapping of the lookups.  Lane l = 4*rho + gam (rho = 0..7 picks one of 8
// rows of a step -- row 8*step + rho of the rowblock, so that a step's 8 rows
// are contiguous in the sliced layout -- and gam = 0..3 one of four 16-byte
// word groups of the row).  At
// step (r, jj) the lane reads register r of its group (with the two halves of
// the group swapped when rho >= 4) and byte (jj + rho) % 4 of that word, so
// the 32 lanes touch 32 chunks in 32 different banks.  A single PRMT merges the
// sign byte (the entry index) with a per-lane constant that also carries the
// table's address bits, so a lookup is PRMT + LDS + FADD.
//
// Sign words are loaded straight into registers with 128-bit non-allocating
// loads, kDepth rowblocks ahead of their use; shared memory only holds the
// tables, whose bandwidth the lookups need.
//
// Work split.  A job (one matrix) is cut into units of 32 rows x one slice.
// The host deals each CTA a contiguous, cost-balanced range of units; a CTA
// takes its range in batches of at most two tiles (a tile = the units of one
// slice of one job), stages the batch's vector slices, builds their tables
// and streams the rowblocks.  Partial row sums over a slice go to the fp32
// output with red.global.add, so the V-contraction result t stays in L2
// between the two phases.
//
// Phases are separated by a grid-wide wait (bounded spin); the kernel is
// launched cooperatively so that every CTA is resident.  Between announcing
// the end of a phase and waiting for the others, a CTA switches to the next
// phase's plan (fetched asynchronously one phase ahead) and loads the scales
// it will stage.  It keeps bulk loads out of the memory queues until the wait
// and the staging loads after it, which are on the critical path, have been
// issued.
#include <vector>

#include "lb_internal.cuh"

namespace lb {
namespace {

constexpr long long kSpinLimitCycles = 4000000000LL;   // ~2 s at 2 GHz
constexpr int kMaxTiles = kTables;                      // tiles of one batch

struct Smem {
    float* vec;       // kTables staged slices; element j at j + 4*(j/64)
    float* red;       // 32 floats of reduction scratch
    int* flag;        // one int
    LbPhase* phase;   // the current phase, copied from the plan
    int* range;       // this CTA's unit range in it (from the split table)
    LbStart* start;   // this CTA's first batch of it (when the plan has a start table)
    LbJob* jobs;      // its jobs (at most kMaxPhaseJobs), copied from the plan
};

// Two plan buffers (phase header, unit range, first batch, jobs): the current
// phase's and the next one's, which is copied in while the current phase runs.
constexpr int kOffPlan = 4 * kTables * kVecPad + 4 * 32 + 64;
constexpr int kPlanBufBytes = 128 + kMaxPhaseJobs * (int)sizeof(LbJob);
static_assert(kOffPlan % 64 == 0, "plan buffers must be 64-byte aligned");
static_assert(kOffPlan + 2 * kPlanBufBytes == kMiscBytes, "shared layout out of step");

__device__ __forceinline__ unsigned char* dyn_smem() {
    extern __shared__ __align__(64) unsigned char dsmem[];
    return dsmem;
}

__device__ __forceinline__ void use_plan_buf(Smem& s, int b) {
    unsigned char* base = dyn_smem() + kOffPlan + b * kPlanBufBytes;
    s.phase = reinterpret_cast<LbPhase*>(base);
    s.range = reinterpret_cast<int*>(base + sizeof(LbPhase));
    s.start = reinterpret_cast<LbStart*>(base + 64);
    s.jobs = reinterpret_cast<LbJob*>(base + 128);
}

__device__ __forceinline__ Smem smem_layout() {
    unsigned char* dsmem = dyn_smem();
    Smem s;
    s.vec = reinterpret_cast<float*>(dsmem);
    s.red = s.vec + kTables * kVecPad;
    s.flag = reinterpret_cast<int*>(s.red + 32);
    use_plan_buf(s, 0);
    return s;
}

__device__ __forceinline__ int vpad(int j) { return j + 4 * (j >> 6); }

// Index of this CTA's first unit of phase q in the split table, or -1 when
// the table has no room for the grid.
__device__ __forceinline__ int split_index(int q) {
    return blockIdx.x + 1 <= kMaxGrid ? q * (kMaxGrid + 1) + (int)blockIdx.x : -1;
}

// Copy phase q, its jobs and this CTA's unit range into plan buffer b, with
// every thread of the CTA (plan data never changes during a call).
__device__ void cache_plan(const LbPhase* phases, int q, const LbJob* jobs, const int* splits,
                           const LbStart* starts, int b) {
    Smem s;
    use_plan_buf(s, b);
    const LbPhase ph = phases[q];
    if (threadIdx.x == 0) *s.phase = ph;
    const int si = split_index(q);
    if (threadIdx.x < 2) s.range[threadIdx.x] = si >= 0 ? splits[si + threadIdx.x] : 0;
    if (starts != nullptr && ph.starts_g == (int)gridDim.x && threadIdx.x < 16)
        reinterpret_cast<int*>(s.start)[threadIdx.x] =
            reinterpret_cast<const int*>(starts + (size_t)q * kMaxGrid + blockIdx.x)[threadIdx.x];
    const int n_words = ph.n_jobs * (int)(sizeof(LbJob) / 4);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(jobs + ph.job_begin);
    uint32_t* dst = reinterpret_cast<uint32_t*>(s.jobs);
    for (int i = threadIdx.x; i < n_words; i += kDecodeThreads) dst[i] = src[i];
}

__device__ __forceinline__ void cp_async(void* dst, const void* src, int bytes) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    if (bytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(d), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" :: "r"(d), "l"(src) : "memory");
}

// The same copy done asynchronously by one warp (the plan must be in global
// memory); the job range comes from the previous phase's header.  Completed
// by plan_wait in the same warp before a CTA barrier.
__device__ void cache_plan_async(const LbPhase* phases, int q, int job_begin, int n_jobs,
                                 const LbJob* jobs, const int* splits, const LbStart* starts,
                                 int b) {
    Smem s;
    use_plan_buf(s, b);
    const int lane = threadIdx.x & 31;
    constexpr int kHdrPieces = (int)sizeof(LbPhase) / 16;
    constexpr int kJobPieces = (int)sizeof(LbJob) / 16;
    const int n = kHdrPieces + n_jobs * kJobPieces;
    for (int i = lane; i < n; i += 32) {
        if (i < kHdrPieces)
            cp_async(reinterpret_cast<uint4*>(s.phase) + i,
                     reinterpret_cast<const uint4*>(phases + q) + i, 16);
        else
            cp_async(reinterpret_cast<uint4*>(s.jobs) + (i - kHdrPieces),
                     reinterpret_cast<const uint4*>(jobs + job_begin) + (i - kHdrPieces), 16);
    }
    const int si = split_index(q);
    if (lane < 2 && si >= 0) cp_async(s.range + lane, splits + si + lane, 4);
    // the start record (used only if the phase header says the table was made for this grid)
    if (starts != nullptr && si >= 0 && lane >= 4 && lane < 8)
        cp_async(reinterpret_cast<uint4*>(s.start) + (lane - 4),
                 reinterpret_cast<const uint4*>(starts + (size_t)q * kMaxGrid + blockIdx.x) +
                     (lane - 4), 16);
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void plan_wait() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }

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

// Grid-wide wait, split in two so a CTA can set up the next phase between
// announcing that it is done (grid_arrive) and waiting for everyone else
// (grid_wait).  The arrival is a release-add: every write of the
// CTA made before it (ordered by the preceding __syncthreads) is visible to a
// CTA whose acquire-load sees the count.  The wait gives up after
// kSpinLimitCycles and records LB_ERR_TIMEOUT; it returns false if this CTA
// must stop.
__device__ __forceinline__ void grid_arrive(WsHeader* hdr) {
    __syncthreads();
    if (threadIdx.x == 0) red_release_add_u32(&hdr->barrier, 1u);
}

__device__ bool grid_wait(WsHeader* hdr, unsigned target, int* flag) {
    if (threadIdx.x == 0) {
        int ok = 1;
        const long long t0 = clock64();
        unsigned spins = 0;
        while (ld_acquire_u32(&hdr->barrier) < target) {
            __nanosleep(32);
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

// This CTA's unit range of the phase in sm: from the host's cost-balanced
// split table when it was made for this grid, else an even split.
__device__ __forceinline__ void unit_range(const Smem& sm, int& u, int& u_end) {
    const LbPhase& ph = *sm.phase;
    const int G = gridDim.x, cta = blockIdx.x;
    if (ph.split_g == G) {
        u = sm.range[0];
        u_end = sm.range[1];
    } else {
        u = (int)(((long long)ph.n_units * cta) / G);
        u_end = (int)(((long long)ph.n_units * (cta + 1)) / G);
    }
}

// Element j of a job's vector source, before its scale: a is the source
// value (the gate for VK_SILU_MUL, whose up value goes to b).
__device__ __forceinline__ void load_src(const LbJob& J, const void* src, int j, float& a,
                                         float& b) {
    switch (J.kind) {
        case VK_X_F16: a = __half2float(reinterpret_cast<const __half*>(src)[j]); break;
        case VK_X_BF16: a = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[j]); break;
        case VK_X_F32:
        case VK_T: a = __ldcg(reinterpret_cast<const float*>(src) + j); break;
        case VK_GQA:
            a = __ldcg(reinterpret_cast<const float*>(src) + (j / J.gqa_ghd) * J.gqa_hd +
                       (j % J.gqa_hd));
            break;
        default:  // VK_SILU_MUL
            a = __ldcg(reinterpret_cast<const float*>(src) + j);
            b = __ldcg(J.src2 + j);
            break;
    }
}

// Entries m and m + 16 (m = kM .. 15) of one chunk; entry offsets are
// immediates of the stores.
template <int kM>
__device__ __forceinline__ void store_entries(uint32_t base, const float (&p01)[4],
                                              const float (&p23)[4], float c0, float c1) {
    if constexpr (kM < 16) {
        const float l4 = p01[kM & 3] + p23[kM >> 2];
        sts_f32_off<kM * 256>(base, l4 + c0);
        sts_f32_off<(kM + 16) * 256>(base, l4 + c1);
        store_entries<kM + 1>(base, p01, p23, c0, c1);
    }
}

// Build the table of one staged slice at shared address taddr.  Thread t owns
// chunk c (slot i = t & 63: qb = i&3, wb1 = (i>>2)&1, gam = (i>>3)&3,
// reg&1 = i>>5) and the 32 entries e = 32*(t>>6) + m, m = 0..31; a warp's 32
// lanes write one entry of 32 chunks in 32 different banks.  Entry
// e = L(m) + H(t>>6) with L the signed sum of elements 0..4 and H that of 5..7.
__device__ __forceinline__ void build_table(const float* vec, uint32_t taddr) {
    const int t = threadIdx.x;
    const int i = t & 63, k = t >> 6;
    const int qb = i & 3, wb1 = (i >> 2) & 1, gam = (i >> 3) & 3, w0 = i >> 5;
    const int c = 4 * (4 * gam + 2 * wb1 + w0) + qb;
    const float4 lo = *reinterpret_cast<const float4*>(vec + vpad(8 * c));
    const float4 hi = *reinterpret_cast<const float4*>(vec + vpad(8 * c) + 4);
    // bit q of the entry index set <=> element q enters with sign -1
    const float p01[4] = {lo.x + lo.y, lo.y - lo.x, lo.x - lo.y, -lo.x - lo.y};
    const float p23[4] = {lo.z + lo.w, lo.w - lo.z, lo.z - lo.w, -lo.z - lo.w};
    const float hk = ((k & 1) ? -hi.y : hi.y) + ((k & 2) ? -hi.z : hi.z) + ((k & 4) ? -hi.w : hi.w);
    const float c0 = hk + hi.x, c1 = hk - hi.x;
    const uint32_t base = taddr + (uint32_t)k * (32u * 256u) + (uint32_t)w0 * 128u +
                          (uint32_t)(32 * gam + 16 * wb1 + 4 * qb);
    store_entries<0>(base, p01, p23, c0, c1);
}

// ---- tiles and batches ----------------------------------------------------
// What the lookup loop needs of one tile of the current batch.
struct TileRt {
    const uint32_t* P;       // first word of the slice in row 0
    const __half* h;         // row scales (second contraction) or nullptr
    float* out;
    int ldw, rows, wrem;     // row pitch, rows, words of the slice holding signs (<= 16)
    int rb0, nrb;
    uint32_t tb;             // table address bits (kTableAddr0 + t * 64 KB)
};

// This CTA's place in a phase and the batch about to run.  sc[k] is this
// thread's element of tile k's vector scale (g or l), which does not depend
// on earlier phases and is loaded before the grid-wide wait.
struct Cursor {
    int u, u_end, j;
    int nt, n_rb;
    LbTile t[kMaxTiles];
    TileRt rt[kMaxTiles];
    unsigned short sc[kMaxTiles];   // fp16 bits
};

// One rowblock (32 rows x 16 words of a slice) as this lane holds it: row
// step i covers row 8*i + rho, the lane's words 4*gam .. 4*gam+3, so with a
// 16-word pitch one load instruction of the warp reads 512 contiguous bytes;
// h is the row scale of the lane's output row (row 8*gam + rho).
struct RB {
    uint4 d[4];
    unsigned short h;   // fp16 bits, converted at use so the load does not stall the warp
};

__device__ __forceinline__ uint2 ld_stream_v2(const uint32_t* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

// Load rowblock rb of tile T into R.  Rows past the matrix and words past the
// signs are zero (their vector elements are zero, so any value would do; the
// point is to read neither outside the matrix nor a padded row's pitch).
__device__ __forceinline__ void load_rb(const TileRt& T, int rb, RB& R) {
    const int lane = threadIdx.x & 31;
    const int rho = lane >> 2, gam = lane & 3;
    const int w = 4 * gam;
    if (((T.wrem | T.ldw) & 3) == 0 && rb * kRowBlock + kRowBlock <= T.rows) {
        // the usual case: all 32 rows inside, whole 16-byte groups (lanes past
        // the slice's words hold zeros)
        const uint32_t* p = T.P + (size_t)(rb * kRowBlock + rho) * (size_t)T.ldw + w;
        const bool in = w < T.wrem;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            R.d[i] = in ? ld_stream_v4(p + (size_t)(8 * i) * T.ldw) : make_uint4(0u, 0u, 0u, 0u);
    } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = rb * kRowBlock + 8 * i + rho;
        uint4 d = make_uint4(0u, 0u, 0u, 0u);
        if (row < T.rows && w < T.wrem) {
            const uint32_t* p = T.P + (size_t)row * (size_t)T.ldw + w;
            if ((T.ldw & 3) == 0 && w + 4 <= T.wrem) {
                d = ld_stream_v4(p);
            } else if ((T.ldw & 1) == 0) {
                const uint2 a = ld_stream_v2(p);
                d.x = a.x; d.y = a.y;
                if (w + 2 < T.wrem) {
                    const uint2 b = ld_stream_v2(p + 2);
                    d.z = b.x; d.w = b.y;
                }
            } else {
                d.x = ld_stream_u32(p);
                if (w + 1 < T.wrem) d.y = ld_stream_u32(p + 1);
                if (w + 2 < T.wrem) d.z = ld_stream_u32(p + 2);
                if (w + 3 < T.wrem) d.w = ld_stream_u32(p + 3);
            }
        }
        R.d[i] = d;
    }
    }
    R.h = 0x3C00u;   // 1.0
    if (T.h != nullptr) {
        const int orow = rb * kRowBlock + 8 * gam + rho;
        R.h = orow < T.rows ? __ldg(reinterpret_cast<const unsigned short*>(T.h) + orow) : 0u;
    }
}

// Look up rowblock R against the table at address bits tb and add the row
// sums (times the row scale) to out.
// The 16 lookups of one 16-byte group (register R of the group, byte jj
// chosen per lane by the selector), written out by template recursion so every
// register and constant index is known at compile time.  Odd registers sit in
// the upper half of each entry row: offset 128.
template <int R, int JJ>
__device__ __forceinline__ void group_lookups(const uint32_t (&w4)[4], const uint32_t (&B)[2][4],
                                              const uint32_t (&S)[4], float& a0, float& a1) {
    const uint32_t addr = prmt(w4[R], B[R >> 1][JJ], S[JJ]);
    const float v = lds_f32_off<(R & 1) * 128>(addr);
    if (JJ & 1) a1 += v; else a0 += v;
    if constexpr (JJ < 3) group_lookups<R, JJ + 1>(w4, B, S, a0, a1);
    else if constexpr (R < 3) group_lookups<R + 1, 0>(w4, B, S, a0, a1);
}

// Slice sums of the four row steps of a rowblock (lanes with rho >= 4 read the
// halves of their group swapped).
template <int I>
__device__ __forceinline__ void step_sums(const RB& Rb, bool swap, const uint32_t (&B)[2][4],
                                          const uint32_t (&S)[4], float (&acc)[4]) {
    uint32_t w4[4];
    w4[0] = swap ? Rb.d[I].z : Rb.d[I].x;
    w4[1] = swap ? Rb.d[I].w : Rb.d[I].y;
    w4[2] = swap ? Rb.d[I].x : Rb.d[I].z;
    w4[3] = swap ? Rb.d[I].y : Rb.d[I].w;
    float a0 = 0.0f, a1 = 0.0f;
    group_lookups<0, 0>(w4, B, S, a0, a1);
    acc[I] = a0 + a1;
    if constexpr (I < 3) step_sums<I + 1>(Rb, swap, B, S, acc);
}

__device__ __forceinline__ void consume_rb(const RB& R, const TileRt& T, int rb,
                                           const uint32_t (&Bc)[2][4], const uint32_t (&S)[4]) {
    const int lane = threadIdx.x & 31;
    const int rho = lane >> 2, gam = lane & 3;
    const bool swap = rho >= 4;
    uint32_t B[2][4];
#pragma unroll
    for (int rh = 0; rh < 2; ++rh)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) B[rh][jj] = Bc[rh][jj] + T.tb;
    float acc[4];
    step_sums<0>(R, swap, B, S, acc);
    // Transpose-reduce over the 4 lanes of a row group (gam = lane bits 0-1):
    // afterwards lane gam of group rho holds the slice sum of row step gam,
    // i.e. of row 8*gam + rho of the rowblock.
    const bool up2 = (gam & 2) != 0, up1 = (gam & 1) != 0;
    float n2[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float send = up2 ? acc[k] : acc[k + 2];
        const float keep = up2 ? acc[k + 2] : acc[k];
        n2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const float send1 = up1 ? n2[0] : n2[1];
    const float keep1 = up1 ? n2[1] : n2[0];
    const float tot = (keep1 + __shfl_xor_sync(0xffffffffu, send1, 1)) *
                      __half2float(__ushort_as_half(R.h));
    // The 32 lanes hold the rowblock's 32 rows, so one reduction per lane is
    // a single coalesced 128-byte reduction for the warp.
    const int row = rb * kRowBlock + 8 * gam + rho;       // the row this lane holds
    if (row < T.rows) red_add_f32(T.out + row, tot);
}

// Rowblock n of a batch (n < n_rb): its tile (selected field by field, so
// the cursor stays in registers) and its rowblock index.
__device__ __forceinline__ TileRt batch_tile(const Cursor& c, int n, int& rb) {
    const bool k = c.nt > 1 && n >= c.rt[0].nrb;
    TileRt T;
    T.P = k ? c.rt[1].P : c.rt[0].P;
    T.h = k ? c.rt[1].h : c.rt[0].h;
    T.out = k ? c.rt[1].out : c.rt[0].out;
    T.ldw = k ? c.rt[1].ldw : c.rt[0].ldw;
    T.rows = k ? c.rt[1].rows : c.rt[0].rows;
    T.wrem = k ? c.rt[1].wrem : c.rt[0].wrem;
    T.rb0 = k ? c.rt[1].rb0 : c.rt[0].rb0;
    T.nrb = k ? c.rt[1].nrb : c.rt[0].nrb;
    T.tb = k ? c.rt[1].tb : c.rt[0].tb;
    rb = T.rb0 + (k ? n - c.rt[0].nrb : n);
    return T;
}

// Issue this warp's first kDepth rowblocks of the batch into buf.  Register
// loads can stall a warp at issue once the SM's outstanding misses fill up,
// so they are issued only after the batch's tables are built.
__device__ __forceinline__ void batch_loads(const Cursor& c, RB (&buf)[kDepth], int d0 = 0) {
    const int wp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
        if (d < d0) continue;
        const int n = wp + d * kDecodeWarps;
        if (n < c.n_rb) {
            int rb;
            const TileRt T = batch_tile(c, n, rb);
            load_rb(T, rb, buf[d]);
        }
    }
}

// Stream this warp's rowblocks of the batch (n = wp, wp + 16, ...) through
// the register ring buf, kDepth ahead of their use; the first kDepth were
// issued by batch_loads.
__device__ __forceinline__ void batch_lookups(const Cursor& c, RB (&buf)[kDepth],
                                              const uint32_t (&Bc)[2][4], const uint32_t (&S)[4]) {
    const int wp = threadIdx.x >> 5;
    for (int n0 = wp; n0 < c.n_rb; n0 += kDepth * kDecodeWarps) {
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            const int n = n0 + d * kDecodeWarps;
            if (n < c.n_rb) {
                int rb;
                const TileRt T = batch_tile(c, n, rb);
                consume_rb(buf[d], T, rb, Bc, S);
                const int nn = n + kDepth * kDecodeWarps;
                if (nn < c.n_rb) {
                    int rb2;
                    const TileRt T2 = batch_tile(c, nn, rb2);
                    load_rb(T2, rb2, buf[d]);
                }
            }
        }
    }
}

// Tile k of the batch (c.t[k] set): what the lookup loop needs of it, and
// this thread's element of its vector scale.  Reads only plan data and weights.
__device__ __forceinline__ void tile_setup(const Smem& sm, const CallArgs& args, Cursor& c, int k) {
    const LbTile& t = c.t[k];
    const LbJob& J = sm.jobs[t.job];
    TileRt& T = c.rt[k];
    const int nw = (J.cols + 31) / 32;
    if (J.sliced) {   // the slice is a contiguous block of rows
        T.P = J.P + (size_t)kSliceWords * (size_t)J.rows * (size_t)t.slice;
        T.ldw = (int)sliced_pitch(nw, t.slice);
    } else {
        T.P = J.P + (size_t)t.slice * kSliceWords;
        T.ldw = J.ldw;
    }
    T.h = J.oscale;
    T.out = resolve(J.out, args);
    T.rows = J.rows;
    // words of the slice a lane may read: in the sliced layout the whole pitch
    // (padding words hold bits of columns whose vector elements are zero)
    T.wrem = J.sliced ? T.ldw : min(kSliceWords, nw - t.slice * kSliceWords);
    T.rb0 = t.rb0;
    T.nrb = t.nrb;
    T.tb = kTableAddr0 + (uint32_t)k * (uint32_t)kLutBytes;
    const int col = t.slice * kSliceElems + (int)threadIdx.x;
    if (col < J.cols) c.sc[k] = __ldg(reinterpret_cast<const unsigned short*>(J.vscale) + col);
}

// Collect the next batch at c.u and load this thread's scale elements.
__device__ __forceinline__ void batch_begin(const Smem& sm, const CallArgs& args, Cursor& c) {
    c.nt = 0;
    c.n_rb = 0;
#pragma unroll
    for (int k = 0; k < kMaxTiles; ++k) {
        c.sc[k] = 0u;
        if (c.u + c.n_rb < c.u_end) {
            c.t[k] = next_tile(sm.jobs, sm.phase->n_jobs, c.j, c.u + c.n_rb, c.u_end);
            c.nt = k + 1;
            c.n_rb += c.t[k].nrb;
            tile_setup(sm, args, c, k);
        }
    }
}

// Stage the batch's vector slices into shared memory (zero past cols): all
// source loads are issued before any is used, so the batch costs one round
// trip to L2.  The owner of a slice (the CTA holding its first rowblock) also
// seeds the residual and adds the slice's sum of squares for RMSNorm; only
// the first job of a phase carries acc_sumsq, so there is one sum per batch.
// Ends with a CTA barrier.
__device__ __forceinline__ void stage_batch(const Smem& sm, const CallArgs& args, const Cursor& c) {
    static_assert(kSliceElems == kDecodeThreads, "one slice element per thread");
    const int e = threadIdx.x;
    float a[kMaxTiles], a2[kMaxTiles], nrm[kMaxTiles];
#pragma unroll
    for (int k = 0; k < kMaxTiles; ++k) {
        a[k] = 0.0f;
        a2[k] = 0.0f;
        nrm[k] = -1.0f;
        if (k < c.nt) {
            const LbJob& J = sm.jobs[c.t[k].job];
            const int col = c.t[k].slice * kSliceElems + e;
            if (col < J.cols) load_src(J, resolve(J.src, args), col, a[k], a2[k]);
            if (J.kind == VK_T && J.norm_sumsq != nullptr) nrm[k] = __ldcg(J.norm_sumsq);
        }
    }
    float sq = 0.0f;
    float* acc = nullptr;
#pragma unroll
    for (int k = 0; k < kMaxTiles; ++k) {
        if (k >= c.nt) break;
        const LbJob& J = sm.jobs[c.t[k].job];
        const int col = c.t[k].slice * kSliceElems + e;
        const bool owner = c.t[k].rb0 == 0;
        float v = 0.0f;
        if (col < J.cols) {
            const float raw = J.kind == VK_SILU_MUL ? silu(a[k]) * a2[k] : a[k];
            const float rs = nrm[k] >= 0.0f ? rsqrtf(nrm[k] / (float)J.norm_n + kRmsEps) : 1.0f;
            v = __half2float(__ushort_as_half(c.sc[k])) * (raw * rs);
            if (owner) {
                if (J.acc_sumsq != nullptr) sq += raw * raw;
                float* ri = resolve(J.resid_init, args);
                if (ri != nullptr) ri[col] = raw;
            }
        }
        if (owner && J.acc_sumsq != nullptr) acc = J.acc_sumsq;
        sm.vec[k * kVecPad + vpad(e)] = v;
    }
    if (acc != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if ((threadIdx.x & 31) == 0) sm.red[threadIdx.x >> 5] = sq;
    }
    __syncthreads();
    if (acc != nullptr && threadIdx.x == 0) {
        float tot = 0.0f;
        for (int w = 0; w < kDecodeWarps; ++w) tot += sm.red[w];
        atomicAdd(acc, tot);
    }
}

// The part of a phase that does not depend on earlier phases: this CTA's
// unit range and its first batch.  sm.phase / sm.jobs must hold the phase.
// The first batch comes from the plan's start table when it was made for this
// grid (the same tiles batch_begin would find), else from batch_begin.
__device__ __forceinline__ void phase_begin(const Smem& sm, const CallArgs& args, Cursor& c) {
    if (sm.phase->starts_g == (int)gridDim.x) {
        const LbStart& S = *sm.start;
        c.u = S.u;
        c.u_end = S.u_end;
        c.j = S.j;
        c.nt = S.nt;
        c.n_rb = S.n_rb;
#pragma unroll
        for (int k = 0; k < kMaxTiles; ++k) {
            c.sc[k] = 0u;
            if (k < c.nt) {
                c.t[k] = S.t[k];
                tile_setup(sm, args, c, k);
            }
        }
        return;
    }
    unit_range(sm, c.u, c.u_end);
    c.j = 0;
    c.nt = 0;
    c.n_rb = 0;
    if (c.u < c.u_end) batch_begin(sm, args, c);
}

// Request this warp's first rowblock of the current batch into R.
__device__ __forceinline__ void first_load(const Cursor& c, RB& R) {
    const int n = (int)(threadIdx.x >> 5);
    if (n < c.n_rb) {
        int rb;
        const TileRt T = batch_tile(c, n, rb);
        load_rb(T, rb, R);
    }
}

// The rest of the phase, after the grid-wide wait.  loaded: this warp's first
// rowblock of the first batch is already requested (during the wait).
__device__ __forceinline__ void run_phase(const Smem& sm, const CallArgs& args, Cursor& c,
                                          RB (&buf)[kDepth],
                                          const uint32_t (&Bc)[2][4], const uint32_t (&S)[4],
                                          bool loaded) {
    const int G = gridDim.x, cta = blockIdx.x;
    float* zp = resolve(sm.phase->zero_ptr, args);
    const int zn = sm.phase->zero_n;
    if (zp != nullptr) {
        for (int i = cta * kDecodeThreads + threadIdx.x; i < zn; i += G * kDecodeThreads)
            zp[i] = 0.0f;
    }
    bool skip = loaded;
    while (c.u < c.u_end) {
        // each warp's first rowblock is requested before the vector is staged
        // (32 KB per CTA), its second after the tables are built
        {
            const int n = (int)(threadIdx.x >> 5);
            const bool sk = skip;
            skip = false;
            if (!sk && n < c.n_rb) {
                int rb;
                const TileRt T = batch_tile(c, n, rb);
                load_rb(T, rb, buf[0]);
            }
        }
        stage_batch(sm, args, c);
        for (int k = 0; k < c.nt; ++k)
            build_table(sm.vec + k * kVecPad, kTableAddr0 + (uint32_t)k * (uint32_t)kLutBytes);
        batch_loads(c, buf, 1);
        __syncthreads();
        batch_lookups(c, buf, Bc, S);
        c.u += c.n_rb;
        if (c.u < c.u_end) batch_begin(sm, args, c);
        __syncthreads();
    }
}

template <bool kAsyncPlan>
__device__ __forceinline__ void run_program(const LbPhase* phases, int n_phases, const LbJob* jobs,
                                            const int* splits, const LbStart* starts,
                                            WsHeader* hdr, const CallArgs& args) {
    Smem sm = smem_layout();
    const unsigned G = gridDim.x;
    if (*reinterpret_cast<volatile int*>(&hdr->error) != 0) return;   // sticky after a timeout
    // the tables must sit above the plan cache at their fixed addresses
    if ((uint32_t)__cvta_generic_to_shared(dyn_smem()) + (uint32_t)kMiscBytes > kTableAddr0) {
        if (threadIdx.x == 0) atomicExch(&hdr->error, (int)LB_ERR_UNSUPPORTED);
        return;
    }
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int rho = lane >> 2, gam = lane & 3;
    const uint32_t swap = (uint32_t)(rho >> 2);
    uint32_t Bc[2][4], S[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const uint32_t qbj = (uint32_t)((jj + rho) & 3);
        S[jj] = 0x7604u | (qbj << 4);                    // [B.b0, word.byte qbj, B.b2, B.b3]
#pragma unroll
        for (int rh = 0; rh < 2; ++rh)
            Bc[rh][jj] = (8u * (uint32_t)gam + 4u * ((uint32_t)rh ^ swap) + qbj) * 4u;
    }
    // The first two phases' plans are copied in by the whole CTA; each later
    // one is fetched asynchronously by the last warp one phase ahead.
    cache_plan(phases, 0, jobs, splits, starts, 0);
    if (n_phases > 1) cache_plan(phases, 1, jobs, splits, starts, 1);
    __syncthreads();
    Cursor cur;
    RB buf[kDepth];
    phase_begin(sm, args, cur);
    bool loaded = false;
    for (int p = 0; p < n_phases; ++p) {
        run_phase(sm, args, cur, buf, Bc, S, loaded);
        if (p + 1 < n_phases) {
            // Announce completion, then use the wait: switch to the next
            // phase's plan, load the scales of its first batch, fetch the
            // plan of the phase after it into the buffer this phase used and
            // request the first rowblocks.
            grid_arrive(hdr);
            if (wp == kDecodeWarps - 1) plan_wait();
            __syncthreads();
            const int nb = (p + 1) & 1;
            use_plan_buf(sm, nb);
            phase_begin(sm, args, cur);
            if (kAsyncPlan && wp == kDecodeWarps - 1 && p + 2 < n_phases)
                cache_plan_async(phases, p + 2, sm.phase->next_job_begin, sm.phase->next_n_jobs,
                                 jobs, splits, starts, nb ^ 1);
            if (!kAsyncPlan && p + 2 < n_phases) {   // (not reached: such plans have two phases)
                __syncthreads();
                cache_plan(phases, p + 2, jobs, splits, starts, nb ^ 1);
            }
            // The sign words do not depend on earlier phases, so every warp but
            // the poller's requests its first rowblock now and the HBM latency
            // overlaps the wait; the poller's warp keeps no loads in flight
            // ahead of its polls (measured: loads there delay the acquire).
            loaded = wp != 0;
            if (loaded && cur.u < cur.u_end) first_load(cur, buf[0]);
            if (!grid_wait(hdr, (unsigned)(p + 1) * G, sm.flag)) {
                if (wp == kDecodeWarps - 1) plan_wait();
                return;
            }
        }
    }
    // The last CTA out resets the arrival counter for the next call.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&hdr->exit_count, 1u);
        if (prev == G - 1) {
            hdr->barrier = 0u;
            hdr->exit_count = 0u;
            __threadfence();
        }
    }
}

__global__ void __launch_bounds__(kDecodeThreads, kCtasPerSm)
linear_program_kernel(const __grid_constant__ LinearPlan plan, int n_phases, WsHeader* hdr) {
    const CallArgs args = {nullptr, nullptr};
    run_program<false>(plan.phases, n_phases, plan.jobs, plan.split, nullptr, hdr, args);
}

__global__ void __launch_bounds__(kDecodeThreads, kCtasPerSm)
stack_program_kernel(const LbPhase* __restrict__ phases, const LbJob* __restrict__ jobs,
                     const int* __restrict__ splits, const LbStart* __restrict__ starts,
                     int n_phases, WsHeader* hdr, const void* x, float* y) {
    const CallArgs args = {x, y};
    run_program<true>(phases, n_phases, jobs, splits, starts, hdr, args);
}

cudaError_t launch_coop(const void* fn, void** args, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(device_sm_count() * kCtasPerSm));
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

int decode_grid() { return device_sm_count() * kCtasPerSm; }

// Contiguous unit ranges for G CTAs with the smallest largest cost.  A CTA
// takes its tiles in batches of up to kTables; a batch costs kBatchCost
// (staging its vectors) plus kTileCost per tile (a table build) plus its
// rowblocks (see rb_cost), all in 1/16 of a round of 16 rowblocks.
// Units run job by job, slice-major inside a job, so a phase is a list of
// tiles of n_rowblocks units each; a greedy fill is optimal for a given bound,
// which a bisection minimises.
namespace {
template <class F>
void for_each_tile(const LbJob* jobs, int n_jobs, F f) {
    for (int j = 0; j < n_jobs; ++j)
        for (int g0 = 0; g0 < jobs[j].n_rowblocks; g0 += jobs[j].rg)
            for (int s = 0; s < jobs[j].n_slices; ++s)
                f(std::min(jobs[j].rg, jobs[j].n_rowblocks - g0));
}
// A batch's rowblocks cost one each in the rounds where all 16 warps have one
// (the lookups are bound by the SM's shared-memory pipe); a last, partial
// round costs in proportion to its rowblocks, but at least kPartialRound,
// since each of its warps still waits out a rowblock's latency.
constexpr long long kPartialRound = 8;
long long rb_cost(long long k) {
    const long long full = k / kDecodeWarps * kDecodeWarps, rest = k - full;
    return full + (rest > 0 ? std::max(rest, kPartialRound) : 0);
}
// The most rowblocks whose cost fits in `avail`.
long long rb_room(long long avail) {
    if (avail <= 0) return 0;
    const long long full = avail / kDecodeWarps * kDecodeWarps, rest = avail - full;
    return full + (rest >= kPartialRound ? rest : 0);
}
struct Fill {
    long long closed;   // cost of the CTA's finished batches
    int tiles;          // tiles in its open batch
    long long rb;       // rowblocks in its open batch
};
// The CTA's state and cost once `take` rowblocks of a new tile join it.
long long open_cost(const Fill& g) { return kBatchCost + g.tiles * kTileCost; }
long long join(const Fill& f, long long take, Fill& g) {
    g = f;
    if (g.tiles == kTables) {
        g.closed += open_cost(g) + rb_cost(g.rb);
        g.tiles = 0;
        g.rb = 0;
    }
    g.tiles += 1;
    g.rb += take;
    return g.closed + open_cost(g) + rb_cost(g.rb);
}
// CTAs a greedy fill under cost bound T needs; boundaries go to `out` if set.
int greedy_fill(const LbJob* jobs, int n_jobs, long long T, int* out) {
    int used = 1, u = 0;
    Fill f = {0, 0, 0};
    for_each_tile(jobs, n_jobs, [&](int n) {
        while (n > 0) {
            Fill g;
            if (join(f, 1, g) > T) {
                if (out) out[used] = u;
                ++used;
                f = Fill{0, 0, 0};
            }
            join(f, 0, g);
            const long long room = rb_room(T - g.closed - open_cost(g)) - g.rb;
            const int take = (int)std::max<long long>(1, std::min<long long>(n, room));
            join(f, take, f);
            n -= take;
            u += take;
        }
    });
    return used;
}

// A job gets about alpha times as many row groups as the CTAs its share of
// the phase's units would occupy, divided by its slices, so that a CTA's range
// is usually one tile and the n_slices CTAs of a group read the same rows.
void row_groups(LbJob* jobs, int n_jobs, int n_units, int G, double alpha) {
    for (int j = 0; j < n_jobs; ++j) {
        LbJob& J = jobs[j];
        const double ctas = (double)G * (double)(J.n_slices * J.n_rowblocks) / (double)n_units;
        const int groups = std::max(1, (int)(alpha * ctas / J.n_slices + 0.5));
        J.rg = (J.n_rowblocks + groups - 1) / groups;
    }
}
}  // namespace

long long balanced_split(const LbJob* jobs, int n_jobs, int n_units, int G, int* out);

// Row groups of a phase: with `search`, the scaling of the CTA-proportional
// count whose cost-balanced split has the smallest largest cost (rounding the
// count to the nearest integer can leave most CTAs with a range across two
// tiles, and so two table builds, where one tile per CTA fits in the same
// time); stack plans, made once, search; single-linear calls plan on every
// call and take the unscaled count.
void plan_row_groups(LbJob* jobs, int n_jobs, int n_units, int G, bool search) {
    if (!search) {
        row_groups(jobs, n_jobs, n_units, G, 1.0);
        return;
    }
    static const double kAlphas[] = {1.0, 0.9, 0.8, 0.7, 0.6, 0.5, 1.15, 1.3};
    std::vector<int> split(G + 1);
    double best_alpha = 1.0;
    long long best = -1;
    for (double a : kAlphas) {
        row_groups(jobs, n_jobs, n_units, G, a);
        const long long c = balanced_split(jobs, n_jobs, n_units, G, split.data());
        if (best < 0 || c < best) { best = c; best_alpha = a; }
    }
    row_groups(jobs, n_jobs, n_units, G, best_alpha);
}

long long balanced_split(const LbJob* jobs, int n_jobs, int n_units, int G, int* out) {
    long long lo = kBatchCost + kTileCost + kDecodeWarps, hi = lo;
    {
        Fill f = {0, 0, 0};
        for_each_tile(jobs, n_jobs, [&](int n) { hi = join(f, n, f); });
        hi = std::max(hi, lo);
    }
    while (lo < hi) {   // smallest bound a fill of at most G CTAs meets
        const long long mid = (lo + hi) / 2;
        if (greedy_fill(jobs, n_jobs, mid, nullptr) <= G) hi = mid;
        else lo = mid + 1;
    }
    const int used = greedy_fill(jobs, n_jobs, lo, out);
    out[0] = 0;
    for (int c = used; c <= G; ++c) out[c] = n_units;
    return lo;
}

void plan_starts(LbPhase* phases, int n_phases, const LbJob* jobs, const int* split, int G,
                 LbStart* out) {
    for (int q = 0; q < n_phases; ++q) {
        LbPhase& ph = phases[q];
        ph.starts_g = -1;
        if (G > kMaxGrid || ph.split_g != G) continue;
        const LbJob* pj = jobs + ph.job_begin;
        const int* sp = split + ph.split_off;
        for (int c = 0; c < G; ++c) {
            LbStart S = {};
            S.u = sp[c];
            S.u_end = sp[c + 1];
            // the tiles of the first batch, as the kernel's batch_begin takes them
            for (int k = 0; k < kTables; ++k) {
                if (S.u + S.n_rb >= S.u_end) break;
                S.t[k] = next_tile(pj, ph.n_jobs, S.j, S.u + S.n_rb, S.u_end);
                S.nt = k + 1;
                S.n_rb += S.t[k].nrb;
            }
            out[(size_t)q * kMaxGrid + c] = S;
        }
        ph.starts_g = G;
    }
}

cudaError_t decode_configure() {
    for (const void* fn : {reinterpret_cast<const void*>(linear_program_kernel),
                           reinterpret_cast<const void*>(stack_program_kernel)}) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kDecodeSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kDecodeThreads, kDecodeSmem);
        if (e != cudaSuccess) return e;
        if (nb < kCtasPerSm) return cudaErrorCooperativeLaunchTooLarge;
    }
    return cudaSuccess;
}

cudaError_t launch_linear_plan(const LinearPlan& plan, WsHeader* hdr, int n_phases,
                               cudaStream_t s) {
    void* args[] = {const_cast<LinearPlan*>(&plan), &n_phases, &hdr};
    return launch_coop(reinterpret_cast<const void*>(linear_program_kernel), args, s);
}

cudaError_t launch_stack_plan(const LbPhase* phases, const LbJob* jobs, const int* splits,
                              const LbStart* starts, int n_phases, WsHeader* hdr, const void* x,
                              float* y, cudaStream_t s) {
    void* args[] = {&phases, &jobs, &splits, &starts, &n_phases, &hdr, &x, &y};
    return launch_coop(reinterpret_cast<const void*>(stack_program_kernel), args, s);
}

}  // namespace lb
