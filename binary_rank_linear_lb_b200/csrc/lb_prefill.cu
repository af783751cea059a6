// Large-M (prefill) path: the two contractions of the layer as tcgen05 GEMMs.
//
// The layer ("Samsung LittleBit: A 13B LLM Under 1 GB ...", "How it works",
// items 1-3), for a block of M rows of x:
//   stage 1:  T[m, b*r + k]  = l_b[k] * sum_j x[m, j] * (g_b[j] * sign(V_b[j, k]))
//   stage 2:  y[m, i]        = sum_b sum_k T[m, b*r + k] * (h_b[i] * sign(U_b[i, k]))
// Both are dense contractions, so they run on the 5th-generation tensor cores
// (tcgen05.mma kind::f16: fp16 operands, fp32 accumulation in TMEM).
//
// Operands.  A (x, then T) is fp16, row-major, loaded by TMA with the 128-byte
// swizzle.  B is never stored in HBM: producer warps expand the packed sign
// bits in shared memory into fp16 tiles, each element a scale with its sign bit
// flipped (g_b[j] for stage 1, h_b[i] for stage 2), which is exact in fp16.
// Rows of x are brought into fp16 range by a power of two a_m; stage 1 writes
// T multiplied by another power of two c_m chosen from the bound
// |T[m, .]| <= max_k |l_k| * sum_j |g_j x[m, j]|, so T never overflows fp16 and
// keeps fp16's relative precision.  Stage 2 divides c_m out again.
//
// Kernel shape: one CTA per SM, persistent over output tiles of MT x 128 rows
// by 256 columns (MT = 1 or 2 M sub-tiles share each expanded B tile, so with
// MT = 2 a B tile is expanded once per 256 output rows).  Warp-specialised:
// warps 0-7 drain the TMEM accumulators, warp 8 issues the TMA loads of A,
// warp 9 allocates TMEM and issues the MMAs (one thread), warps 10-17 expand
// B.  TMEM holds 512 fp32 columns: two 256-column accumulators, used as a
// double buffer (MT = 1) or as the two M sub-tiles of one tile (MT = 2).
// Pipeline stages of (A MT x 16 KB + B 32 KB) in shared memory, synchronised
// with mbarriers.  Every wait is bounded: on time-out the kernel records
// LB_ERR_TIMEOUT, lets every role finish, frees its TMEM and returns.
#include <cuda.h>

#include <algorithm>
#include <cstdlib>

#include "lb_internal.cuh"

namespace lb {
namespace {

constexpr int kTileM = 128;                       // rows of one M sub-tile (one MMA)
constexpr int kTileN = 256;
constexpr int kBlockK = 64;                       // fp16 elements per stage (128 bytes)
constexpr int kABytes = kTileM * kBlockK * 2;     // 16 KB per M sub-tile
constexpr int kBBytes = kTileN * kBlockK * 2;     // 32 KB
constexpr int kGBytes = kBlockK * 2;              // g slice of the K block (stage 1)
constexpr int kPrefillThreads = 576;              // 18 warps
constexpr int kEpiWarps = 8;                      // warps 0..7 drain TMEM (lane quarter = warp & 3)
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kExpandWarp0 = 10;                  // warps 10..17 expand B, one row per thread
constexpr int kExpandWarps = 8;
constexpr int kTmemCols = 512;                    // two 256-column accumulators
constexpr long long kWaitLimit = 4000000000LL;    // cycles (~2 s)
constexpr uint32_t kSuspendNs = 20000;            // longest hardware suspension per try_wait
constexpr int kMaxStages = 4;
constexpr int kPartFloats = 8 * 32 * 32;          // one epilogue warp's share of a tile (8 chunks)
constexpr int kSplit2Max = 4;                      // K parts of a stage-2 tile at most
constexpr int kSplitMaxParts = 160;               // stage-1 tile parts the split buffer holds
constexpr int kSplitMax = 4;                      // K parts of one stage-1 tile (the last one folds the others)

constexpr int kEpiBytes = 32 * 128;                // per-warp epilogue staging: 32 rows x 128 bytes
constexpr int kBitsAhead = 4;                     // K blocks of sign bits held in registers ahead

// Shared memory of one CTA, from the 1024-aligned base: the pipeline stages
// (A sub-tiles then the B tile, each 1024-aligned), the epilogue staging
// buffers, the g slices of the stages (stage 1), the control block.
template <int MT>
struct Shape {
    static constexpr int kStageBytes = MT * kABytes + kBBytes;
    static constexpr int kStages = MT == 1 ? 4 : 3;
    static constexpr int kOffEpi = kStages * kStageBytes;
    static constexpr int kOffG = kOffEpi + kEpiWarps * kEpiBytes;
    static constexpr int kOffCtl = kOffG + kStages * kGBytes;
    static constexpr int kSmem = kOffCtl + 256 /*barriers*/ + 1024 /*align*/;
    static constexpr int kBufs = 2 / MT;                                // accumulator buffers
};
static_assert(Shape<1>::kSmem <= 232448 && Shape<2>::kSmem <= 232448, "shared memory");

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
struct Ctl {                 // shared control block
    uint64_t full_a[kMaxStages], full_b[kMaxStages], empty[kMaxStages];
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort;
};

// Bounded wait on an mbarrier phase; on time-out raises the CTA abort flag
// and the workspace error.  Returns false if the caller must stop.
// try_wait that may suspend the thread in hardware for up to `ns` nanoseconds;
// it resumes when the phase completes, so a waiting warp takes no issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(ns) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool wait_bar(Ctl* c, uint64_t* bar, uint32_t parity, int* err) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(a, parity, kSuspendNs)) return true;
        if (*reinterpret_cast<volatile int*>(&c->abort)) return false;
        if (clock64() - t0 > kWaitLimit) {
            atomicExch(&c->abort, 1);
            atomicExch(err, (int)LB_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes (stride byte offset 1024), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, fp16 A and B, both
// K-major, M = 128, N = 256.
constexpr uint32_t kInstrDesc = (1u << 4) | ((uint32_t)(kTileN >> 3) << 17) |
                                ((uint32_t)(kTileM >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem_d), "l"(a), "l"(b), "r"(kInstrDesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Tensor store of the box at (x, y) from shared memory (bulk async-group of the
// issuing thread); the shared source must be made visible to the async proxy
// first (fence.proxy.async) and stay untouched until wait_group.read.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 :: "l"(map), "r"(src), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {      // sources of earlier stores reusable
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {       // earlier stores complete
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 lanes x 32 columns of fp32 from TMEM (one row per lane).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 columns of fp32 from / to TMEM (one row per lane).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
           "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
           "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
           "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
           "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
           "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
}

}  // namespace

// ------------------------------------------------------------------ problem
// One GEMM of the prefill path.  N is cut into segments (stage 1: one per
// branch, rows of Vp_b; stage 2: one, the output features) and K into segments
// (stage 1: one, the input features; stage 2: one per branch, rows of T).
struct PrefillGemm {
    int M, n_seg_rows, n_nseg, n_kseg, k_seg_len;   // N = n_nseg * n_seg_rows, K = n_kseg * k_seg_len
    int stage;                                       // 1 or 2
    const uint32_t* P[2];                            // packed signs per branch
    int ldw[2];                                      // words per packed row, per branch (rows layout)
    int sliced[2];                                   // branch packed in LB_LAYOUT_SLICES
    int nw;                                          // words holding the K = k_seg_len signs of a row
    const __half* bscale[2];                         // stage 1: g_b (per k); stage 2: h_b (per n)
    const __half* lscale[2];                         // stage 1: l_b (per output column)
    const float* row_sa;                             // [M] 2^a_m (stage 1 divides it out)
    const float* row_sc;                             // [M] 2^c_m
    __half* T;                                       // stage 1 output [M][n_nseg * n_seg_rows]
    int n_cat;                                       // stage 1 with one sub-tile: the N tiles run
                                                     // over the segments back to back (row R of
                                                     // segment R / n_seg_rows), so two branches of
                                                     // low rank share a tile instead of half-filling
                                                     // one each
    float* y;                                        // stage 2 output [M][n_seg_rows]
    int* err;
};

// Both GEMMs of a call as one persistent launch: the tile list is stage 1's
// tiles, then stage 2's, dealt round-robin to the CTAs.  A stage-2 tile reads
// the rows of T of its M block, so before loading them its TMA thread waits
// until every epilogue warp of the block's stage-1 tiles has published its
// rows (done[mb] reaching done_target).  Every CTA reaches all its stage-1
// tiles before any stage-2 tile, and the other roles never wait for the TMA
// thread, so a stage-1 tile is never held up behind a waiting stage-2 tile.
// With few stage-1 tiles (small M, low rank) stage 1 is split along K into
// `split` parts, adjacent in the tile list.  For each of its chunks an
// epilogue warp writes its fp32 partial sums to `partial` and takes a ticket
// for its region of the tile; the warp that draws the last ticket adds the
// other parts' partials to its own accumulator and finishes the region into T.
// With few stage-2 tiles, stage 2 is split along K too (`split2` parts); its
// parts add their sums into y, which the host zeroes first.
struct PrefillPlan {
    PrefillGemm g[2];
    int n_tiles[2];      // tiles of each GEMM (stage 1: tiles x split)
    int* done;           // [M blocks] stage-1 epilogue warps finished, zeroed per call
    int done_target;     // kEpiWarps * (stage-1 tiles of one M block)
    int split;           // K parts of a stage-1 tile (1: no split)
    float* partial;      // [tile][part][epilogue warp][kPartFloats] fp32 partial sums
    int* tickets;        // [tile][epilogue warp], zeroed per call
    int split2;          // K parts of a stage-2 tile (1: no split; else y, zeroed first,
                         // takes each part's sums by reduction)
    int y_tma;           // stage 2 writes y with tensor stores (ymap); needs split2 == 1,
                         // a 16-byte aligned y and out % 4 == 0
};

namespace {

// Rows one N tile list runs over, and how many such lists (segments) a GEMM has.
__host__ __device__ __forceinline__ int tile_span(const PrefillGemm& g) {
    return g.n_cat ? g.n_nseg * g.n_seg_rows : g.n_seg_rows;
}
__host__ __device__ __forceinline__ int tile_segs(const PrefillGemm& g) {
    return g.n_cat ? 1 : g.n_nseg;
}

// Segment and row within it of row n of tile list nseg (n_cat: the segment
// holding row n of the concatenation; past its end, segment 0 and row
// n_seg_rows, which reads as zeros).
__device__ __forceinline__ void seg_row(const PrefillGemm& g, int nseg, int n, int& s, int& rin) {
    if (!g.n_cat) { s = nseg; rin = n; return; }
    s = n / g.n_seg_rows;
    rin = n - s * g.n_seg_rows;
    if (s >= g.n_nseg) { s = 0; rin = g.n_seg_rows; }
}

__device__ __forceinline__ void tile_coords(const PrefillGemm& g, int t, int& mb, int& nseg,
                                            int& nt) {
    const int nt_per_seg = (tile_span(g) + kTileN - 1) / kTileN;
    const int n_tiles = tile_segs(g) * nt_per_seg;
    mb = t / n_tiles;
    const int r = t - mb * n_tiles;
    nseg = r / nt_per_seg;
    nt = r - nseg * nt_per_seg;
}

// Expand row n of one 256 x 64 B tile (K-major, 128-byte swizzle) from its 64
// packed sign bits.  Element k is the scale with its sign bit flipped when the
// bit is set: stage 1 scales per k (the K block's 64 values of g: read from
// global memory, every thread the same 128 bytes, with one M sub-tile per
// tile, so the expansion need not wait for the A tile; copied in with the A
// tile and read from shared memory with two, where the expansion's loads
// measured slower), stage 2 per row (hh = h[row] in both halves).  Per 16-byte piece (8 elements): one
// multiply spreads four sign bits to the top bits of the four bytes of a word
// (bit i to bit 8i + 7; the partial products never overlap, so nothing
// carries); PRMT in sign-replicating mode copies the top bit of byte 2p and
// 2p + 1 over bytes 0-1 and 2-3 of the fp16 pair p; one LOP3 keeps bits 15
// and 31 of that and flips them into the scales.  Rows past the matrix are
// expanded from whatever bits they get: only output columns that are never
// stored read them.
template <bool kGlobalG>
__device__ __forceinline__ void expand_row(uint32_t b_smem, const __half* gk, uint32_t g_smem, int n,
                                           uint2 bits, bool per_k, uint32_t hh) {
    // 16-byte piece c of row n sits at slot c ^ (n & 7) of the row's 128 bytes
    const uint32_t rowx = (uint32_t)(n >> 3) * 1024u + (uint32_t)(n & 7) * 144u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {                    // k = 8c .. 8c+7
        const uint32_t word = c < 4 ? bits.x : bits.y;
        const uint32_t byte = c & 3 ? (word >> (8 * (c & 3))) & 0xFFu : word & 0xFFu;
        const uint32_t slo = (byte & 0xFu) * 0x10204080u;
        const uint32_t shi = (byte >> 4) * 0x10204080u;
        uint4 base = make_uint4(hh, hh, hh, hh);
        if (per_k) {
            if (kGlobalG) {
                base = __ldg(reinterpret_cast<const uint4*>(gk) + c);
            } else {
                asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(base.x), "=r"(base.y), "=r"(base.z), "=r"(base.w)
                             : "r"(g_smem + 16u * (uint32_t)c));
            }
        }
        const uint32_t o0 = base.x ^ (prmt(slo, 0u, 0x9988u) & 0x80008000u);
        const uint32_t o1 = base.y ^ (prmt(slo, 0u, 0xBBAAu) & 0x80008000u);
        const uint32_t o2 = base.z ^ (prmt(shi, 0u, 0x9988u) & 0x80008000u);
        const uint32_t o3 = base.w ^ (prmt(shi, 0u, 0xBBAAu) & 0x80008000u);
        const uint32_t addr = b_smem + (rowx ^ (uint32_t)(c * 16));
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                     :: "r"(addr), "r"(o0), "r"(o1), "r"(o2), "r"(o3) : "memory");
    }
}

__device__ __forceinline__ uint2 load_bits(const PrefillGemm& g, int branch, int row, int kb) {
    if (row >= g.n_seg_rows) return make_uint2(0u, 0u);
    // a 64-sign K block is two words of one 16-word slice, so it is contiguous in both layouts
    const size_t off = g.sliced[branch]
                           ? (size_t)sliced_offset(g.n_seg_rows, g.nw, row, 2 * kb)
                           : (size_t)row * g.ldw[branch] + kb * 2;
    return __ldg(reinterpret_cast<const uint2*>(g.P[branch] + off));
}

__device__ __forceinline__ int ld_acquire_s32(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// The GEMM, tensor map, tile within its GEMM, K part and K-block range
// [kb0, kb1) of global tile t.
struct TileRef {
    const PrefillGemm* g;
    const CUtensorMap* map;
    int stage2, t, part, mb, nseg, nt, kb_per_seg, kb0, kb1;
};
template <bool SPLIT, bool SPLIT2>
__device__ __forceinline__ TileRef tile_ref(const PrefillPlan& plan, const CUtensorMap* amap1,
                                            const CUtensorMap* amap2, int t) {
    TileRef r;
    r.stage2 = t >= plan.n_tiles[0] ? 1 : 0;
    r.g = r.stage2 ? &plan.g[1] : &plan.g[0];
    r.map = r.stage2 ? amap2 : amap1;
    const int parts = r.stage2 ? (SPLIT2 ? plan.split2 : 1) : (SPLIT ? plan.split : 1);
    const int tl = t - (r.stage2 ? plan.n_tiles[0] : 0);
    r.t = tl / parts;
    r.part = tl - r.t * parts;
    tile_coords(*r.g, r.t, r.mb, r.nseg, r.nt);
    r.kb_per_seg = r.g->k_seg_len / kBlockK;
    const int n_kb = r.g->n_kseg * r.kb_per_seg;
    r.kb0 = (int)((long long)n_kb * r.part / parts);
    r.kb1 = (int)((long long)n_kb * (r.part + 1) / parts);
    return r;
}

// Piece p (8 fp16 values, l[n0 + 8p .. n0 + 8p + 7]) of segment nseg's l,
// zero past the segment.
__device__ __forceinline__ uint4 load_l8(const PrefillGemm& g, int nseg, int n0, int p) {
    const __half* lb = g.lscale[nseg] + n0 + 8 * p;
    if (n0 + 8 * p + 8 <= g.n_seg_rows && (reinterpret_cast<uintptr_t>(lb) & 15) == 0)
        return __ldg(reinterpret_cast<const uint4*>(lb));
    uint32_t e2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = n0 + 8 * p + 2 * i;
        const uint32_t lo = n < g.n_seg_rows ? __half_as_ushort(__ldg(lb + 2 * i)) : 0u;
        const uint32_t hi = n + 1 < g.n_seg_rows ? __half_as_ushort(__ldg(lb + 2 * i + 1)) : 0u;
        e2[i] = lo | (hi << 16);
    }
    return make_uint4(e2[0], e2[1], e2[2], e2[3]);
}

template <int MT, bool SPLIT, bool SPLIT2>
__global__ void __launch_bounds__(kPrefillThreads, 1)
prefill_gemm_kernel(const __grid_constant__ CUtensorMap amap1,
                    const __grid_constant__ CUtensorMap amap2,
                    const __grid_constant__ CUtensorMap ymap,
                    const __grid_constant__ PrefillPlan plan) {
    using S = Shape<MT>;
    constexpr int kStages = S::kStages, kStageBytes = S::kStageBytes;
    extern __shared__ __align__(1024) unsigned char dsm[];
    const uint32_t raw = smem_u32(dsm);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* basep = dsm + (base - raw);
    Ctl* ctl = reinterpret_cast<Ctl*>(basep + S::kOffCtl);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int n_tiles = plan.n_tiles[0] + plan.n_tiles[1];
    int* const err = plan.g[0].err;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctl->full_a[s]), 1);
            mbar_init(smem_u32(&ctl->full_b[s]), kExpandWarps);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&ctl->acc_full[i]), 1);
            mbar_init(smem_u32(&ctl->acc_empty[i]), kEpiWarps);
        }
        ctl->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(&ctl->tmem_base)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == kTmaWarp) {
        // ---------------- TMA producer for A (and, with two sub-tiles, the g slice
        // of stage 1); a stage-2 tile's boxes only once its rows of T are complete.
        // (A is not pulled into L2 ahead of the loads: the pre-pass has just
        // written it, and the prefetches only held up the TMA unit.)
        if (lane == 0) {
            auto acol = [](const TileRef& r, int kb) {
                const int ks = kb / r.kb_per_seg;
                return ks * r.g->k_seg_len + (kb - ks * r.kb_per_seg) * kBlockK;
            };
            int it = 0;
            for (int t = blockIdx.x; t < n_tiles && !ctl->abort; t += gridDim.x) {
                const TileRef r = tile_ref<SPLIT, SPLIT2>(plan, &amap1, &amap2, t);
                const PrefillGemm& g = *r.g;
                if (r.stage2) {
                    // wait (bounded) for the M block's rows of T, then order the TMA
                    // reads after the generic-proxy writes that produced them
                    const long long t0 = clock64();
                    while (ld_acquire_s32(plan.done + r.mb) < plan.done_target) {
                        if (*reinterpret_cast<volatile int*>(&ctl->abort)) break;
                        if (clock64() - t0 > kWaitLimit) {
                            atomicExch(&ctl->abort, 1);
                            atomicExch(err, (int)LB_ERR_TIMEOUT);
                            break;
                        }
                        __nanosleep(64);
                    }
                    if (ctl->abort) break;
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                for (int kb = r.kb0; kb < r.kb1; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t par = ((it / kStages) & 1) ^ 1;
                    if (!wait_bar(ctl, &ctl->empty[s], par, err)) break;
                    const uint32_t fb = smem_u32(&ctl->full_a[s]);
                    const int kcol = acol(r, kb);
                    const uint32_t sa = base + s * kStageBytes;
                    if (MT == 2 && !r.stage2) {   // the g slice, for the expansion (see expand_row)
                        const int kloc = kcol - (kb / r.kb_per_seg) * g.k_seg_len;
                        mbar_expect_tx(fb, MT * kABytes + kGBytes);
                        bulk_load(base + S::kOffG + s * kGBytes, g.bscale[r.nseg] + kloc, kGBytes, fb);
                    } else {
                        mbar_expect_tx(fb, MT * kABytes);
                    }
#pragma unroll
                    for (int j = 0; j < MT; ++j)
                        tma_load_2d(sa + j * kABytes, r.map, fb, kcol, (r.mb * MT + j) * kTileM);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int it = 0, tl = 0;
            for (int t = blockIdx.x; t < n_tiles && !ctl->abort; t += gridDim.x, ++tl) {
                const int buf = tl % S::kBufs;
                const uint32_t use = (uint32_t)(tl / S::kBufs);
                if (!wait_bar(ctl, &ctl->acc_empty[buf], (use & 1) ^ 1, err)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * MT * kTileN);
                const TileRef r = tile_ref<SPLIT, SPLIT2>(plan, &amap1, &amap2, t);
                bool ok = true;
                for (int kb = r.kb0; kb < r.kb1; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t par = (it / kStages) & 1;
                    if (!wait_bar(ctl, &ctl->full_a[s], par, err) ||
                        !wait_bar(ctl, &ctl->full_b[s], par, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_s = base + s * kStageBytes;
                    const uint64_t bd = sw128_desc(a_s + MT * kABytes);
#pragma unroll
                    for (int kk = 0; kk < kBlockK / 16; ++kk)
#pragma unroll
                        for (int j = 0; j < MT; ++j)
                            mma_f16(d + (uint32_t)(j * kTileN), sw128_desc(a_s + j * kABytes) + 2ull * kk,
                                    bd + 2ull * kk, (kb != r.kb0) || (kk != 0));
                    mma_commit(smem_u32(&ctl->empty[s]));
                }
                if (!ok) break;
                mma_commit(smem_u32(&ctl->acc_full[buf]));
            }
        }
    } else if (warp < kEpiWarps) {
        // ---------------- epilogue: TMEM -> registers -> shared staging -> global.
        // Warp w reads lane quarter w & 3; with MT = 2 the upper four warps drain
        // the second M sub-tile, with MT = 1 they take the upper 128 columns.
        // Each 32 x 32 chunk is scaled in registers (lane = row), written to
        // the warp's staging buffer (16-byte piece c of row r at slot c ^ (r & 7),
        // conflict-free both ways) and read back so that every store
        // instruction writes whole row segments (128 bytes of y, 64 of T).
        // The staging layout is the tensor map's 128-byte swizzle, so with
        // plan.y_tma a chunk of y leaves as one tensor store issued by lane 0
        // (rows and columns past y clipped by the map), and the warp goes on
        // to the next chunk while the TMA unit writes it.
        const int q = warp & 3, hw = warp >> 2;
        const int sub = MT == 2 ? hw : 0;
        const int c_begin = MT == 2 ? 0 : hw * (kTileN / 2);
        const int c_end = MT == 2 ? kTileN : c_begin + kTileN / 2;
        const uint32_t stg = base + S::kOffEpi + (uint32_t)warp * kEpiBytes;
        const uint32_t my_row = stg + (uint32_t)lane * 128u;
        int tl = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tl) {
            const TileRef r = tile_ref<SPLIT, SPLIT2>(plan, &amap1, &amap2, t);
            const PrefillGemm& g = *r.g;
            const int mb = r.mb, nseg = r.nseg, nt = r.nt;
            const int ldt = g.n_nseg * g.n_seg_rows;      // T row pitch (stage 1)
            const int buf = tl % S::kBufs;
            // per-tile loads go out before the wait: the row scales, and (stage 1)
            // l of the first chunk; l of chunk c+1 is loaded while chunk c is stored
            const int m0 = (mb * MT + sub) * kTileM + q * 32;     // first row of this warp
            const int m = m0 + lane;
            const bool mok = m < g.M;
            const float sa = mok ? __ldg(g.row_sa + m) : 1.0f;
            const float sc = mok ? __ldg(g.row_sc + m) : 1.0f;
            // (stage 1) lane p < 4 holds piece p of the next chunk's l
            uint4 lnext = make_uint4(0u, 0u, 0u, 0u);
            const int span = tile_span(g);
            if (g.stage == 1 && lane < 4 && nt * kTileN + c_begin < span) {
                int ls, ln;
                seg_row(g, nseg, nt * kTileN + c_begin, ls, ln);
                lnext = load_l8(g, ls, ln, lane);
            }
            // every lane waits; the warp stops together so the .sync.aligned loads stay converged
            if (!__all_sync(0xffffffffu, wait_bar(ctl, &ctl->acc_full[buf],
                                                  (uint32_t)(tl / S::kBufs) & 1, err)))
                break;
            tc_fence_after();
            const float f = g.stage == 1 ? sc / sa : 1.0f / sc;
            const uint32_t tacc = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)((buf * MT + sub) * kTileN);
            // K split of stage 1: write this warp's partial sums (lane-interleaved
            // 16-byte pieces, so every access of the warp is 512 contiguous bytes),
            // then take a ticket; the last of the parts finishes the region
            const bool split = SPLIT && !r.stage2 && plan.split > 1;
            bool finish = true;
            if constexpr (SPLIT) if (split) {
                float* pw = plan.partial +
                            ((size_t)(r.t * plan.split + r.part) * kEpiWarps + warp) * kPartFloats;
                for (int c0 = c_begin, ci = 0; c0 < c_end; c0 += 32, ++ci) {
                    float v[32];
                    __syncwarp();
                    tmem_ld32(tacc + (uint32_t)c0, v);
                    // rows past M are never stored, so their partial sums are not kept
                    if (mok) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            __stcg(reinterpret_cast<float4*>(pw + ci * 1024 + (i * 32 + lane) * 4),
                                   make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
                    }
                }
                __syncwarp();
                int ticket = 0;
                if (lane == 0)
                    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                                 : "=r"(ticket) : "l"(plan.tickets + r.t * kEpiWarps + warp) : "memory");
                finish = __shfl_sync(0xffffffffu, ticket, 0) == plan.split - 1;
                __syncwarp();
                if (finish) {
                    // fold the other parts' sums into this warp's accumulator in TMEM,
                    // half a chunk (16 columns) at a time
                    const float* p0 = plan.partial + (size_t)r.t * plan.split * kEpiWarps * kPartFloats +
                                      (size_t)warp * kPartFloats;
                    for (int h = 0; h < (c_end - c_begin) / 16; ++h) {
                        // every other part's piece is requested before any is added, so
                        // a half chunk costs one round trip to L2, not one per part
                        float4 o[kSplitMax - 1][4];
#pragma unroll
                        for (int q = 0; q < kSplitMax - 1; ++q) {
                            const int p = q < r.part ? q : q + 1;   // the parts other than this one
                            const bool use = p < plan.split && mok;
                            const float* pc = p0 + (size_t)p * kEpiWarps * kPartFloats + h * 512;
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                o[q][i] = use ? __ldcg(reinterpret_cast<const float4*>(pc + (i * 32 + lane) * 4))
                                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        }
                        float v[16];
                        __syncwarp();
                        tmem_ld16(tacc + (uint32_t)(c_begin + 16 * h), v);
#pragma unroll
                        for (int q = 0; q < kSplitMax - 1; ++q) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                v[4 * i] += o[q][i].x;
                                v[4 * i + 1] += o[q][i].y;
                                v[4 * i + 2] += o[q][i].z;
                                v[4 * i + 3] += o[q][i].w;
                            }
                        }
                        tmem_st16(tacc + (uint32_t)(c_begin + 16 * h), v);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                }
            }
            for (int c0 = c_begin; finish && c0 < c_end; c0 += 32) {
                float v[32];
                __syncwarp();
                tmem_ld32(tacc + (uint32_t)c0, v);
                const int n0 = nt * kTileN + c0;       // row within the N tile list
                if (n0 >= span) continue;              // warp-uniform
                if (g.stage == 1) {
                    // T = l * t * 2^c with t = D / 2^a, fp16, 4 pieces of 16 bytes per row.
                    // This chunk's l goes to the half of row 0 of the staging buffer
                    // that the chunk leaves unused (slots 4-7); the next chunk's l is
                    // requested meanwhile.
                    const uint32_t lbuf = stg + 64u;
                    if (lane < 4) {
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(lbuf + 16u * (uint32_t)lane), "r"(lnext.x), "r"(lnext.y),
                                        "r"(lnext.z), "r"(lnext.w) : "memory");
                        if (c0 + 32 < c_end && n0 + 32 < span) {
                            int ls, ln;      // (a chunk never straddles two segments: r % 32 == 0)
                            seg_row(g, nseg, n0 + 32, ls, ln);
                            lnext = load_l8(g, ls, ln, lane);
                        }
                    }
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t w[4];
                        uint4 lv;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(lv.x), "=r"(lv.y), "=r"(lv.z), "=r"(lv.w)
                                     : "r"(lbuf + 16u * (uint32_t)c));
                        const uint32_t lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            const float2 l2 = __half22float2(*reinterpret_cast<const __half2*>(&lw[p]));
                            const __half2 h2 = __floats2half2_rn(v[8 * c + 2 * p] * f * l2.x,
                                                                 v[8 * c + 2 * p + 1] * f * l2.y);
                            w[p] = *reinterpret_cast<const uint32_t*>(&h2);
                        }
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(my_row + (uint32_t)((c ^ (lane & 7)) * 16)),
                                        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
                    }
                    __syncwarp();
                    const int cc = lane & 3;
                    const int col = n0 + 8 * cc;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {              // rows 8i .. 8i+7, 4 lanes per row
                        const int rr = 8 * i + (lane >> 2);
                        uint4 o;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
                                     : "r"(stg + (uint32_t)rr * 128u + (uint32_t)((cc ^ (rr & 7)) * 16)));
                        if (m0 + rr < g.M && col < span) {
                            __half* dst = g.T + (size_t)(m0 + rr) * ldt +
                                          (size_t)(g.n_cat ? 0 : nseg) * g.n_seg_rows + col;
                            if (col + 8 <= span) {
                                *reinterpret_cast<uint4*>(dst) = o;
                            } else {
                                const uint32_t ow[4] = {o.x, o.y, o.z, o.w};
                                for (int e = 0; e < 8 && col + e < span; ++e)
                                    reinterpret_cast<uint16_t*>(dst)[e] = (uint16_t)(ow[e >> 1] >> (16 * (e & 1)));
                            }
                        }
                    }
                } else {
                    // y = D / 2^c, fp32, 8 pieces of 16 bytes per row
                    if (plan.y_tma) {   // the previous chunk's store has read the buffer
                        if (lane == 0) bulk_wait_read();
                        __syncwarp();
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(my_row + (uint32_t)((c ^ (lane & 7)) * 16)),
                                        "f"(v[4 * c] * f), "f"(v[4 * c + 1] * f), "f"(v[4 * c + 2] * f),
                                        "f"(v[4 * c + 3] * f) : "memory");
                    if (plan.y_tma) {
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                        if (lane == 0 && m0 < g.M) {   // (rows past M: nothing to store)
                            tma_store_2d(&ymap, stg, n0, m0);
                            bulk_commit();
                        }
                        continue;
                    }
                    __syncwarp();
                    const int cc = lane & 7;
                    const int col = n0 + 4 * cc;
                    const bool vec = (g.n_seg_rows & 3) == 0;
                    const bool add = SPLIT2 && plan.split2 > 1;   // K parts reduce into y
#pragma unroll
                    for (int i = 0; i < 8; ++i) {              // rows 4i .. 4i+3, 8 lanes per row
                        const int rr = 4 * i + (lane >> 3);
                        float4 o;
                        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                     : "=f"(o.x), "=f"(o.y), "=f"(o.z), "=f"(o.w)
                                     : "r"(stg + (uint32_t)rr * 128u + (uint32_t)((cc ^ (rr & 7)) * 16)));
                        if (m0 + rr < g.M && col < g.n_seg_rows) {
                            float* dst = g.y + (size_t)(m0 + rr) * g.n_seg_rows + col;
                            if (vec) {
                                if (add)
                                    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                                                 :: "l"(dst), "f"(o.x), "f"(o.y), "f"(o.z), "f"(o.w)
                                                 : "memory");
                                else
                                    *reinterpret_cast<float4*>(dst) = o;
                            } else {
                                const float ov[4] = {o.x, o.y, o.z, o.w};
                                for (int e = 0; e < 4 && col + e < g.n_seg_rows; ++e) {
                                    if (add) atomicAdd(dst + e, ov[e]);
                                    else dst[e] = ov[e];
                                }
                            }
                        }
                    }
                }
                __syncwarp();                          // staging buffer free for the next chunk
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&ctl->acc_empty[buf]));
                // stage 1: this warp's rows of T are written; publish them to the
                // stage-2 tiles of the M block (release orders the warp's stores)
                if (!r.stage2 && finish)
                    asm volatile("red.release.gpu.global.add.s32 [%0], 1;"
                                 :: "l"(plan.done + mb) : "memory");
            }
        }
        if (plan.y_tma && lane == 0) bulk_wait_all();   // this warp's tensor stores are done
    } else if (warp >= kExpandWarp0) {
        // ---------------- B producers: packed signs -> fp16 tile, one row per thread
        const int e = threadIdx.x - kExpandWarp0 * 32;
        int s = 0;                                   // pipeline slot of the current K block
        uint32_t ph = 0;                             // and the parity of its current use
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const TileRef r = tile_ref<SPLIT, SPLIT2>(plan, &amap1, &amap2, t);
            const PrefillGemm& g = *r.g;
            const int nseg = r.nseg, nt = r.nt, kb_per_seg = r.kb_per_seg;
            const int n_kb = r.kb1 - r.kb0;          // K blocks of this tile (its part of K)
            const int row = nt * kTileN + e;
            int bseg = nseg, brow = row;             // stage 1: this row's branch and row in it
            if (g.stage == 1) seg_row(g, nseg, row, bseg, brow);
            uint32_t hh0 = 0u, hh1 = 0u;             // h[row] of each branch in both fp16 halves
            if (g.stage == 2 && row < g.n_seg_rows) {
                const uint32_t h0 = __half_as_ushort(__ldg(g.bscale[0] + row));
                hh0 = h0 | (h0 << 16);
                if (g.n_kseg > 1) {
                    const uint32_t h1 = __half_as_ushort(__ldg(g.bscale[1] + row));
                    hh1 = h1 | (h1 << 16);
                }
            }
            // sign bits, fetched kBitsAhead K blocks ahead into a register ring;
            // (fs, fk) = K segment and block within it of the next fetch
            const int seg0 = r.kb0 / kb_per_seg, kin0 = r.kb0 - seg0 * kb_per_seg;
            int fs = seg0, fk = kin0;
            auto fetch = [&]() {
                const uint2 v = g.stage == 1 ? load_bits(g, bseg, brow, fk) : load_bits(g, fs, row, fk);
                if (++fk == kb_per_seg) { fk = 0; ++fs; }
                return v;
            };
            uint2 nx[kBitsAhead];
#pragma unroll
            for (int j = 0; j < kBitsAhead; ++j) nx[j] = j < n_kb ? fetch() : make_uint2(0u, 0u);
            int seg = seg0, kin = kin0;              // K segment of the current block, block within it
            for (int kb0 = 0; kb0 < n_kb && ok; kb0 += kBitsAhead) {
#pragma unroll
                for (int j = 0; j < kBitsAhead; ++j) {
                    const int kb = kb0 + j;
                    if (kb >= n_kb) break;
                    const uint2 cur = nx[j];
                    if (kb + kBitsAhead < n_kb) nx[j] = fetch();
                    // with one sub-tile the expansion reads g from memory and does not
                    // wait for the A tile; with two it reads the copy that came with it
                    constexpr bool kGlobalG = MT == 1;
                    bool w = wait_bar(ctl, &ctl->empty[s], ph ^ 1, err);
                    if (!kGlobalG && w && g.stage == 1) w = wait_bar(ctl, &ctl->full_a[s], ph, err);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
                    const uint32_t sb = base + s * kStageBytes + MT * kABytes;
                    const __half* gk = g.stage == 1 ? g.bscale[bseg] + (size_t)kin * kBlockK : nullptr;
                    expand_row<kGlobalG>(sb, gk, base + S::kOffG + s * kGBytes, e, cur, g.stage == 1,
                                         (seg & 1) ? hh1 : hh0);
                    fence_async_smem();              // make the stores visible to the tensor core
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&ctl->full_b[s]));
                    if (++s == kStages) { s = 0; ph ^= 1; }
                    if (++kin == kb_per_seg) { kin = 0; ++seg; }
                }
            }
        }
    }

    // Drain: every role is done (or aborted).  Give in-flight TMA loads time to
    // land before the shared memory goes away, then free TMEM.
    __syncthreads();
    if (ctl->abort && threadIdx.x == 0) {
        const long long t0 = clock64();
        while (clock64() - t0 < 2000000LL) { }
    }
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// Pre-pass: per row m, 2^a_m (brings max|x| into [2^14, 2^15)), the fp16 copy
// of x * 2^a_m, and 2^c_m (keeps |T| <= 65504; see the header comment).  Every
// thread takes 8 consecutive elements at a time with 16-byte loads (in is a
// multiple of 64 and x, g are 16-byte aligned).
__device__ __forceinline__ void cvt8_x(uint4 u, int x_kind, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (x_kind == VK_X_F16) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            v[2 * i] = f.x; v[2 * i + 1] = f.y;
        } else {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            v[2 * i] = f.x; v[2 * i + 1] = f.y;
        }
    }
}
// The 16 bytes of a 16-bit x at element `at` (raw), unused for fp32 x.
__device__ __forceinline__ uint4 raw8_x(const void* x, int x_kind, size_t at) {
    if (x_kind == VK_X_F32) return make_uint4(0u, 0u, 0u, 0u);
    return *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + at);
}
__device__ __forceinline__ void load8_x(const void* x, int x_kind, size_t at, float (&v)[8]) {
    if (x_kind == VK_X_F32) {
        const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + at);
        const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + at + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        return;
    }
    cvt8_x(raw8_x(x, x_kind, at), x_kind, v);
}
__device__ __forceinline__ void load8_h(const __half* p, size_t at, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p + at));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        v[2 * i] = f.x; v[2 * i + 1] = f.y;
    }
}

constexpr int kPrepassThreads = 512;
constexpr int kPrepassRows = 4;                               // rows of x per block
constexpr int kRowThreads = kPrepassThreads / kPrepassRows;   // threads per row
constexpr int kRowStep = 8 * kRowThreads;                     // elements of a row per step
constexpr int kCachedSteps = 4;                               // steps kept in registers

// One block takes kPrepassRows rows (kRowThreads threads each), three blocks
// to an SM (40 registers a thread), so that an SM has several rows' loads in
// flight; a thread's first kCachedSteps steps of a
// 16-bit x stay in registers for the second pass (rows up to 4096 elements are
// read once), and all of them are requested before the first is used.  The
// block also takes max_k |l_b[k]| and max_k |g_b[k]| of each branch itself.
// The launch also clears what the GEMM kernel counts or adds into (the
// workspace header, the per-M-block completion counts, the split tickets and,
// when the second GEMM is split along K, y), so a call is two launches.
struct PrepassZero {
    int* i[3];
    int ni[3];
    float* f;          // 16-byte aligned
    long long nf;
};

__global__ void __launch_bounds__(kPrepassThreads, 3) prefill_prepass_kernel(
    const void* __restrict__ x, int x_kind, int M, int in, int nb,
    const __half* __restrict__ g0, const __half* __restrict__ g1,
    const __half* __restrict__ l0, const __half* __restrict__ l1, int r,
    __half* __restrict__ X16, float* __restrict__ row_sa, float* __restrict__ row_sc,
    const PrepassZero z) {
    constexpr int kWarps = kPrepassThreads / 32, kGroupWarps = kRowThreads / 32;
    {
        const long long tid = (long long)blockIdx.x * kPrepassThreads + threadIdx.x;
        const long long nth = (long long)gridDim.x * kPrepassThreads;
        for (int k = 0; k < 3; ++k)
            for (long long i = tid; i < z.ni[k]; i += nth) z.i[k][i] = 0;
        const long long n4 = z.nf / 4;
        for (long long i = tid; i < n4; i += nth)
            reinterpret_cast<float4*>(z.f)[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (long long i = 4 * n4 + tid; i < z.nf; i += nth) z.f[i] = 0.0f;
    }
    __shared__ float red[kWarps][2];
    __shared__ float lred[kWarps][2];
    const int grp = threadIdx.x / kRowThreads, t = threadIdx.x % kRowThreads;
    const int m = blockIdx.x * kPrepassRows + grp;
    const bool row_ok = m < M;
    const size_t row = (size_t)(row_ok ? m : 0) * in;
    // the row's first steps of x, all requested before any is used
    uint4 xc[kCachedSteps];
#pragma unroll
    for (int c = 0; c < kCachedSteps; ++c) {
        const int j0 = c * kRowStep + 8 * t;
        xc[c] = row_ok && j0 < in ? raw8_x(x, x_kind, row + j0) : make_uint4(0u, 0u, 0u, 0u);
    }
    // max |l| and max |g| of each branch, over the block (their loads go out with x's)
    float lm0 = 0.0f, lm1 = 0.0f, gm0 = 0.0f, gm1 = 0.0f;
    for (int k = threadIdx.x; k < r; k += kPrepassThreads) {
        lm0 = fmaxf(lm0, fabsf(__half2float(__ldg(l0 + k))));
        if (nb > 1) lm1 = fmaxf(lm1, fabsf(__half2float(__ldg(l1 + k))));
    }
    for (int k = 8 * threadIdx.x; k < in; k += 8 * kPrepassThreads) {
        float gv[8];
        load8_h(g0, k, gv);
#pragma unroll
        for (int i = 0; i < 8; ++i) gm0 = fmaxf(gm0, fabsf(gv[i]));
        if (nb > 1) {
            load8_h(g1, k, gv);
#pragma unroll
            for (int i = 0; i < 8; ++i) gm1 = fmaxf(gm1, fabsf(gv[i]));
        }
    }
    // max |x| and sum |x| of the row
    float mx = 0.0f, sx = 0.0f;
    auto take = [&](const float (&xv)[8]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mx = fmaxf(mx, fabsf(xv[i]));
            sx += fabsf(xv[i]);
        }
    };
#pragma unroll
    for (int c = 0; c < kCachedSteps; ++c) {
        const int j0 = c * kRowStep + 8 * t;
        if (!row_ok || j0 >= in) continue;
        float xv[8];
        if (x_kind == VK_X_F32) load8_x(x, x_kind, row + j0, xv);
        else cvt8_x(xc[c], x_kind, xv);
        take(xv);
    }
    for (int j0 = kCachedSteps * kRowStep + 8 * t; row_ok && j0 < in; j0 += kRowStep) {
        float xv[8];
        load8_x(x, x_kind, row + j0, xv);
        take(xv);
    }
    const int w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        sx += __shfl_xor_sync(0xffffffffu, sx, o);
        lm0 = fmaxf(lm0, __shfl_xor_sync(0xffffffffu, lm0, o));
        lm1 = fmaxf(lm1, __shfl_xor_sync(0xffffffffu, lm1, o));
        gm0 = fmaxf(gm0, __shfl_xor_sync(0xffffffffu, gm0, o));
        gm1 = fmaxf(gm1, __shfl_xor_sync(0xffffffffu, gm1, o));
    }
    if ((threadIdx.x & 31) == 0) {
        red[w][0] = mx; red[w][1] = sx;
        lred[w][0] = lm0 * gm0; lred[w][1] = lm1 * gm1;
    }
    __syncthreads();
    float M0 = 0.0f, L0 = 0.0f, lg = 0.0f;
    for (int v = 0; v < kWarps; ++v) lg = fmaxf(lg, fmaxf(lred[v][0], nb > 1 ? lred[v][1] : 0.0f));
    for (int v = grp * kGroupWarps; v < (grp + 1) * kGroupWarps; ++v) {
        M0 = fmaxf(M0, red[v][0]);
        L0 += red[v][1];
    }
    if (!row_ok) return;
    // 2^a: the largest power of two with max|x| * 2^a < 2^15
    float sa = 1.0f;
    if (M0 > 0.0f && isfinite(M0)) sa = exp2f(fminf(fmaxf(14.0f - floorf(log2f(M0)), -126.0f), 126.0f));
    // 2^c: the largest power of two with bound * 2^c <= 2^15 (< 65504), where
    // |T| <= max|l| max|g| sum|x|; the bound is padded by 1/64 for fp32 rounding
    // in the sums.
    const float bound = L0 * lg * (1.0f + 1.0f / 64);
    float sc = 1.0f;
    if (bound > 0.0f && isfinite(bound))
        sc = exp2f(fminf(fmaxf(15.0f - ceilf(log2f(bound)), -126.0f), 126.0f));
    if (t == 0) {
        row_sa[m] = sa;
        row_sc[m] = sc;
    }
    auto put = [&](int j0, const float (&xv)[8]) {
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h2 = __floats2half2_rn(xv[2 * i] * sa, xv[2 * i + 1] * sa);
            q[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(X16 + row + j0) = make_uint4(q[0], q[1], q[2], q[3]);
    };
#pragma unroll
    for (int c = 0; c < kCachedSteps; ++c) {
        const int j0 = c * kRowStep + 8 * t;
        if (j0 >= in) continue;
        float xv[8];
        if (x_kind == VK_X_F32) load8_x(x, x_kind, row + j0, xv);
        else cvt8_x(xc[c], x_kind, xv);
        put(j0, xv);
    }
    for (int j0 = kCachedSteps * kRowStep + 8 * t; j0 < in; j0 += kRowStep) {
        float xv[8];
        load8_x(x, x_kind, row + j0, xv);
        put(j0, xv);
    }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encode() {
    static EncodeTiled fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    }
    return fn;
}

// Row-major fp32 [rows][cols] (cols % 4 == 0, 16-byte aligned) with a 32 x 32
// box and the 128-byte swizzle: one epilogue chunk of y.
bool make_ymap(CUtensorMap* map, float* ptr, int rows, int cols) {
    EncodeTiled enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ptr, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major fp16 [rows][cols] with a 64 x 128 box and the 128-byte swizzle.
bool make_amap(CUtensorMap* map, const __half* ptr, int rows, int cols) {
    EncodeTiled enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {kBlockK, kTileM};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(ptr), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t prefill_configure() {
    const void* fns[6] = {(const void*)prefill_gemm_kernel<1, false, false>,
                          (const void*)prefill_gemm_kernel<1, true, false>,
                          (const void*)prefill_gemm_kernel<1, true, true>,
                          (const void*)prefill_gemm_kernel<2, false, false>,
                          (const void*)prefill_gemm_kernel<2, true, false>,
                          (const void*)prefill_gemm_kernel<2, true, true>};
    const int smem[6] = {Shape<1>::kSmem, Shape<1>::kSmem, Shape<1>::kSmem,
                         Shape<2>::kSmem, Shape<2>::kSmem, Shape<2>::kSmem};
    for (int i = 0; i < 6; ++i) {
        const cudaError_t e =
            cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, smem[i]);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Stage 1 may be split along K only when it has fewer tiles than the split
// buffer has parts even with one sub-tile and two branches; the buffer is
// reserved for exactly those shapes.
static bool split_possible(int64_t M, int64_t r) {
    const int64_t tiles = ((M + kTileM - 1) / kTileM) * 2 * ((r + kTileN - 1) / kTileN);
    return tiles < kSplitMaxParts;
}

static size_t split_bytes(int64_t M, int64_t r) {
    if (!split_possible(M, r)) return 0;
    return (size_t)kSplitMaxParts * kEpiWarps * kPartFloats * sizeof(float) +
           (size_t)kSplitMaxParts * kEpiWarps * sizeof(int);
}

size_t prefill_workspace_bytes(int64_t M, int64_t in, int64_t r, bool with_split) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    return up(sizeof(WsHeader)) + up(2 * (size_t)M * in) + up(2 * (size_t)M * 2 * r) +
           up(8 * (size_t)M) + 256 + up(4 * (size_t)((M + kTileM - 1) / kTileM)) +
           (with_split ? up(split_bytes(M, r)) : 0);
}

bool prefill_shape_ok(int64_t M, int64_t in, int64_t out, int64_t r) {
    return M >= 1 && in % kBlockK == 0 && r % kBlockK == 0 && out >= 1 && in <= (1 << 20) &&
           r <= (1 << 16) && out <= (1 << 24) && M <= (1 << 24);
}

// Sub-tiles per B tile: two halve the sign expansion per MMA but double the
// tile, so on few tiles the coarser grain can cost a round of the persistent
// grid.  Pick the shape with the smaller estimated time, a two-sub-tile tile
// costing kTile2Cost one-sub-tile tiles.  LB_PREFILL_SUBTILES=1 or 2 in the
// environment (read on every call) fixes the choice; both give the same result.
static long long gemm_tiles(const PrefillGemm& p, int mt) {
    return (long long)tile_segs(p) * ((tile_span(p) + kTileN - 1) / kTileN) *
           ((p.M + mt * kTileM - 1) / (mt * kTileM));
}

static int pick_subtiles(const PrefillGemm* p, int grid) {
    constexpr double kTile2Cost = 1.35;
    if (const char* env = std::getenv("LB_PREFILL_SUBTILES")) {
        if (env[0] == '1' && env[1] == 0) return 1;
        if (env[0] == '2' && env[1] == 0) return 2;
    }
    if (p[0].M <= kTileM) return 1;
    // makespan estimate: the K blocks of all tiles spread over the grid, plus
    // one tile of imbalance (tiles are dealt round-robin)
    double c[3] = {0.0, 0.0, 0.0};
    for (int mt = 1; mt <= 2; ++mt) {
        const double cost = mt == 2 ? kTile2Cost : 1.0;
        double work = 0.0, lump = 0.0;
        for (int i = 0; i < 2; ++i) {
            const double n_kb = (double)p[i].n_kseg * (double)(p[i].k_seg_len / kBlockK);
            work += (double)gemm_tiles(p[i], mt) * n_kb * cost;
            lump = n_kb * cost > lump ? n_kb * cost : lump;
        }
        c[mt] = work / (double)grid + lump;
    }
    return c[2] < c[1] ? 2 : 1;
}

// The K splits of both GEMMs for tiles of MT sub-tiles on `grid` CTAs (host only).
template <int MT>
static void plan_gemms(PrefillPlan& plan, int grid) {
    const int tiles1 = (int)gemm_tiles(plan.g[0], MT);
    // split stage 1 along K while it would leave SMs idle: up to kSplitMax parts of at
    // least 8 K blocks each, at most kSplitMaxParts parts in all
    int split = 1;
    if (plan.partial != nullptr) {
        const int n_kb = plan.g[0].n_kseg * (plan.g[0].k_seg_len / kBlockK);
        while (split < kSplitMax && tiles1 * (split + 1) <= grid && tiles1 * (split + 1) <= kSplitMaxParts &&
               n_kb / (split + 1) >= 8)
            ++split;
    }
    plan.split = split;
    plan.n_tiles[0] = tiles1 * split;
    // and stage 2 the same way (its parts reduce into y, zeroed first)
    const int tiles2 = (int)gemm_tiles(plan.g[1], MT);
    const int n_kb2 = plan.g[1].n_kseg * (plan.g[1].k_seg_len / kBlockK);
    int split2 = 1;
    while (split2 < kSplit2Max && tiles2 * (split2 + 1) <= grid && n_kb2 / (split2 + 1) >= 8)
        ++split2;
    // LB_PREFILL_SPLIT2=1..4 in the environment (read on every call) fixes the
    // split, at most one part per K block so that no part is empty
    if (const char* env = std::getenv("LB_PREFILL_SPLIT2")) {
        const int v = std::atoi(env);
        if (v >= 1 && v <= kSplit2Max) split2 = v < n_kb2 ? v : n_kb2;
    }
    plan.split2 = split2;
    plan.n_tiles[1] = tiles2 * split2;
    plan.done_target = kEpiWarps * tile_segs(plan.g[0]) * ((tile_span(plan.g[0]) + kTileN - 1) / kTileN);
}

template <int MT>
static cudaError_t launch_gemms(const PrefillPlan& plan, const CUtensorMap& m1,
                                const CUtensorMap& m2, const CUtensorMap& ym, int grid,
                                cudaStream_t s) {
    // the split instantiations cost registers, so shapes that split nothing run without them
    if (plan.split2 > 1)
        prefill_gemm_kernel<MT, true, true><<<grid, kPrefillThreads, Shape<MT>::kSmem, s>>>(m1, m2, ym, plan);
    else if (plan.split > 1)
        prefill_gemm_kernel<MT, true, false><<<grid, kPrefillThreads, Shape<MT>::kSmem, s>>>(m1, m2, ym, plan);
    else
        prefill_gemm_kernel<MT, false, false><<<grid, kPrefillThreads, Shape<MT>::kSmem, s>>>(m1, m2, ym, plan);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const void* x, int x_kind, int64_t M, int64_t in, int64_t out,
                           int64_t r, const lb_branch* br, int nb, float* y, void* workspace,
                           cudaStream_t s, bool allow_split) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    size_t off = up(sizeof(WsHeader));
    __half* X16 = reinterpret_cast<__half*>(ws + off);
    off += up(2 * (size_t)M * in);
    __half* T = reinterpret_cast<__half*>(ws + off);
    off += up(2 * (size_t)M * 2 * r);
    float* sa = reinterpret_cast<float*>(ws + off);
    float* sc = sa + M;
    off += up(8 * (size_t)M);
    off += 256;                                     // (reserved)
    int* done = reinterpret_cast<int*>(ws + off);   // per M block, stage-1 tiles finished
    off += up(4 * (size_t)((M + kTileM - 1) / kTileM));
    float* partial = nullptr;                       // stage-1 K split: partial sums, tickets
    int* tickets = nullptr;
    if (allow_split && split_possible(M, r)) {
        partial = reinterpret_cast<float*>(ws + off);
        tickets = reinterpret_cast<int*>(ws + off + (size_t)kSplitMaxParts * kEpiWarps * kPartFloats * sizeof(float));
    }

    PrefillPlan plan = {};
    plan.done = done;
    plan.partial = partial;
    plan.tickets = tickets;
    // stage 1: T = (x 2^a) (g o sign V)^T, epilogue applies l, 2^-a, 2^c
    CUtensorMap amap1, amap2;
    if (!make_amap(&amap1, X16, (int)M, (int)in)) return cudaErrorInvalidValue;
    {
        PrefillGemm& p = plan.g[0];
        p.M = (int)M; p.n_seg_rows = (int)r; p.n_nseg = nb; p.n_kseg = 1; p.k_seg_len = (int)in;
        p.stage = 1;
        p.nw = (int)((in + 31) / 32);
        for (int b = 0; b < 2; ++b) {
            const lb_branch& B = br[b < nb ? b : 0];
            p.P[b] = B.Vp;
            p.ldw[b] = (int)(B.ld_v ? B.ld_v : (in + 31) / 32);
            p.sliced[b] = B.layout == LB_LAYOUT_SLICES ? 1 : 0;
            p.bscale[b] = reinterpret_cast<const __half*>(B.g);
            p.lscale[b] = reinterpret_cast<const __half*>(B.l);
        }
        p.row_sa = sa; p.row_sc = sc; p.T = T; p.y = nullptr; p.err = &hdr->error;
    }
    // stage 2: y = (T) (h o sign U)^T over K = nb * r, epilogue divides 2^c out
    if (!make_amap(&amap2, T, (int)M, (int)(nb * r))) return cudaErrorInvalidValue;
    {
        PrefillGemm& p = plan.g[1];
        p.M = (int)M; p.n_seg_rows = (int)out; p.n_nseg = 1; p.n_kseg = nb; p.k_seg_len = (int)r;
        p.stage = 2;
        p.nw = (int)((r + 31) / 32);
        for (int b = 0; b < 2; ++b) {
            const lb_branch& B = br[b < nb ? b : 0];
            p.P[b] = B.Up;
            p.ldw[b] = (int)(B.ld_u ? B.ld_u : (r + 31) / 32);
            p.sliced[b] = B.layout == LB_LAYOUT_SLICES ? 1 : 0;
            p.bscale[b] = reinterpret_cast<const __half*>(B.h);
            p.lscale[b] = nullptr;
        }
        p.row_sa = sa; p.row_sc = sc; p.T = nullptr; p.y = y; p.err = &hdr->error;
    }
    const int grid = device_sm_count();
    const int mt = pick_subtiles(plan.g, grid);
    // with one sub-tile (the expansion then reads g per row from memory) the
    // branches of stage 1 share N tiles when that takes fewer of them
    if (mt == 1 && nb > 1) {
        PrefillGemm cat = plan.g[0];
        cat.n_cat = 1;
        if (gemm_tiles(cat, 1) < gemm_tiles(plan.g[0], 1)) plan.g[0].n_cat = 1;
    }
    if (mt == 2) plan_gemms<2>(plan, grid);
    else plan_gemms<1>(plan, grid);

    // pre-pass (and the clearing the GEMM kernel relies on), then both GEMMs
    PrepassZero z = {};
    z.i[0] = reinterpret_cast<int*>(hdr);
    z.ni[0] = (int)(sizeof(WsHeader) / sizeof(int));
    z.i[1] = done;
    z.ni[1] = (int)((M + mt * kTileM - 1) / (mt * kTileM));
    z.i[2] = tickets;
    z.ni[2] = plan.split > 1 ? (int)(plan.n_tiles[0] / plan.split) * kEpiWarps : 0;
    z.f = plan.split2 > 1 ? y : nullptr;
    z.nf = plan.split2 > 1 ? (long long)M * out : 0;
    const long long row_blocks = (M + kPrepassRows - 1) / kPrepassRows;
    const long long zero_blocks = std::min<long long>(4LL * grid, (z.nf / 4 + kPrepassThreads - 1) / kPrepassThreads);
    const __half* l1 = reinterpret_cast<const __half*>(br[nb > 1 ? 1 : 0].l);
    const __half* g1 = reinterpret_cast<const __half*>(br[nb > 1 ? 1 : 0].g);
    prefill_prepass_kernel<<<(unsigned)std::max(row_blocks, zero_blocks), kPrepassThreads, 0, s>>>(
        x, x_kind, (int)M, (int)in, nb, reinterpret_cast<const __half*>(br[0].g), g1,
        reinterpret_cast<const __half*>(br[0].l), l1, (int)r, X16, sa, sc, z);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // y by tensor stores when nothing reduces into it and the map can describe it
    CUtensorMap ymap = {};
    plan.y_tma = plan.split2 == 1 && out % 4 == 0 && (reinterpret_cast<uintptr_t>(y) & 15) == 0 &&
                 make_ymap(&ymap, y, (int)M, (int)out);
    return mt == 2 ? launch_gemms<2>(plan, amap1, amap2, ymap, grid, s)
                   : launch_gemms<1>(plan, amap1, amap2, ymap, grid, s);
}

}  // namespace lb
