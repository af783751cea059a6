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
// qb of the word) the table entry lives at byte
//     e*256 + (reg&1)*128 + 4*(8*gam + 4*(reg>>1) + qb)
// of the 64 KB table, i.e. in bank 8*gam + 4*(reg>>1) + qb.
//
// Lane mapping of the lookups.  Lane l = 4*rho + gam (rho = 0..7 picks one of 8
// rows of a step, gam = 0..3 one of four 16-byte word groups of the row).  At
// step (r, jj) the lane reads register r of its group (with the two halves of
// the group swapped when rho >= 4) and byte (jj + rho) % 4 of that word, so
// the 32 lanes touch 32 chunks in 32 different banks.  A single PRMT merges the
// sign byte (the entry index) with a per-lane constant into the address, so a
// lookup is PRMT + LDS + FADD.
//
// Work split.  A job (one matrix) is cut into units of 32 rows x one slice.
// The units of a phase are dealt to the CTAs in contiguous, equal ranges; a CTA
// rebuilds its table whenever its range enters a new (job, slice).  Partial
// row sums over a slice go to the fp32 output with red.global.add, so the
// V-contraction result t stays in L2 between the two phases.
//
// Phases are separated by a grid-wide wait (bounded spin); the kernel is
// launched cooperatively so that every CTA is resident.  At the start of each
// phase a CTA issues L2 prefetches for the sign rows it will read in the next
// phase, so HBM keeps streaming through the waits.
#include "lb_internal.cuh"

namespace lb {
namespace {

constexpr long long kSpinLimitCycles = 4000000000LL;   // ~2 s at 2 GHz
constexpr int kPrefetchSegments = 2048;                 // next-phase 64-byte segments per CTA
constexpr int kMaxTiles = 4;                            // tiles whose vectors are staged together

struct Smem {
    uint32_t lut;     // shared-window address of the 64 KB table
    uint32_t ring;    // per-warp rings of sign rowblocks (kRingSlots x 2 KB per warp)
    float* vec;       // staged vector slices (kMaxTiles of them), index e + e/32
    float* red;       // 32 floats of reduction scratch
    int* flag;        // one int
    LbPhase* phase;   // the current phase, copied from the plan
    LbJob* jobs;      // its jobs (at most kMaxPhaseJobs), copied from the plan
    uint32_t bars;    // per-warp ring mbarriers (kRingSlots per warp), shared address
};

__device__ __forceinline__ Smem smem_layout() {
    extern __shared__ __align__(16) unsigned char dsmem[];
    Smem s;
    s.lut = (uint32_t)__cvta_generic_to_shared(dsmem);
    s.ring = s.lut + kLutBytes;
    s.vec = reinterpret_cast<float*>(dsmem + kLutBytes + kRingBytes);
    s.red = s.vec + 4 * kVecPad;
    s.flag = reinterpret_cast<int*>(s.red + 32);
    s.phase = reinterpret_cast<LbPhase*>(dsmem + kLutBytes + kRingBytes + 4 * 4 * kVecPad + 4 * 32 + 64);
    s.jobs = reinterpret_cast<LbJob*>(reinterpret_cast<unsigned char*>(s.phase) + 64);
    s.bars = (uint32_t)__cvta_generic_to_shared(s.jobs + kMaxPhaseJobs);
    return s;
}

// Copy phase ph and its jobs into shared memory (plan data never changes
// during a call, so this can run before the grid-wide wait).
__device__ void cache_phase(const LbPhase* phases, int p, const LbJob* jobs, const Smem& sm) {
    const LbPhase ph = phases[p];
    if (threadIdx.x == 0) *sm.phase = ph;
    const int n_words = ph.n_jobs * (int)(sizeof(LbJob) / 4);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(jobs + ph.job_begin);
    uint32_t* dst = reinterpret_cast<uint32_t*>(sm.jobs);
    for (int i = threadIdx.x; i < n_words; i += kDecodeThreads) dst[i] = src[i];
}

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

// Local copy of a job with the call's x / y substituted for their tags.
__device__ __forceinline__ LbJob fetch_job(const LbJob* jobs, int j, const CallArgs& a) {
    LbJob J = jobs[j];
    J.src = resolve(J.src, a);
    J.out = resolve(J.out, a);
    J.resid_init = resolve(J.resid_init, a);
    return J;
}

// Grid-wide wait, split in two so a CTA can issue the next phase's loads and
// prefetches between announcing that it is done (grid_arrive) and waiting for
// everyone else (grid_wait).  The arrival is a release-add: every write of the
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

// First unit of CTA `cta` in phase ph: from the host's cost-balanced split
// table when there is one, else an even split of the units.
__device__ __forceinline__ int unit_split(const LbPhase& ph, const int* splits, int cta, int G) {
    if (ph.split_g == G) return splits[ph.split_off + cta];
    return (int)(((long long)ph.n_units * cta) / G);
}

// Element j of a job's vector source, before its scale: a is the source
// value (the gate for VK_SILU_MUL, whose up value goes to b).
__device__ __forceinline__ void load_src(const LbJob& J, int j, float& a, float& b) {
    switch (J.kind) {
        case VK_X_F16: a = __half2float(reinterpret_cast<const __half*>(J.src)[j]); break;
        case VK_X_BF16: a = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(J.src)[j]); break;
        case VK_X_F32:
        case VK_T: a = __ldcg(reinterpret_cast<const float*>(J.src) + j); break;
        case VK_GQA:
            a = __ldcg(reinterpret_cast<const float*>(J.src) + (j / J.gqa_ghd) * J.gqa_hd +
                       (j % J.gqa_hd));
            break;
        default:  // VK_SILU_MUL
            a = __ldcg(reinterpret_cast<const float*>(J.src) + j);
            b = __ldcg(J.src2 + j);
            break;
    }
}

// Build the 64 chunk tables of the staged slice.  Warp wp fills words with
// reg & 1 == wp & 1 and high nibbles (wp >> 1)*4 .. +3; lane = 8*gam + 4*h2 + qb
// owns chunk 4*(4*gam + 2*h2 + (wp&1)) + qb, which sits in bank `lane`.
__device__ void build_lut(const Smem& sm, const float* vec) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int gam = lane >> 3, h2 = (lane >> 2) & 1, qb = lane & 3;
    const int w = 4 * gam + 2 * h2 + (wp & 1);
    const int e0 = 32 * w + 8 * qb;                    // first element of the chunk
    const float* u = vec + e0 + (e0 >> 5);
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
    const uint32_t base = sm.lut + (uint32_t)(wp & 1) * 128u + (uint32_t)lane * 4u;
    constexpr int kNibPerWarp = 16 / (kDecodeWarps / 2);
    const int hb = (wp >> 1) * kNibPerWarp;
#pragma unroll
    for (int n = 0; n < kNibPerWarp; ++n) {
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

// L2 prefetch of the slice-s segment of one row (the one or two 128-byte
// lines it touches; plain prefetches go through the LSU, which issues them far
// faster than the bulk-copy engine would take one small request at a time).
__device__ __forceinline__ void prefetch_segment(const LbJob& J, int s, int row) {
    const int w0 = s * kSliceWords;
    if (row < J.rows && w0 < J.ldw) {
        const uint32_t* p = J.P + (size_t)row * (size_t)J.ldw + w0;
        const int nw = min(kSliceWords, J.ldw - w0);
        prefetch_l2(p);
        if ((reinterpret_cast<uintptr_t>(p) >> 7) != (reinterpret_cast<uintptr_t>(p + nw - 1) >> 7))
            prefetch_l2(p + nw - 1);
    }
}

// ---- per-warp ring of sign rowblocks, filled with cp.async ----------------
// Lane l = 4*rho + gam copies exactly the 16 bytes it later reads (words
// 4*gam .. 4*gam+3 of row 8*i + rho of the rowblock, i = 0..3) to
// ring + slot*2KB + i*512 + l*16, so no cross-lane synchronisation is needed:
// cp.async.wait_group on the lane's own groups is enough.  Bytes outside the
// matrix are zero-filled (source size 0).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t n) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src, uint32_t n) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" :: "r"(dst), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t n) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(dst), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory");
}

// Slot layout: 4 row-steps x 32 lanes x 16 bytes of signs, then 32 lanes x
// 4 bytes holding the fp16 row scale h of the lane's output row.
__device__ __forceinline__ uint32_t ring_slot(const Smem& sm, int slot) {
    return sm.ring + (uint32_t)((((threadIdx.x >> 5) * kRingSlots) + slot) * kRingSlotBytes) +
           (uint32_t)(threadIdx.x & 31) * 16u;
}
__device__ __forceinline__ uint32_t ring_hslot(uint32_t slot_lane_addr) {
    // slot base + 2048 + lane*4 (slot_lane_addr = slot base + lane*16)
    const uint32_t lane = threadIdx.x & 31;
    return slot_lane_addr - lane * 16u + (uint32_t)kRowBlockBytes + lane * 4u;
}

// Issue this lane's copies of rowblock rb (slice s) into the ring slot at dst.
// Lanes with rho >= 4 store the two 8-byte halves of their 16 bytes swapped,
// which is the order their lookups read them in.  The lane also copies the
// 4-byte word holding h[row] of its output row (second contraction only).
__device__ __forceinline__ void issue_rowblock(const LbJob& J, int s, int rb, uint32_t dst) {
    const int lane = threadIdx.x & 31;
    const int rho = lane >> 2, gam = lane & 3;
    const uint32_t sw = (rho >> 2) ? 8u : 0u;
    const int w = s * kSliceWords + 4 * gam;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = rb * kRowBlock + 8 * i + rho;
        const bool rok = row < J.rows;
        const uint32_t* p = rok ? J.P + (size_t)row * (size_t)J.ldw + w : J.P;
        const uint32_t d = dst + (uint32_t)i * 512u;
        if ((J.ldw & 1) == 0) {
            cp_async_8(d + sw, p, (rok && w < J.ldw) ? 8u : 0u);
            cp_async_8(d + (8u - sw), rok && w + 2 < J.ldw ? p + 2 : J.P,
                       (rok && w + 2 < J.ldw) ? 8u : 0u);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                cp_async_4(d + (((uint32_t)(4 * q) + sw) & 15u), rok && w + q < J.ldw ? p + q : J.P,
                           (rok && w + q < J.ldw) ? 4u : 0u);
        }
    }
    if (J.oscale != nullptr) {
        const int orow = rb * kRowBlock + 8 * gam + rho;
        const int h0 = orow & ~1;                        // h is 4-byte aligned (checked on entry)
        const uint32_t nb = orow >= J.rows ? 0u : (h0 + 1 < J.rows ? 4u : 2u);
        cp_async_4(ring_hslot(dst), nb ? J.oscale + h0 : J.oscale, nb);
    }
}

// ---- TMA-fed ring (rows with a 16-byte pitch) -----------------------------
// Lane 0 of a warp loads a whole rowblock (32 rows x 16 words, 2 KB) with one
// 2-D tensor copy into the warp's ring slot; the slot's mbarrier counts the
// bytes.  The box lands row-major, 64 bytes per row, which is the same layout
// the cp.async path writes (minus the half swap of rows 4..7 of each step).
// ring_it counts the rowblocks this warp has consumed so far in this launch;
// slot = it % kRingSlots, mbarrier phase parity = (it / kRingSlots) & 1.
__device__ __forceinline__ uint32_t ring_bar(const Smem& sm, uint32_t it) {
    return sm.bars + (uint32_t)(((threadIdx.x >> 5) * kRingSlots + (int)(it % kRingSlots)) * 8);
}
__device__ __forceinline__ uint32_t ring_slot_base(const Smem& sm, uint32_t it) {
    return sm.ring + (uint32_t)((((threadIdx.x >> 5) * kRingSlots) + (int)(it % kRingSlots)) *
                                kRingSlotBytes);
}
// Issue (lane 0) the TMA of rowblock rb of slice s as ring entry `it`.  The
// slot was last read by this warp: every lane has passed __syncwarp, and the
// proxy fence orders those reads before the tensor copy's writes.
__device__ __forceinline__ void tma_issue(const LbJob* Jg, int s, int rb, const Smem& sm,
                                          uint32_t it) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        fence_proxy_async_smem();
        const uint32_t bar = ring_bar(sm, it);
        mbar_expect_tx(bar, (uint32_t)kRowBlockBytes);
        tma_load_2d(ring_slot_base(sm, it), &Jg->tmap, bar, s * kSliceWords, rb * kRowBlock);
    }
}
// Bounded wait for ring entry `it`; on time-out records LB_ERR_TIMEOUT.
__device__ __forceinline__ void tma_wait(const Smem& sm, uint32_t it, int* err) {
    const uint32_t bar = ring_bar(sm, it), par = (it / kRingSlots) & 1u;
    if (mbar_try_wait(bar, par)) return;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, par)) {
        if (clock64() - t0 > kSpinLimitCycles) {
            atomicExch(err, (int)LB_ERR_TIMEOUT);
            return;
        }
    }
}

// Number of rowblocks warp wp takes in a tile of nrb rowblocks.
__device__ __forceinline__ int warp_rowblocks(int nrb) {
    const int wp = threadIdx.x >> 5;
    return wp < nrb ? (nrb - wp + kDecodeWarps - 1) / kDecodeWarps : 0;
}

// First kRingDepth rowblocks of this warp's share of a tile (issued before the
// tile's vector is staged, so the copies overlap staging and table build).
// The cp.async path always commits exactly kRingDepth groups.
__device__ __forceinline__ void ring_prologue(const LbJob& J, const LbJob* Jg, int s, int rb0,
                                              int nrb, const Smem& sm, uint32_t ring_it) {
    const int wp = threadIdx.x >> 5;
    const int nit = warp_rowblocks(nrb);
    if (J.use_tma) {
        for (int d = 0; d < kRingDepth && d < nit; ++d)
            tma_issue(Jg, s, rb0 + wp + d * kDecodeWarps, sm, ring_it + d);
        return;
    }
#pragma unroll
    for (int d = 0; d < kRingDepth; ++d) {
        if (d < nit) issue_rowblock(J, s, rb0 + wp + d * kDecodeWarps, ring_slot(sm, d));
        cp_async_commit();
    }
}

// Look up this warp's rowblocks of slice s of job J against the table; the
// rowblocks stream through the warp's ring kRingDepth ahead of use.  kBase is
// the table's shared-window address when it is the usual 1024 (then it folds
// into the load's immediate offset), else 0 and tbase is added at run time.
template <uint32_t kBase, bool kTma>
__device__ __forceinline__ void lookup_rowblocks(const LbJob& J, const LbJob* Jg, int s, int rb0,
                                                 int nrb, const Smem& sm, uint32_t& ring_it,
                                                 int* err) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int rho = lane >> 2, gam = lane & 3;
    const uint32_t swap = (uint32_t)(rho >> 2);
    uint32_t B[2][4], S[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        const uint32_t qbj = (uint32_t)((jj + rho) & 3);
        S[jj] = 0x7604u | (qbj << 4);                    // [B.b0, word.byte qbj, B.b2, B.b3]
#pragma unroll
        for (int rh = 0; rh < 2; ++rh)
            B[rh][jj] = (8u * (uint32_t)gam + 4u * ((uint32_t)rh ^ swap) + qbj) * 4u +
                        (kBase == 0 ? sm.lut : 0u);
    }
    const int nit = warp_rowblocks(nrb);
    const bool has_h = J.oscale != nullptr;
    for (int n = 0; n < nit; ++n) {
        const int rb = rb0 + wp + n * kDecodeWarps;
        uint32_t src;
        float hs_early = 1.0f;
        const int orow_e = rb * kRowBlock + 8 * gam + rho;
        if (kTma) {
            if (n + kRingDepth < nit)
                tma_issue(Jg, s, rb + kRingDepth * kDecodeWarps, sm, ring_it + n + kRingDepth);
            if (has_h && orow_e < J.rows) hs_early = __half2float(__ldg(J.oscale + orow_e));
            tma_wait(sm, ring_it + n, err);
            src = ring_slot_base(sm, ring_it + n) + (uint32_t)lane * 16u;
        } else {
            if (n + kRingDepth < nit)
                issue_rowblock(J, s, rb + kRingDepth * kDecodeWarps,
                               ring_slot(sm, (n + kRingDepth) % kRingSlots));
            cp_async_commit();
            cp_async_wait<kRingDepth>();                 // rowblock n has landed
            src = ring_slot(sm, n % kRingSlots);
        }
        float acc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t w4[4];
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                         : "r"(src + (uint32_t)i * 512u));
            if (kTma && swap) {                          // rows 4..7 read the halves swapped
                const uint32_t t0 = w4[0], t1 = w4[1];
                w4[0] = w4[2]; w4[1] = w4[3]; w4[2] = t0; w4[3] = t1;
            }
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint32_t addr = prmt(w4[r], B[r >> 1][jj], S[jj]) +
                                          (uint32_t)(r & 1) * 128u + kBase;
                    const float v = lds_f32(addr);
                    if (jj & 1) a1 += v; else a0 += v;
                }
            }
            acc[i] = a0 + a1;
        }
        const int orow = orow_e;                           // output row of this lane
        float hs = hs_early;
        if (!kTma && has_h) {
            uint32_t hw;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(hw) : "r"(ring_hslot(src)));
            const unsigned short hb = (unsigned short)((orow & 1) ? (hw >> 16) : (hw & 0xFFFFu));
            hs = __half2float(__ushort_as_half(hb));
        }
        // Transpose-reduce over the 4 lanes of a row (gam = lane bits 0-1):
        // afterwards lane gam holds the slice sum of row-step i = gam.
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
        const float tot = keep1 + __shfl_xor_sync(0xffffffffu, send1, 1);
        if (orow < J.rows) red_add_f32(J.out + orow, tot * hs);
    }
    if (kTma) ring_it += (uint32_t)nit;
    else cp_async_wait<0>();
}

__device__ __forceinline__ int find_job(const LbJob* jobs, int j, int j_end, int u) {
    while (j + 1 < j_end && jobs[j + 1].unit_begin <= u) ++j;
    return j;
}

struct Tile {
    int job, slice, rb0, nrb;
};

// Up to kMaxTiles tiles of this CTA's unit range, starting at unit u.
__device__ __forceinline__ int collect_tiles(const Smem& sm, int n_jobs, int& j, int u, int u_end,
                                             Tile (&t)[kMaxTiles]) {
    int n = 0;
    while (u < u_end && n < kMaxTiles) {
        j = find_job(sm.jobs, j, n_jobs, u);
        const LbJob& J = sm.jobs[j];
        const int local = u - J.unit_begin;
        const int s = local / J.n_rowblocks;
        const int rb0 = local - s * J.n_rowblocks;
        const int nrb = min(J.n_rowblocks - rb0, u_end - u);
        t[n++] = Tile{j, s, rb0, nrb};
        u += nrb;
    }
    return n;
}

// A batch of up to kMaxTiles tiles whose vectors are staged together.  sc[k]
// is this thread's element of tile k's vector scale (g or l), which does not
// depend on earlier phases and is loaded before the grid-wide wait.
struct Batch {
    int nt;
    Tile t[kMaxTiles];
    float sc[kMaxTiles];
};
static_assert(kSliceElems == kDecodeThreads, "one slice element per thread");

// This CTA's place in a phase: units [u, u_end), the job cursor, the batch
// about to run and how many TMA ring entries this warp has in flight for it.
struct Cursor {
    int u, u_end, j, in_flight;
    Batch b;
};

// Collect the next batch at c.u, start its first tile's rows streaming and
// load its scale elements.
__device__ void batch_begin(const Smem& sm, const CallArgs& args, const LbJob* jobs_g,
                            uint32_t ring_it, Cursor& c) {
    const LbPhase& ph = *sm.phase;
    Batch& b = c.b;
    b.nt = collect_tiles(sm, ph.n_jobs, c.j, c.u, c.u_end, b.t);
    const LbJob J0 = fetch_job(sm.jobs, b.t[0].job, args);
    ring_prologue(J0, jobs_g + ph.job_begin + b.t[0].job, b.t[0].slice, b.t[0].rb0, b.t[0].nrb,
                  sm, ring_it);
    c.in_flight = J0.use_tma ? min(kRingDepth, warp_rowblocks(b.t[0].nrb)) : 0;
#pragma unroll
    for (int k = 0; k < kMaxTiles; ++k) {
        b.sc[k] = 0.0f;
        if (k < b.nt) {
            const LbJob& J = sm.jobs[b.t[k].job];
            const int col = b.t[k].slice * kSliceElems + (int)threadIdx.x;
            if (col < J.cols) b.sc[k] = __half2float(__ldg(J.vscale + col));
        }
    }
}

// Stage the batch's vector slices into shared memory (zero past cols): all
// source loads are issued before any is used, so the batch costs one round
// trip to L2.  The owner of a slice (the CTA holding its first rowblock) also
// seeds the residual and adds the slice's sum of squares for RMSNorm; only
// the first job of a phase carries acc_sumsq, so there is one sum per batch.
__device__ void stage_batch(const Smem& sm, const CallArgs& args, const Batch& b) {
    const int e = threadIdx.x;
    float a[kMaxTiles], a2[kMaxTiles], nrm[kMaxTiles];
#pragma unroll
    for (int k = 0; k < kMaxTiles; ++k) {
        a[k] = 0.0f;
        a2[k] = 0.0f;
        nrm[k] = -1.0f;
        if (k < b.nt) {
            const LbJob J = fetch_job(sm.jobs, b.t[k].job, args);
            const int col = b.t[k].slice * kSliceElems + e;
            if (col < J.cols) load_src(J, col, a[k], a2[k]);
            if (J.kind == VK_T && J.norm_sumsq != nullptr) nrm[k] = __ldcg(J.norm_sumsq);
        }
    }
    float sq = 0.0f;
    float* acc = nullptr;
#pragma unroll
    for (int k = 0; k < kMaxTiles; ++k) {
        if (k >= b.nt) break;
        const LbJob J = fetch_job(sm.jobs, b.t[k].job, args);
        const int col = b.t[k].slice * kSliceElems + e;
        float v = 0.0f;
        if (col < J.cols) {
            const float raw = J.kind == VK_SILU_MUL ? silu(a[k]) * a2[k] : a[k];
            const float rs = nrm[k] >= 0.0f ? rsqrtf(nrm[k] / (float)J.norm_n + kRmsEps) : 1.0f;
            v = b.sc[k] * (raw * rs);
            if (b.t[k].rb0 == 0) {
                if (J.acc_sumsq != nullptr) sq += raw * raw;
                if (J.resid_init != nullptr) J.resid_init[col] = raw;
            }
        }
        if (b.t[k].rb0 == 0 && J.acc_sumsq != nullptr) acc = J.acc_sumsq;
        sm.vec[k * kVecPad + e + (e >> 5)] = v;
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

// The part of a phase that does not depend on earlier phases, run before the
// grid-wide wait: this CTA's unit range and its first batch (rows in flight,
// scales loaded).  sm.phase / sm.jobs must hold the phase.
__device__ void phase_begin(const Smem& sm, const CallArgs& args, const LbJob* jobs_g,
                            const int* splits, uint32_t ring_it, Cursor& c) {
    const LbPhase& ph = *sm.phase;
    c.u = unit_split(ph, splits, blockIdx.x, gridDim.x);
    c.u_end = unit_split(ph, splits, blockIdx.x + 1, gridDim.x);
    c.j = 0;
    c.in_flight = 0;
    c.b.nt = 0;
    if (c.u < c.u_end) batch_begin(sm, args, jobs_g, ring_it, c);
}

// Wait (bounded) for the ring entries a cursor has in flight, before leaving
// the kernel early: no copy may still be writing this CTA's shared memory.
__device__ void drain_ring(const Smem& sm, const Cursor& c, uint32_t ring_it, int* err) {
    for (int d = 0; d < c.in_flight; ++d) tma_wait(sm, ring_it + d, err);
    cp_async_wait<0>();
}

// The rest of the phase, after the grid-wide wait.
__device__ void run_phase(const Smem& sm, const CallArgs& args, const LbJob* jobs_g, Cursor& c,
                          uint32_t& ring_it, int* err) {
    const int G = gridDim.x, cta = blockIdx.x;
    const LbPhase ph = *sm.phase;
    float* zp = resolve(ph.zero_ptr, args);
    if (zp != nullptr) {
        for (int i = cta * kDecodeThreads + threadIdx.x; i < ph.zero_n; i += G * kDecodeThreads)
            zp[i] = 0.0f;
    }
    bool first = true;
    while (c.u < c.u_end) {
        if (!first) batch_begin(sm, args, jobs_g, ring_it, c);
        first = false;
        const Batch& b = c.b;
        stage_batch(sm, args, b);
        for (int k = 0; k < b.nt; ++k) {
            const LbJob J = fetch_job(sm.jobs, b.t[k].job, args);
            const LbJob* Jg = jobs_g + ph.job_begin + b.t[k].job;
            if (k > 0) ring_prologue(J, Jg, b.t[k].slice, b.t[k].rb0, b.t[k].nrb, sm, ring_it);
            build_lut(sm, sm.vec + k * kVecPad);
            const bool b1024 = sm.lut == 1024u;
            if (J.use_tma) {
                if (b1024) lookup_rowblocks<1024u, true>(J, Jg, b.t[k].slice, b.t[k].rb0, b.t[k].nrb, sm, ring_it, err);
                else lookup_rowblocks<0u, true>(J, Jg, b.t[k].slice, b.t[k].rb0, b.t[k].nrb, sm, ring_it, err);
            } else {
                if (b1024) lookup_rowblocks<1024u, false>(J, Jg, b.t[k].slice, b.t[k].rb0, b.t[k].nrb, sm, ring_it, err);
                else lookup_rowblocks<0u, false>(J, Jg, b.t[k].slice, b.t[k].rb0, b.t[k].nrb, sm, ring_it, err);
            }
            __syncthreads();
            c.u += b.t[k].nrb;
        }
    }
    c.in_flight = 0;
}

// L2 prefetch of the sign segments this CTA will read in phase ph (up to
// kPrefetchSegments of them, in the order it will read them).
__device__ void prefetch_phase(const LbPhase& ph, const LbJob* jobs, const int* splits) {
    const int G = gridDim.x, cta = blockIdx.x;
    int u = unit_split(ph, splits, cta, G);
    const int u_end = unit_split(ph, splits, cta + 1, G);
    int j = ph.job_begin;
    const int j_end = ph.job_begin + ph.n_jobs;
    int budget = kPrefetchSegments;
    while (u < u_end && budget > 0) {
        j = find_job(jobs, j, j_end, u);
        const LbJob& J = jobs[j];
        const int local = u - J.unit_begin;
        const int s = local / J.n_rowblocks;
        const int rb0 = local - s * J.n_rowblocks;
        const int nrb = min(J.n_rowblocks - rb0, u_end - u);
        const int rows = min(nrb * kRowBlock, budget);
        for (int i = threadIdx.x; i < rows; i += kDecodeThreads)
            prefetch_segment(J, s, rb0 * kRowBlock + i);
        // the scales this tile will read: its slice of g or l, its rows of h
        const int t = threadIdx.x - (kDecodeThreads - 32);          // last warp
        if (t >= 0) {
            const int c0 = s * kSliceElems, c1 = min(J.cols, c0 + kSliceElems);
            if (t < 8 && c0 + 64 * t < c1) prefetch_l2(J.vscale + c0 + 64 * t);
            if (J.oscale != nullptr) {
                const int r0 = rb0 * kRowBlock, r1 = min(J.rows, (rb0 + nrb) * kRowBlock);
                for (int r = r0 + 64 * (t - 8); t >= 8 && r < r1; r += 64 * 24)
                    prefetch_l2(J.oscale + r);
            }
        }
        budget -= rows;
        u += nrb;
    }
}

__device__ void run_program(const LbPhase* phases, int n_phases, const LbJob* jobs,
                            const int* splits, WsHeader* hdr, const CallArgs& args) {
    const Smem sm = smem_layout();
    const unsigned G = gridDim.x;
    if (*reinterpret_cast<volatile int*>(&hdr->error) != 0) return;   // sticky after a timeout
    if (threadIdx.x < kDecodeWarps * kRingSlots) mbar_init(sm.bars + 8u * threadIdx.x, 1u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    cache_phase(phases, 0, jobs, sm);
    __syncthreads();
    uint32_t ring_it = 0;
    Cursor cur;
    phase_begin(sm, args, jobs, splits, ring_it, cur);
    prefetch_phase(phases[0], jobs, splits);
    for (int p = 0; p < n_phases; ++p) {
        run_phase(sm, args, jobs, cur, ring_it, &hdr->error);
        if (p + 1 < n_phases) {
            // Announce completion, then use the wait: bring in the next
            // phase's plan, start its first rows streaming into the ring and
            // prefetch the rest of this CTA's rows to L2.
            grid_arrive(hdr);
            cache_phase(phases, p + 1, jobs, sm);
            __syncthreads();
            phase_begin(sm, args, jobs, splits, ring_it, cur);
            prefetch_phase(phases[p + 1], jobs, splits);
            if (!grid_wait(hdr, (unsigned)(p + 1) * G, sm.flag)) {
                drain_ring(sm, cur, ring_it, &hdr->error);
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
    run_program(plan.phases, n_phases, plan.jobs, plan.split, hdr, args);
}

__global__ void __launch_bounds__(kDecodeThreads, kCtasPerSm)
stack_program_kernel(const LbPhase* __restrict__ phases, const LbJob* __restrict__ jobs,
                     const int* __restrict__ splits, int n_phases, WsHeader* hdr, const void* x,
                     float* y) {
    const CallArgs args = {x, y};
    run_program(phases, n_phases, jobs, splits, hdr, args);
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

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_sign_tmap(CUtensorMap* map, const uint32_t* P, int rows, int ldw) {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    if (!fn || rows <= 0 || ldw <= 0 || (ldw & 3) != 0) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)ldw, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ldw * 4};
    const cuuint32_t box[2] = {(cuuint32_t)kSliceWords, (cuuint32_t)kRowBlock};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(P), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

int decode_grid() { return device_sm_count() * kCtasPerSm; }

// Contiguous unit ranges for G CTAs with the smallest largest cost.  The
// warps of a CTA take a tile's rowblocks kDecodeWarps at a time, so a CTA
// that takes k rowblocks of a tile spends ceil(k / kDecodeWarps) warp
// iterations on them, plus kTileCost (in 1/kDecodeWarps iterations) to stage
// the tile's vector and build its tables.  Units run job by job, slice-major
// inside a job, so a phase is a list of tiles of n_rowblocks units each; a
// greedy fill is optimal for a given bound, which a bisection minimises.
namespace {
template <class F>
void for_each_tile(const LbJob* jobs, int n_jobs, F f) {
    for (int j = 0; j < n_jobs; ++j)
        for (int s = 0; s < jobs[j].n_slices; ++s) f(jobs[j].n_rowblocks);
}
long long take_cost(long long k) {
    return kTileCost + (k + kDecodeWarps - 1) / kDecodeWarps * kDecodeWarps;
}
// CTAs a greedy fill under cost bound T needs; boundaries go to `out` if set.
int greedy_fill(const LbJob* jobs, int n_jobs, long long T, int* out) {
    int used = 1, u = 0;
    long long cost = 0;
    for_each_tile(jobs, n_jobs, [&](int n) {
        while (n > 0) {
            if (cost + take_cost(1) > T) {
                if (out) out[used] = u;
                ++used;
                cost = 0;
            }
            const long long room = (T - cost - kTileCost) / kDecodeWarps * kDecodeWarps;
            const int take = (int)std::min<long long>(n, room);
            cost += take_cost(take);
            n -= take;
            u += take;
        }
    });
    return used;
}
}  // namespace

void balanced_split(const LbJob* jobs, int n_jobs, int n_units, int G, int* out) {
    long long lo = take_cost(1), hi = lo;
    for_each_tile(jobs, n_jobs, [&](int n) { hi += take_cost(n); });
    while (lo < hi) {   // smallest bound a fill of at most G CTAs meets
        const long long mid = (lo + hi) / 2;
        if (greedy_fill(jobs, n_jobs, mid, nullptr) <= G) hi = mid;
        else lo = mid + 1;
    }
    const int used = greedy_fill(jobs, n_jobs, lo, out);
    out[0] = 0;
    for (int c = used; c <= G; ++c) out[c] = n_units;
}

cudaError_t decode_configure() {
    cudaError_t e = cudaFuncSetAttribute(linear_program_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kDecodeSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(stack_program_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDecodeSmem);
    if (e != cudaSuccess) return e;
    for (const void* fn : {reinterpret_cast<const void*>(linear_program_kernel),
                           reinterpret_cast<const void*>(stack_program_kernel)}) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
    }
    for (const void* fn : {reinterpret_cast<const void*>(linear_program_kernel),
                           reinterpret_cast<const void*>(stack_program_kernel)}) {
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
                              int n_phases, WsHeader* hdr, const void* x, float* y,
                              cudaStream_t s) {
    void* args[] = {&phases, &jobs, &splits, &n_phases, &hdr, &x, &y};
    return launch_coop(reinterpret_cast<const void*>(stack_program_kernel), args, s);
}

}  // namespace lb
