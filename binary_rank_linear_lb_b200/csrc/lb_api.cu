// Host side of liblb.so: argument validation, workspace layout, plan building
// and launches for every entry point declared in include/lb.h.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "lb_internal.cuh"

namespace lb {

namespace {

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
int g_sm_count[kMaxDevices];
int g_cc_major[kMaxDevices];
cudaError_t g_cfg_err[kMaxDevices];

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

void init_device(int d) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, d) != cudaSuccess) {
        g_cfg_err[d] = cudaErrorInvalidDevice;
        return;
    }
    g_sm_count[d] = prop.multiProcessorCount;
    g_cc_major[d] = prop.major;
    g_cfg_err[d] = prop.major == 10 ? decode_configure() : cudaErrorInvalidDeviceFunction;
    if (g_cfg_err[d] == cudaSuccess) g_cfg_err[d] = prefill_configure();
}

// Returns LB_OK when the current device is an sm_100 part and the kernels are configured.
lb_status ensure_device() {
    const int d = current_device();
    if (d < 0 || d >= kMaxDevices) return LB_ERR_CUDA;
    std::call_once(g_dev_once[d], init_device, d);
    if (g_cc_major[d] != 10) return LB_ERR_UNSUPPORTED;
    return g_cfg_err[d] == cudaSuccess ? LB_OK : LB_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int vec_kind_for(lb_dtype t) {
    switch (t) {
        case LB_F16: return VK_X_F16;
        case LB_BF16: return VK_X_BF16;
        default: return VK_X_F32;
    }
}

// Fill the size fields of a job whose matrix has `rows` packed rows of `cols`
// signs with a pitch of `ld` words (0: unpadded), and its TMA descriptor when
// the pitch allows one (16-byte rows).
void set_job_shape(LbJob& J, int64_t rows, int64_t cols, int64_t ld, int layout) {
    J.rows = (int)rows;
    J.cols = (int)cols;
    J.sliced = layout == LB_LAYOUT_SLICES ? 1 : 0;
    J.ldw = J.sliced ? kSliceWords : (int)(ld ? ld : cdiv(cols, 32));
    J.n_slices = (int)cdiv(cols, kSliceElems);
    J.n_rowblocks = (int)cdiv(rows, kRowBlock);
    J.rg = J.n_rowblocks;
}

bool ld_ok(int64_t ld, int64_t k) { return ld == 0 || (ld >= cdiv(k, 32) && ld <= (1 << 26)); }

// Give each phase a cost-balanced split of its units over G CTAs, written to
// `split` (kMaxGrid+1 ints per phase); phases keep the even split if G does
// not fit the table.
void plan_splits(LbPhase* phases, int n_phases, LbJob* jobs, int G, int* split,
                 bool search = false) {
    for (int p = 0; p < n_phases; ++p) {
        phases[p].next_job_begin = p + 1 < n_phases ? phases[p + 1].job_begin : 0;
        phases[p].next_n_jobs = p + 1 < n_phases ? phases[p + 1].n_jobs : 0;
        phases[p].split_off = p * (kMaxGrid + 1);
        phases[p].split_g = -1;
        phases[p].starts_g = -1;   // no start table unless plan_starts makes one
        plan_row_groups(jobs + phases[p].job_begin, phases[p].n_jobs, phases[p].n_units,
                        std::max(G, 1), search);
        if (G < 1 || G > kMaxGrid) continue;
        balanced_split(jobs + phases[p].job_begin, phases[p].n_jobs, phases[p].n_units, G,
                       split + phases[p].split_off);
        phases[p].split_g = G;
    }
}

// Append `J` to phase `ph`, assigning its unit range.
void add_job(LbPhase& ph, std::vector<LbJob>& jobs, LbJob J) {
    J.unit_begin = ph.n_units;
    ph.n_units += J.n_slices * J.n_rowblocks;
    ph.n_jobs += 1;
    jobs.push_back(J);
}

bool branch_ok(const lb_branch& b) {
    if (!(b.Vp && b.Up && b.h && b.g && b.l && b.ld_v >= 0 && b.ld_u >= 0)) return false;
    if (b.layout == LB_LAYOUT_SLICES) return b.ld_v == 0 && b.ld_u == 0;
    return b.layout == LB_LAYOUT_ROWS;
}
bool branch_aligned(const lb_branch& b) {
    return aligned(b.Vp, 16) && aligned(b.Up, 16) && aligned(b.h, 4) && aligned(b.g, 2) &&
           aligned(b.l, 2);
}

// ------------------------------------------------------------ stack layout
// Accumulators are laid out phase by phase: region p holds everything phase p
// accumulates into (t of its first contractions, outputs of its second
// contractions, the RMSNorm sum of squares).  The kernel zeroes region p+1
// during phase p and region 0 during the last phase, so a call leaves the
// workspace ready for the next one; lb_stack_prepare zeroes it once.
struct StackLayout {
    std::vector<size_t> sumsq_off;   // [layer][2] (attention norm, MLP norm)
    std::vector<size_t> t_off;       // [layer][proj][branch]
    std::vector<size_t> o_off;       // [layer][proj] outputs of q,k,v,gate,up (else 0)
    std::vector<size_t> region_off;  // [phase] first byte of the phase's region
    std::vector<size_t> region_len;  // [phase] bytes (0: nothing, or y for MLP-only)
    size_t acc_end;                  // end of the accumulator area
    size_t x_dev, y_dev;             // staging for lb_stack_forward_host
    size_t phases, jobs, splits;     // plan
    size_t starts;                   // [phase][kMaxGrid] first batches of the CTAs
    int n_phases, n_jobs;
    size_t total;
};

// in / out features of projection p.
void proj_shape(const lb_stack_desc* d, int p, int64_t& in, int64_t& out) {
    const int64_t kv = (int64_t)d->n_kv_heads * d->head_dim;
    switch (p) {
        case LB_Q: in = d->hidden; out = d->hidden; break;
        case LB_K: case LB_V: in = d->hidden; out = kv; break;
        case LB_O: in = d->hidden; out = d->hidden; break;
        case LB_GATE: case LB_UP: in = d->hidden; out = d->inter; break;
        default: in = d->inter; out = d->hidden; break;
    }
}

bool stack_desc_ok(const lb_stack_desc* d) {
    if (!d || !d->lin || !d->ranks) return false;
    if (d->n_layers <= 0 || d->hidden <= 0 || d->inter <= 0) return false;
    if (d->n_layers > 4096 || d->hidden > (1 << 24) || d->inter > (1 << 24)) return false;
    if (d->n_branches < 1 || d->n_branches > 2) return false;
    const bool mlp_only = (d->flags & LB_STACK_MLP_ONLY) != 0;
    if (d->flags & ~LB_STACK_MLP_ONLY) return false;
    if (mlp_only) {
        if (d->n_layers != 1) return false;
    } else {
        if (d->n_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0) return false;
        if ((int64_t)d->n_heads * d->head_dim != d->hidden) return false;
        if (d->n_heads % d->n_kv_heads != 0) return false;
    }
    for (int L = 0; L < d->n_layers; ++L)
        for (int p = 0; p < LB_N_PROJ; ++p) {
            const bool used = !mlp_only || p >= LB_GATE;
            if (!used) continue;
            if (d->ranks[L * LB_N_PROJ + p] <= 0 || d->ranks[L * LB_N_PROJ + p] > (1 << 24))
                return false;
            int64_t in, out;
            proj_shape(d, p, in, out);
            const int64_t r = d->ranks[L * LB_N_PROJ + p];
            for (int b = 0; b < d->n_branches; ++b) {
                const lb_branch& B = d->lin[(L * LB_N_PROJ + p) * d->n_branches + b];
                if (!branch_ok(B) || !ld_ok(B.ld_v, in) || !ld_ok(B.ld_u, r)) return false;
            }
        }
    return true;
}

bool proj_used(const lb_stack_desc* d, int p) {
    return !(d->flags & LB_STACK_MLP_ONLY) || p >= LB_GATE;
}

// The phases of one decoder layer (or of the MLP-only block): which
// projections each phase covers and whether it is the first contraction.
struct PhaseSpec {
    int projs[3];
    int n_projs;
    bool first;      // first contraction (writes t) or second (writes outputs)
    int norm;        // -1, or which RMSNorm sum of squares (0 attention, 1 MLP)
};

std::vector<PhaseSpec> layer_phases(bool mlp_only) {
    if (mlp_only)
        return {{{LB_GATE, LB_UP, 0}, 2, true, -1}, {{LB_GATE, LB_UP, 0}, 2, false, -1},
                {{LB_DOWN, 0, 0}, 1, true, -1}, {{LB_DOWN, 0, 0}, 1, false, -1}};
    return {{{LB_Q, LB_K, LB_V}, 3, true, 0}, {{LB_Q, LB_K, LB_V}, 3, false, 0},
            {{LB_O, 0, 0}, 1, true, -1},      {{LB_O, 0, 0}, 1, false, -1},
            {{LB_GATE, LB_UP, 0}, 2, true, 1}, {{LB_GATE, LB_UP, 0}, 2, false, 1},
            {{LB_DOWN, 0, 0}, 1, true, -1},   {{LB_DOWN, 0, 0}, 1, false, -1}};
}

StackLayout stack_layout(const lb_stack_desc* d) {
    StackLayout L;
    const int nl = d->n_layers, nb = d->n_branches;
    const bool mlp_only = (d->flags & LB_STACK_MLP_ONLY) != 0;
    const std::vector<PhaseSpec> spec = layer_phases(mlp_only);
    L.sumsq_off.assign((size_t)nl * 2, 0);
    L.t_off.assign((size_t)nl * LB_N_PROJ * nb, 0);
    L.o_off.assign((size_t)nl * LB_N_PROJ, 0);
    size_t off = sizeof(WsHeader);
    for (int l = 0; l < nl; ++l)
        for (const PhaseSpec& ps : spec) {
            const size_t begin = off;
            if (ps.first && ps.norm >= 0) {
                L.sumsq_off[(size_t)l * 2 + ps.norm] = off;
                off += 256;
            }
            for (int i = 0; i < ps.n_projs; ++i) {
                const int p = ps.projs[i];
                if (ps.first) {
                    const int64_t r = d->ranks[l * LB_N_PROJ + p];
                    for (int b = 0; b < nb; ++b) {
                        L.t_off[((size_t)l * LB_N_PROJ + p) * nb + b] = off;
                        off = round_up(off + sizeof(float) * (size_t)r, 256);
                    }
                } else if (p != LB_O && p != LB_DOWN) {
                    int64_t in, out;
                    proj_shape(d, p, in, out);
                    L.o_off[(size_t)l * LB_N_PROJ + p] = off;
                    off = round_up(off + sizeof(float) * (size_t)out, 256);
                }
            }
            L.region_off.push_back(begin);
            L.region_len.push_back(off - begin);
        }
    L.acc_end = off;
    L.x_dev = off;
    off = round_up(off + 2 * (size_t)d->hidden, 256);
    L.y_dev = off;
    off = round_up(off + 4 * (size_t)d->hidden, 256);
    L.n_phases = (int)spec.size() * nl;
    // jobs: one per projection and branch in each of the two contractions
    int per_layer = 0;
    for (const PhaseSpec& ps : spec) per_layer += ps.n_projs * nb;
    L.n_jobs = per_layer * nl;
    L.phases = off;
    off = round_up(off + sizeof(LbPhase) * (size_t)L.n_phases, 256);
    L.jobs = off;
    off = round_up(off + sizeof(LbJob) * (size_t)L.n_jobs, 256);
    L.splits = off;
    off = round_up(off + sizeof(int) * (size_t)(kMaxGrid + 1) * (size_t)L.n_phases, 256);
    L.starts = off;
    off = round_up(off + sizeof(LbStart) * (size_t)kMaxGrid * (size_t)L.n_phases, 256);
    L.total = off;
    return L;
}

// Build the phase program of a stack (host copies; pointers into `ws`).
void build_stack_plan(const lb_stack_desc* d, const StackLayout& L, char* ws,
                      std::vector<LbPhase>& phases, std::vector<LbJob>& jobs) {
    const int nb = d->n_branches;
    const bool mlp_only = (d->flags & LB_STACK_MLP_ONLY) != 0;
    const std::vector<PhaseSpec> spec = layer_phases(mlp_only);
    auto br = [&](int l, int p, int b) -> const lb_branch& {
        return d->lin[((size_t)l * LB_N_PROJ + p) * nb + b];
    };
    auto at = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
    auto tptr = [&](int l, int p, int b) {
        return at(L.t_off[((size_t)l * LB_N_PROJ + p) * nb + b]);
    };
    auto optr = [&](int l, int p) { return at(L.o_off[(size_t)l * LB_N_PROJ + p]); };
    float* yres = const_cast<float*>(reinterpret_cast<const float*>(LB_TAG_Y));
    const int gqa_group = (!mlp_only && d->n_kv_heads > 0) ? d->n_heads / d->n_kv_heads : 1;

    for (int l = 0; l < d->n_layers; ++l) {
        for (const PhaseSpec& ps : spec) {
            LbPhase ph = {};
            ph.job_begin = (int)jobs.size();
            float* norm = ps.norm >= 0 ? at(L.sumsq_off[(size_t)l * 2 + ps.norm]) : nullptr;
            bool first_job = true;
            for (int i = 0; i < ps.n_projs; ++i) {
                const int p = ps.projs[i];
                int64_t in, out;
                proj_shape(d, p, in, out);
                const int64_t r = d->ranks[l * LB_N_PROJ + p];
                for (int b = 0; b < nb; ++b) {
                    LbJob J = {};
                    if (ps.first) {
                        J.P = br(l, p, b).Vp;
                        set_job_shape(J, r, in, br(l, p, b).ld_v, br(l, p, b).layout);
                        J.vscale = reinterpret_cast<const __half*>(br(l, p, b).g);
                        J.out = tptr(l, p, b);
                        if (p == LB_O) {
                            J.kind = VK_GQA;
                            J.src = optr(l, LB_V);
                            J.gqa_hd = d->head_dim;
                            J.gqa_ghd = d->head_dim * gqa_group;
                        } else if (p == LB_DOWN) {
                            J.kind = VK_SILU_MUL;
                            J.src = optr(l, LB_GATE);
                            J.src2 = optr(l, LB_UP);
                        } else if (mlp_only || (l == 0 && p <= LB_V)) {
                            // the call's bf16 input; layer 0's q/k/v also seed the residual
                            J.kind = VK_X_BF16;
                            J.src = LB_TAG_X;
                            if (!mlp_only && first_job && p == LB_Q) J.resid_init = yres;
                        } else {
                            J.kind = VK_X_F32;
                            J.src = LB_TAG_Y;
                        }
                        if (first_job && norm) J.acc_sumsq = norm;
                    } else {
                        J.P = br(l, p, b).Up;
                        set_job_shape(J, out, r, br(l, p, b).ld_u, br(l, p, b).layout);
                        J.kind = VK_T;
                        J.src = tptr(l, p, b);
                        J.vscale = reinterpret_cast<const __half*>(br(l, p, b).l);
                        J.oscale = reinterpret_cast<const __half*>(br(l, p, b).h);
                        J.out = (p == LB_O || p == LB_DOWN) ? yres : optr(l, p);
                        J.norm_sumsq = norm;
                        J.norm_n = d->hidden;
                    }
                    first_job = false;
                    add_job(ph, jobs, J);
                }
            }
            phases.push_back(ph);
        }
    }
    // Phase p zeroes the region of phase p+1; the last phase zeroes region 0
    // for the next call.  The MLP-only block's final phase accumulates into y.
    const int n = (int)phases.size();
    for (int p = 0; p < n; ++p) {
        const int q = (p + 1) % n;
        if (mlp_only && q == n - 1) {
            phases[p].zero_ptr = yres;
            phases[p].zero_n = d->hidden;
        } else if (L.region_len[q] > 0) {
            phases[p].zero_ptr = at(L.region_off[q]);
            phases[p].zero_n = (int)(L.region_len[q] / sizeof(float));
        }
    }
}

}  // namespace

int device_sm_count() {
    const int d = current_device();
    return (d >= 0 && d < kMaxDevices) ? g_sm_count[d] : 0;
}

bool device_is_sm100() {
    const int d = current_device();
    return d >= 0 && d < kMaxDevices && g_cc_major[d] == 10;
}

}  // namespace lb

using namespace lb;

extern "C" {

const char* lb_status_string(lb_status s) {
    switch (s) {
        case LB_OK: return "LB_OK";
        case LB_ERR_INVALID_ARG: return "LB_ERR_INVALID_ARG";
        case LB_ERR_ALIGNMENT: return "LB_ERR_ALIGNMENT";
        case LB_ERR_UNSUPPORTED: return "LB_ERR_UNSUPPORTED";
        case LB_ERR_CUDA: return "LB_ERR_CUDA";
        case LB_ERR_TIMEOUT: return "LB_ERR_TIMEOUT";
        case LB_ERR_WORKSPACE: return "LB_ERR_WORKSPACE";
        default: return "LB_ERR_UNKNOWN";
    }
}

int lb_version(void) { return 100; }

lb_status lb_pack_signs(const float* latent, int64_t rows, int64_t cols, int64_t ld, int axis,
                        uint32_t* packed, int64_t ld_words, void* stream) {
    if (!latent || !packed || rows <= 0 || cols <= 0 || ld < cols) return LB_ERR_INVALID_ARG;
    if (axis != 0 && axis != 1) return LB_ERR_INVALID_ARG;
    const int64_t k = axis == 1 ? cols : rows;
    if (ld_words < cdiv(k, 32)) return LB_ERR_INVALID_ARG;
    if (!aligned(latent, 4) || !aligned(packed, 4)) return LB_ERR_ALIGNMENT;
    const lb_status st = ensure_device();
    if (st != LB_OK) return st;
    return launch_pack(latent, rows, cols, ld, axis, packed, ld_words, false,
                       static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? LB_OK
               : LB_ERR_CUDA;
}

size_t lb_packed_words(int64_t n, int64_t k, int layout, int64_t ld_words) {
    if (n <= 0 || k <= 0 || n > ((int64_t)1 << 40) || k > ((int64_t)1 << 40)) return 0;
    const int64_t nw = cdiv(k, 32);
    if (layout == LB_LAYOUT_SLICES) return (size_t)sliced_words(n, nw);
    if (layout != LB_LAYOUT_ROWS || (ld_words != 0 && ld_words < nw)) return 0;
    return (size_t)(n * (ld_words ? ld_words : nw));
}

lb_status lb_pack_signs_sliced(const float* latent, int64_t rows, int64_t cols, int64_t ld,
                               int axis, uint32_t* packed, void* stream) {
    if (!latent || !packed || rows <= 0 || cols <= 0 || ld < cols) return LB_ERR_INVALID_ARG;
    if (axis != 0 && axis != 1) return LB_ERR_INVALID_ARG;
    if (!aligned(latent, 4) || !aligned(packed, 16)) return LB_ERR_ALIGNMENT;
    const lb_status st = ensure_device();
    if (st != LB_OK) return st;
    return launch_pack(latent, rows, cols, ld, axis, packed, 0, true,
                       static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? LB_OK
               : LB_ERR_CUDA;
}

}  // extern "C"

// LB_LINEAR_PATH=0|1 in the environment (read on every call) forces the
// lookup-table (0) or the tensor-core (1) kernels wherever the shapes allow
// them, for measuring the two paths against each other.
static int forced_path() {
    const char* env = std::getenv("LB_LINEAR_PATH");
    if (env == nullptr || env[1] != 0) return -1;
    return env[0] == '0' ? 0 : env[0] == '1' ? 1 : -1;
}

// The tensor-core path runs for at least kPrefillMinM rows when the shapes
// allow its 64-wide K blocks.
static bool use_prefill(int64_t M, int64_t in, int64_t out, int64_t r) {
    const int f = forced_path();
    if (f >= 0) return f == 1 && prefill_shape_ok(M, in, out, r);
    return M >= kPrefillMinM && prefill_shape_ok(M, in, out, r);
}

namespace lb {

size_t decode_workspace_bytes(int64_t M, int64_t r, int n_branches) {
    const int64_t mc = std::min<int64_t>(M, kMaxDecodeM);
    return sizeof(WsHeader) + round_up(sizeof(float) * (size_t)(mc * n_branches * r), 256);
}

LinearRoute default_route(int64_t M, int64_t in, int64_t out, int64_t r, const lb_branch* br,
                          int n_branches) {
    if (!br || n_branches < 1 || n_branches > 2 || !use_prefill(M, in, out, r))
        return kRouteDecode;
    // the tensor-core path reads g in 16-byte vectors and sign words in pairs
    for (int b = 0; b < n_branches; ++b)
        if (!(aligned(br[b].g, 16) &&
              (br[b].layout == LB_LAYOUT_SLICES ||
               (((br[b].ld_v ? br[b].ld_v : cdiv(in, 32)) & 1) == 0 &&
                ((br[b].ld_u ? br[b].ld_u : cdiv(r, 32)) & 1) == 0))))
            return kRouteDecode;
    return kRoutePrefill;
}

size_t route_workspace_bytes(LinearRoute route, int64_t M, int64_t in, int64_t r, int nb) {
    if (route == kRouteDecode) return decode_workspace_bytes(M, r, nb);
    return prefill_workspace_bytes(M, in, r, route == kRoutePrefill);
}

lb_status linear_forward_route(const void* x, lb_dtype x_dtype, int64_t M, int64_t in,
                               int64_t out, int64_t r, const lb_branch* br, int n_branches,
                               float* y, void* workspace, size_t ws_bytes, size_t ws_need,
                               cudaStream_t s, LinearRoute route) {
    if (!x || !y || !br || !workspace) return LB_ERR_INVALID_ARG;
    if (M <= 0 || in <= 0 || out <= 0 || r <= 0) return LB_ERR_INVALID_ARG;
    if (in > (1 << 28) || out > (1 << 28) || r > (1 << 24)) return LB_ERR_INVALID_ARG;
    if (n_branches < 1 || n_branches > 2) return LB_ERR_INVALID_ARG;
    if (x_dtype != LB_F16 && x_dtype != LB_BF16 && x_dtype != LB_F32) return LB_ERR_INVALID_ARG;
    for (int b = 0; b < n_branches; ++b)
        if (!branch_ok(br[b]) || !ld_ok(br[b].ld_v, in) || !ld_ok(br[b].ld_u, r))
            return LB_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(workspace, 16)) return LB_ERR_ALIGNMENT;
    for (int b = 0; b < n_branches; ++b)
        if (!branch_aligned(br[b])) return LB_ERR_ALIGNMENT;
    if (route != kRouteDecode && default_route(M, in, out, r, br, n_branches) == kRouteDecode)
        return LB_ERR_INVALID_ARG;   // the tensor-core path cannot take these shapes or pointers
    if (ws_bytes < ws_need || ws_bytes < route_workspace_bytes(route, M, in, r, n_branches))
        return LB_ERR_WORKSPACE;
    lb_status st = ensure_device();
    if (st != LB_OK) return st;

    if (route != kRouteDecode)
        return launch_prefill(x, vec_kind_for(x_dtype), M, in, out, r, br, n_branches, y,
                              workspace, s, route == kRoutePrefill) == cudaSuccess
                   ? LB_OK
                   : LB_ERR_CUDA;
    if ((int64_t)std::min<int64_t>(M, kMaxDecodeM) * out > 0x7fffffff) return LB_ERR_INVALID_ARG;
    const size_t xsz = x_dtype == LB_F32 ? 4 : 2;
    WsHeader* hdr = static_cast<WsHeader*>(workspace);
    float* t = reinterpret_cast<float*>(static_cast<char*>(workspace) + sizeof(WsHeader));
    // The header (barrier counter, error) is cleared once per call, together
    // with the first chunk's t accumulators (they follow it), so a device-side
    // time-out in one chunk of rows stays visible after the later chunks (which
    // then return at once); the kernel leaves the barrier counter at zero when
    // it finishes.  Later chunks clear only their t accumulators.
    for (int64_t m0 = 0; m0 < M; m0 += kMaxDecodeM) {
        const int mc = (int)std::min<int64_t>(kMaxDecodeM, M - m0);
        LinearPlan plan;
        std::memset(&plan, 0, sizeof(plan));
        std::vector<LbJob> jobs;
        jobs.reserve(2 * kMaxLinearJobs);
        LbPhase p0 = {};
        p0.job_begin = 0;
        for (int m = 0; m < mc; ++m)
            for (int b = 0; b < n_branches; ++b) {
                LbJob J = {};
                J.P = br[b].Vp;
                set_job_shape(J, r, in, br[b].ld_v, br[b].layout);
                J.kind = vec_kind_for(x_dtype);
                J.src = static_cast<const char*>(x) + (size_t)(m0 + m) * (size_t)in * xsz;
                J.vscale = reinterpret_cast<const __half*>(br[b].g);
                J.out = t + ((size_t)m * n_branches + b) * (size_t)r;
                add_job(p0, jobs, J);
            }
        p0.zero_ptr = y + (size_t)m0 * (size_t)out;
        p0.zero_n = (int)(mc * out);
        LbPhase p1 = {};
        p1.job_begin = (int)jobs.size();
        for (int m = 0; m < mc; ++m)
            for (int b = 0; b < n_branches; ++b) {
                LbJob J = {};
                J.P = br[b].Up;
                set_job_shape(J, out, r, br[b].ld_u, br[b].layout);
                J.kind = VK_T;
                J.src = t + ((size_t)m * n_branches + b) * (size_t)r;
                J.vscale = reinterpret_cast<const __half*>(br[b].l);
                J.oscale = reinterpret_cast<const __half*>(br[b].h);
                J.out = y + (size_t)(m0 + m) * (size_t)out;
                add_job(p1, jobs, J);
            }
        plan.phases[0] = p0;
        plan.phases[1] = p1;
        std::copy(jobs.begin(), jobs.end(), plan.jobs);
        plan_splits(plan.phases, 2, plan.jobs, decode_grid(), plan.split);
        const size_t t_bytes = sizeof(float) * (size_t)mc * n_branches * r;
        if ((m0 == 0 ? cudaMemsetAsync(hdr, 0, sizeof(WsHeader) + t_bytes, s)
                     : cudaMemsetAsync(t, 0, t_bytes, s)) != cudaSuccess)
            return LB_ERR_CUDA;
        if (launch_linear_plan(plan, hdr, 2, s) != cudaSuccess) return LB_ERR_CUDA;
    }
    return LB_OK;
}

}  // namespace lb

extern "C" {

size_t lb_linear_workspace_size(int64_t M, int64_t in, int64_t out, int64_t r, int n_branches) {
    if (M <= 0 || in <= 0 || out <= 0 || r <= 0 || n_branches < 1 || n_branches > 2) return 0;
    if (use_prefill(M, in, out, r)) return prefill_workspace_bytes(M, in, r);
    return decode_workspace_bytes(M, r, n_branches);
}

int lb_linear_path(int64_t M, int64_t in, int64_t out, int64_t r) {
    return use_prefill(M, in, out, r) ? 1 : 0;
}

lb_status lb_linear_forward(const void* x, lb_dtype x_dtype, int64_t M, int64_t in, int64_t out,
                            int64_t r, const lb_branch* br, int n_branches, float* y,
                            void* workspace, size_t ws_bytes, void* stream) {
    return linear_forward_route(x, x_dtype, M, in, out, r, br, n_branches, y, workspace, ws_bytes,
                                lb_linear_workspace_size(M, in, out, r, n_branches),
                                static_cast<cudaStream_t>(stream),
                                default_route(M, in, out, r, br, n_branches));
}

size_t lb_stack_workspace_size(const lb_stack_desc* d) {
    if (!stack_desc_ok(d)) return 0;
    return stack_layout(d).total;
}

namespace {
// Validation shared by the plan builders: descriptor, workspace pointer and
// size, branch alignment.
lb_status stack_plan_args(const lb_stack_desc* d, const void* workspace, size_t ws_bytes,
                          StackLayout& L) {
    if (!stack_desc_ok(d) || !workspace) return LB_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return LB_ERR_ALIGNMENT;
    const int nb = d->n_branches;
    for (int l = 0; l < d->n_layers; ++l)
        for (int p = 0; p < LB_N_PROJ; ++p) {
            if (!proj_used(d, p)) continue;
            for (int b = 0; b < nb; ++b)
                if (!branch_aligned(d->lin[((size_t)l * LB_N_PROJ + p) * nb + b]))
                    return LB_ERR_ALIGNMENT;
        }
    L = stack_layout(d);
    if (ws_bytes < L.total) return LB_ERR_WORKSPACE;
    return LB_OK;
}

// The stack's execution plan for a grid of G CTAs, its pointers into the
// workspace at address ws (host copies; nothing is dereferenced).
struct StackPlan {
    std::vector<LbPhase> phases;
    std::vector<LbJob> jobs;
    std::vector<int> split;
    std::vector<LbStart> starts;
};
bool make_stack_plan(const lb_stack_desc* d, const StackLayout& L, char* ws, int G,
                     StackPlan& P) {
    build_stack_plan(d, L, ws, P.phases, P.jobs);
    if ((int)P.phases.size() != L.n_phases || (int)P.jobs.size() != L.n_jobs) return false;
    P.split.assign((size_t)(kMaxGrid + 1) * L.n_phases, 0);
    plan_splits(P.phases.data(), L.n_phases, P.jobs.data(), G, P.split.data(), true);
    P.starts.assign((size_t)kMaxGrid * L.n_phases, LbStart{});
    plan_starts(P.phases.data(), L.n_phases, P.jobs.data(), P.split.data(), G, P.starts.data());
    return true;
}
}  // namespace

lb_status lb_stack_prepare(const lb_stack_desc* d, void* workspace, size_t ws_bytes,
                           void* stream) {
    StackLayout L;
    lb_status st = stack_plan_args(d, workspace, ws_bytes, L);
    if (st != LB_OK) return st;
    if ((st = ensure_device()) != LB_OK) return st;
    char* ws = static_cast<char*>(workspace);
    StackPlan P;
    if (!make_stack_plan(d, L, ws, decode_grid(), P)) return LB_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, L.acc_end, s) != cudaSuccess) return LB_ERR_CUDA;
    if (cudaMemcpyAsync(ws + L.phases, P.phases.data(), sizeof(LbPhase) * P.phases.size(),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
        return LB_ERR_CUDA;
    if (cudaMemcpyAsync(ws + L.jobs, P.jobs.data(), sizeof(LbJob) * P.jobs.size(),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
        return LB_ERR_CUDA;
    if (cudaMemcpyAsync(ws + L.splits, P.split.data(), sizeof(int) * P.split.size(),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
        return LB_ERR_CUDA;
    if (cudaMemcpyAsync(ws + L.starts, P.starts.data(), sizeof(LbStart) * P.starts.size(),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
        return LB_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LB_ERR_CUDA;
    return LB_OK;
}

lb_status lb_stack_plan_host(const lb_stack_desc* d, int grid, void* image, size_t image_bytes,
                             size_t* offsets, int* counts) {
    StackLayout L;
    const lb_status st = stack_plan_args(d, image, image_bytes, L);
    if (st != LB_OK) return st;
    if (grid < 1 || !offsets || !counts) return LB_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(image);
    StackPlan P;
    if (!make_stack_plan(d, L, ws, grid, P)) return LB_ERR_INVALID_ARG;
    std::memset(ws, 0, L.total);
    std::memcpy(ws + L.phases, P.phases.data(), sizeof(LbPhase) * P.phases.size());
    std::memcpy(ws + L.jobs, P.jobs.data(), sizeof(LbJob) * P.jobs.size());
    std::memcpy(ws + L.splits, P.split.data(), sizeof(int) * P.split.size());
    std::memcpy(ws + L.starts, P.starts.data(), sizeof(LbStart) * P.starts.size());
    offsets[0] = L.phases;
    offsets[1] = L.jobs;
    offsets[2] = L.splits;
    offsets[3] = L.starts;
    offsets[4] = L.acc_end;
    counts[0] = L.n_phases;
    counts[1] = L.n_jobs;
    counts[2] = kMaxGrid;
    counts[3] = (int)sizeof(LbPhase);
    counts[4] = (int)sizeof(LbJob);
    counts[5] = (int)sizeof(LbStart);
    return LB_OK;
}

lb_status lb_stack_forward(const lb_stack_desc* d, void* workspace, size_t ws_bytes,
                           const void* x, float* y, void* stream) {
    if (!stack_desc_ok(d) || !workspace || !x || !y) return LB_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(x, 16) || !aligned(y, 16)) return LB_ERR_ALIGNMENT;
    const StackLayout L = stack_layout(d);
    if (ws_bytes < L.total) return LB_ERR_WORKSPACE;
    lb_status st = ensure_device();
    if (st != LB_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    if (launch_stack_plan(reinterpret_cast<const LbPhase*>(ws + L.phases),
                          reinterpret_cast<const LbJob*>(ws + L.jobs),
                          reinterpret_cast<const int*>(ws + L.splits),
                          reinterpret_cast<const LbStart*>(ws + L.starts), L.n_phases,
                          reinterpret_cast<WsHeader*>(ws), x, y, s) != cudaSuccess)
        return LB_ERR_CUDA;
    return LB_OK;
}

lb_status lb_stack_forward_host(const lb_stack_desc* d, void* workspace, size_t ws_bytes,
                                const void* x_host, float* y_host, void* stream) {
    if (!stack_desc_ok(d) || !workspace || !x_host || !y_host) return LB_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return LB_ERR_ALIGNMENT;
    const StackLayout L = stack_layout(d);
    if (ws_bytes < L.total) return LB_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    void* xd = ws + L.x_dev;
    float* yd = reinterpret_cast<float*>(ws + L.y_dev);
    if (cudaMemcpyAsync(xd, x_host, 2 * (size_t)d->hidden, cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
        return LB_ERR_CUDA;
    lb_status st = lb_stack_forward(d, workspace, ws_bytes, xd, yd, stream);
    if (st != LB_OK) return st;
    if (cudaMemcpyAsync(y_host, yd, 4 * (size_t)d->hidden, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return LB_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LB_ERR_CUDA;
    return LB_OK;
}

lb_status lb_workspace_status(const void* workspace, void* stream) {
    if (!workspace) return LB_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return LB_ERR_CUDA;
    int err = 0;
    if (cudaMemcpy(&err, &static_cast<const WsHeader*>(workspace)->error, sizeof(int),
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return LB_ERR_CUDA;
    return err == 0 ? LB_OK : LB_ERR_TIMEOUT;
}

const float* lb_stack_output(const lb_stack_desc* d, const void* workspace, int layer, int proj) {
    if (!stack_desc_ok(d) || !workspace) return nullptr;
    if (layer < 0 || layer >= d->n_layers || proj < 0 || proj >= LB_N_PROJ) return nullptr;
    if (!proj_used(d, proj) || proj == LB_O || proj == LB_DOWN) return nullptr;
    const StackLayout L = stack_layout(d);
    return reinterpret_cast<const float*>(static_cast<const char*>(workspace) +
                                          L.o_off[(size_t)layer * LB_N_PROJ + proj]);
}

}  // extern "C"
