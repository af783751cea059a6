/*
 * lb.h — C ABI of liblb.so, a B200 (sm_100a) implementation of the inference
 * forward of the LittleBit factorised binary linear layer.
 *
 * The layer ("Samsung LittleBit: A 13B LLM Under 1 GB, and What the Paper
 * Really Shows", section "How it works", items 1-3):
 *
 *   y = sum_{b in {primary, residual}} h_b o ( sign(U_b) . ( l_b o ( sign(V_b)^T . ( g_b o x ) ) ) )
 *
 *   U_b : out x r and V_b : in x r are latent factors of which only the signs
 *         are kept at inference (item 1: "uses only their signs, +1 or -1");
 *   h_b (out), g_b (in), l_b (r) are FP16 scale vectors along the rows, the
 *         columns and the latent dimension of W (item 2);
 *   b runs over a primary and a residual branch whose outputs are summed
 *         (item 3, and the figure of the two-branch layer beside it).
 *   sign(v) = -1 for v < 0 and +1 otherwise, so sign(0) = sign(-0.0) = +1 and a
 *   NaN latent packs as +1.
 *
 * Packed sign format.  A packed row of K signs is ceil(K/32) (or ld_words >=
 * that) little-endian uint32 words; bit (e % 32) of word (e / 32) is 1 exactly
 * when element e is negative (sign -1).  Bits past K are written as 0 by
 * lb_pack_signs and ignored by every forward.  V_b is stored packed along the
 * input dimension (Vp_b[r][ld_v], ld_v >= ceil(in/32)) and U_b packed along the
 * latent dimension (Up_b[out][ld_u], ld_u >= ceil(r/32)).
 *
 * Conventions for every entry point.
 *   - The caller owns all memory.  Device pointers are CUDA device (or managed)
 *     addresses on the current device; host pointers are ordinary host memory.
 *     No forward call allocates device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are stream-ordered and asynchronous unless stated otherwise.
 *   - Argument errors are reported synchronously by the return value, before
 *     anything is launched.  Launch failures return LB_ERR_CUDA.  Faults that
 *     happen later on the device surface at the caller's next synchronisation.
 *   - Matrices are row-major.  x is M x in, y is M x out.
 *   - The library is thread-safe.  On the host it caches per-device properties;
 *     on the device it keeps no state between calls, except the fixed scratch
 *     array of lb_linear_forward_noalloc (see there).
 */
#ifndef LB_H
#define LB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LB_OK = 0,
    LB_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad enum      */
    LB_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte aligned                */
    LB_ERR_UNSUPPORTED = 3,   /* valid but not supported (e.g. no sm_100 device) */
    LB_ERR_CUDA = 4,          /* a CUDA runtime call failed                      */
    LB_ERR_TIMEOUT = 5,       /* a device-side wait gave up (lb_workspace_status) */
    LB_ERR_WORKSPACE = 6      /* workspace missing or smaller than required      */
} lb_status;

typedef enum { LB_F16 = 0, LB_BF16 = 1, LB_F32 = 2 } lb_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
const char *lb_status_string(lb_status s);

/* Library version as major*10000 + minor*100 + patch. */
int lb_version(void);

/*
 * lb_pack_signs — binarise an fp32 latent factor into packed sign words.
 * Defines the "signs only at inference" step (item 1 of "How it works").
 *
 *   latent   : device, rows x cols fp32, row stride ld elements (ld >= cols)
 *   axis = 1 : every row is packed along its columns
 *              -> packed[rows][ld_words], ld_words >= ceil(cols/32)   (U: out x r)
 *   axis = 0 : every column is packed along the rows
 *              -> packed[cols][ld_words], ld_words >= ceil(rows/32)   (V: in x r)
 *   packed   : device, written in full (padding bits and padding words are 0)
 *   bit = 1 exactly when the latent element is < 0.0f (so -0.0 and NaN give 0).
 * Errors: LB_ERR_INVALID_ARG for null pointers, rows/cols <= 0, ld < cols,
 * ld_words too small or axis not in {0, 1}; LB_ERR_ALIGNMENT if latent or
 * packed is not 4-byte aligned.
 */
lb_status lb_pack_signs(const float *latent, int64_t rows, int64_t cols, int64_t ld,
                        int axis, uint32_t *packed, int64_t ld_words, void *stream);

/*
 * Layouts of a packed matrix of n rows of K signs (nw = ceil(K/32) words each).
 *
 *   LB_LAYOUT_ROWS   : row-major, [n][ld] words (ld >= nw), as written by
 *                      lb_pack_signs.  The canonical layout.
 *   LB_LAYOUT_SLICES : the same words regrouped by 512-sign slice, as written
 *                      by lb_pack_signs_sliced.  Slice s (words 16s .. 16s+15
 *                      of every row) is a block of n rows starting at word
 *                      16*n*s; full slices have a pitch of 16 words (64 bytes),
 *                      the last slice the words it holds rounded up to a
 *                      multiple of 4.  Padding words are 0.
 *
 * Both hold the same bits.  The decode kernels read one 512-sign slice of many
 * rows at a time: in the sliced layout that is one contiguous block, which
 * DRAM streams at close to full bandwidth, whereas row-major rows give one
 * 64-byte piece per row and DRAM about half of it.  Prefer LB_LAYOUT_SLICES
 * for weights that are read by the batch-1 path.
 */
typedef enum { LB_LAYOUT_ROWS = 0, LB_LAYOUT_SLICES = 1 } lb_layout;

/* Words a packed matrix of n rows of K signs occupies in `layout`
 * (LB_LAYOUT_ROWS: n * max(ld_words, ceil(K/32))); 0 for bad arguments. */
size_t lb_packed_words(int64_t n, int64_t k, int layout, int64_t ld_words);

/*
 * lb_pack_signs_sliced — lb_pack_signs writing LB_LAYOUT_SLICES: the packed
 * matrix has n = rows (axis 1) or n = cols (axis 0) rows of K = cols (axis 1)
 * or K = rows (axis 0) signs, and `packed` receives lb_packed_words(n, K,
 * LB_LAYOUT_SLICES, 0) words.  Same errors as lb_pack_signs, and
 * LB_ERR_ALIGNMENT unless packed is 16-byte aligned.
 */
lb_status lb_pack_signs_sliced(const float *latent, int64_t rows, int64_t cols, int64_t ld,
                               int axis, uint32_t *packed, void *stream);

/* One branch of a factorised layer (device pointers, row pitches, layout).
 * ld_v / ld_u are the words per packed row of Vp / Up in LB_LAYOUT_ROWS (0
 * means the unpadded ceil(in/32) / ceil(r/32)); with LB_LAYOUT_SLICES they
 * must be 0.  In LB_LAYOUT_ROWS, a pitch that is a multiple of 16 words (64
 * bytes) keeps every slice of every row one aligned DRAM piece.  Padding words
 * are never read.  A zero-initialised `layout` means LB_LAYOUT_ROWS. */
typedef struct {
    const uint32_t *Vp;   /* signs of V_b: r rows of in signs (packed along in)   */
    const uint32_t *Up;   /* signs of U_b: out rows of r signs (packed along r)    */
    const uint16_t *h;    /* [out] FP16 row scale (IEEE binary16 bits), 4-byte aligned */
    const uint16_t *g;    /* [in]  FP16 column scale                         */
    const uint16_t *l;    /* [r]   FP16 latent scale                         */
    int64_t ld_v;         /* words per packed row of Vp, 0 or >= ceil(in/32) */
    int64_t ld_u;         /* words per packed row of Up, 0 or >= ceil(r/32)  */
    int32_t layout;       /* lb_layout of Vp and Up                          */
    int32_t reserved;     /* 0                                               */
} lb_branch;

/*
 * lb_linear_forward — y = the layer applied to the M rows of x (formula above).
 *
 *   x         : device, M x in, dtype x_dtype (LB_F16, LB_BF16 or LB_F32)
 *   br        : host array of n_branches (1 or 2) lb_branch; every branch shares
 *               in, out and r (each branch has its own row pitches)
 *   y         : device, M x out fp32, overwritten
 *   workspace : device scratch of at least lb_linear_workspace_size(...) bytes,
 *               16-byte aligned; contents need not be initialised and are
 *               clobbered.  Concurrent calls need distinct workspaces.
 * Small M runs the lookup-table decode kernels; large M runs the tcgen05
 * tensor-core kernels.  Both accumulate in fp32.
 * Errors: LB_ERR_INVALID_ARG (null pointer, M/in/out/r <= 0, n_branches not 1
 * or 2, bad dtype), LB_ERR_ALIGNMENT (x, y, workspace or a packed pointer not
 * 16-byte aligned, h not 4-byte aligned, g or l not 2-byte aligned),
 * LB_ERR_WORKSPACE, LB_ERR_UNSUPPORTED (no sm_100 device), LB_ERR_CUDA.
 * (The tensor-core path also reads g in 16-byte vectors; a g that is not
 * 16-byte aligned keeps the call on the lookup-table kernels.)
 * The tensor-core path splits either GEMM along K when its tiles would leave
 * SMs idle (small M or low rank); two environment variables, read on every
 * call, fix its choices for testing, with results equal up to rounding:
 * LB_PREFILL_SUBTILES=1|2 (128-row M sub-tiles per expanded sign tile) and
 * LB_PREFILL_SPLIT2=1..4 (K parts of a second-GEMM tile, at most one per 64
 * columns of K).  LB_LINEAR_PATH=0|1, also read on every call (and by
 * lb_linear_workspace_size and lb_linear_path), forces the lookup-table (0) or
 * the tensor-core (1) kernels wherever the shapes allow them, so that the two
 * can be timed against each other; both give the layer within the same bound.
 */
lb_status lb_linear_forward(const void *x, lb_dtype x_dtype, int64_t M, int64_t in,
                            int64_t out, int64_t r, const lb_branch *br, int n_branches,
                            float *y, void *workspace, size_t ws_bytes, void *stream);

size_t lb_linear_workspace_size(int64_t M, int64_t in, int64_t out, int64_t r,
                                int n_branches);

/*
 * lb_linear_forward_noalloc — lb_linear_forward for callers that cannot
 * allocate device memory (code running under another framework's allocator,
 * plugins in a process whose device pool is already taken, real-time paths
 * where an allocation may block or fail).  The pages have no counterpart to
 * this entry point; it only moves the scratch.
 *
 * Same arguments and results as lb_linear_forward, without `workspace`: the
 * scratch lives in a fixed __device__ array of lb_noalloc_scratch_bytes()
 * bytes (256 KiB) inside liblb.so, which every GPU that loads the library holds
 * until the process exits.  Limits, with S = lb_noalloc_scratch_bytes():
 *   - where lb_linear_forward takes the tensor-core path, this call takes it
 *     too if 256 + pad(2*M*in) + pad(4*M*r) + pad(8*M) + 256 + pad(4*ceil(M/128))
 *     <= S (pad = round up to 256 bytes), running stage 1 without its K split
 *     (e.g. M = 17, in = 4096, r = 1472 fits; M = 64, in = 4096 does not);
 *   - otherwise it takes the lookup-table path, which needs
 *     256 + pad(4 * min(M, 8) * n_branches * r) <= S (two branches: r up to
 *     32736 for M = 1, up to 4092 for M >= 8);
 *   - beyond both it returns LB_ERR_WORKSPACE.
 * Both paths give the layer's result within the same fp32 accuracy.
 * A call on a device looks up the array's device address until one lookup
 * succeeds; make the first call on each device before any stream capture.
 * All calls share the array and it keeps the last call's contents; each call
 * clears what must start at zero, and calls that overlap on the GPU (streams
 * not ordered with each other) race on it.  It never calls cudaMalloc,
 * cudaFree or any allocating routine.  A device-side wait that gives up
 * (about 2 s) leaves y undefined; the array's status word is not exposed, so
 * callers that must detect that case should use lb_linear_forward and
 * lb_workspace_status.
 */
lb_status lb_linear_forward_noalloc(const void *x, lb_dtype x_dtype, int64_t M, int64_t in,
                                    int64_t out, int64_t r, const lb_branch *br,
                                    int n_branches, float *y, void *stream);

/*
 * lb_linear_forward_xor — the bit-serial variant of the layer ("The XOR
 * claim" on the same page: with both operands signs, a multiply becomes an
 * XOR plus a popcount).  Each activation vector v (g_b o x, then l_b o t) is
 * quantised to `bits`-bit fixed point in a code whose bit-planes are signs:
 *   D = 2^e, the smallest (e >= -100) with max|v| <= (2^bits - 1) D;
 *   q_j = 2 floor(v_j / 2D) + 1  (odd, |D q_j - v_j| <= D);
 *   q_j = sum_p 2^p sigma_jp with sigma_jp in {-1, +1},
 * and every contraction sum_j s_j q_j = sum_p 2^p (n - 2 popc(s XOR plane_p))
 * is computed exactly in integers on 32-bit words.  The result:
 *   t'_k = fp32(l_k * fp32(D1 * T_k)),  y_i = sum_b h_bi * D2_b * Z_bi  (fp32).
 * With bits = 16 the quantisation error is about 1e-4 of max|y|.
 *   x, br, M, in, out, r, n_branches, y : as lb_linear_forward (any layout,
 *                     packed pointers 4-byte aligned, scales 2-byte aligned)
 *   bits      : 1 .. 24 bit-planes per activation
 *   workspace : device, >= lb_linear_xor_workspace_size(...) bytes, 16-byte
 *               aligned, clobbered.
 * Four kernel launches on `stream`.  Errors: LB_ERR_INVALID_ARG,
 * LB_ERR_ALIGNMENT, LB_ERR_WORKSPACE, LB_ERR_UNSUPPORTED, LB_ERR_CUDA.
 * It is the reference form of the claim, not the fast path: on this GPU the
 * lookup-table kernels of lb_linear_forward need fewer instructions per sign.
 */
lb_status lb_linear_forward_xor(const void *x, lb_dtype x_dtype, int64_t M, int64_t in,
                                int64_t out, int64_t r, const lb_branch *br, int n_branches,
                                int bits, float *y, void *workspace, size_t ws_bytes,
                                void *stream);
size_t lb_linear_xor_workspace_size(int64_t M, int64_t in, int64_t out, int64_t r,
                                    int n_branches, int bits);

/*
 * lb_dual_svid — initialise the branches of a factorised layer from a dense
 * weight ("How it works", item 3: Dual-SVID starts from a truncated SVD of the
 * real weights, maps signs and magnitudes onto the binary factors and the
 * scales, and fits a residual branch to what the first one missed).  Per
 * branch, on the residual R (W for the first):
 *   R ~ U S V^T (rank r; cuSOLVER's randomized truncated SVD),
 *   U' = U S^(1/2), V' = V S^(1/2);  Up, Vp = packed signs of U', V';
 *   |U'| ~ h l_u^T, |V'| ~ g l_v^T (rank-1 fits), h and g scaled to mean 1,
 *   l = l_u o l_v, all rounded to fp16;
 *   R <- R - diag(h) sign(U') diag(l) sign(V')^T diag(g) (from the stored values).
 *   W        : device, out x in fp32 row-major, 16-byte aligned, not modified
 *   r        : 1 .. min(out, in);  n_branches: 1 or 2;  layout: lb_layout of the outputs
 *   Vp[b], Up[b] : device, lb_packed_words(r, in, layout, 0) and
 *              lb_packed_words(out, r, layout, 0) words, 16-byte aligned, written
 *   h[b], g[b], l[b] : device fp16 [out], [in], [r], written
 *   workspace : device, >= lb_dual_svid_workspace_size(...) bytes, 256-byte aligned
 * Synchronous (returns when the branches are written).  It is an offline step:
 * it creates its own cuSOLVER and cuBLAS handles for the call (their internal
 * state is allocated by those libraries).  The SVD is defined up to the signs of
 * its singular-vector pairs, which flip a column of sign(U') and of sign(V')
 * together and leave the branch unchanged.  Errors: LB_ERR_INVALID_ARG,
 * LB_ERR_ALIGNMENT, LB_ERR_WORKSPACE, LB_ERR_UNSUPPORTED, LB_ERR_CUDA (also when
 * the SVD reports a failure).
 */
lb_status lb_dual_svid(const float *W, int64_t out, int64_t in, int64_t r, int n_branches,
                       int layout, uint32_t *const *Vp, uint32_t *const *Up, uint16_t *const *h,
                       uint16_t *const *g, uint16_t *const *l, void *workspace, size_t ws_bytes,
                       void *stream);
size_t lb_dual_svid_workspace_size(int64_t out, int64_t in, int64_t r, int n_branches);

/* Size in bytes of the fixed scratch array used by lb_linear_forward_noalloc. */
size_t lb_noalloc_scratch_bytes(void);

/* Which kernels lb_linear_forward uses for M rows: 0 = decode, 1 = tensor core. */
int lb_linear_path(int64_t M, int64_t in, int64_t out, int64_t r);

/*
 * Decoder stacks.  A stack runs, for one token (batch 1), the linears of
 * n_layers Llama-2-shaped decoder layers and the glue between them:
 *
 *   a = rmsnorm(h) (weightless, eps 1e-5); q,k,v = L_q(a), L_k(a), L_v(a);
 *   attn = v broadcast over the query heads of its key/value group (attention
 *   over one position); h += L_o(attn); a = rmsnorm(h);
 *   h += L_down(silu(L_gate(a)) * L_up(a)).
 *
 * With LB_STACK_MLP_ONLY each layer is y = L_down(silu(L_gate(x)) * L_up(x))
 * (no attention, norm or residual; n_layers must be 1).
 * Activations between linears are fp32; the input is bf16 and the output fp32.
 * The pages describe the layer only: this glue is the plainest decoder around it.
 */
enum { LB_Q = 0, LB_K = 1, LB_V = 2, LB_O = 3, LB_GATE = 4, LB_UP = 5, LB_DOWN = 6,
       LB_N_PROJ = 7 };
enum { LB_STACK_MLP_ONLY = 1 };

typedef struct {
    int n_layers, hidden, inter, n_heads, n_kv_heads, head_dim, n_branches, flags;
    const lb_branch *lin;   /* host array [n_layers][LB_N_PROJ][n_branches]       */
    const int64_t *ranks;   /* host array [n_layers][LB_N_PROJ] latent rank r     */
} lb_stack_desc;

/* Bytes of device workspace a stack needs (header, accumulators, plan). */
size_t lb_stack_workspace_size(const lb_stack_desc *d);

/*
 * lb_stack_prepare — validate the descriptor and write the stack's execution
 * plan into `workspace` (device, 256-byte aligned, >= lb_stack_workspace_size).
 * Synchronous: returns after the plan is on the device.  The plan stays valid
 * while the weights stay where they are; pass the same descriptor and
 * workspace to every lb_stack_forward of that stack.
 * Errors: LB_ERR_INVALID_ARG (null pointer, non-positive or inconsistent
 * sizes: n_heads*head_dim must equal hidden, n_heads a multiple of n_kv_heads,
 * every rank > 0, MLP_ONLY with n_layers != 1), LB_ERR_ALIGNMENT,
 * LB_ERR_WORKSPACE, LB_ERR_UNSUPPORTED, LB_ERR_CUDA.
 */
lb_status lb_stack_prepare(const lb_stack_desc *d, void *workspace, size_t ws_bytes,
                           void *stream);

/*
 * lb_stack_plan_host — for inspection and tests, on the host only (no CUDA
 * call): the plan lb_stack_prepare would write for a grid of `grid` CTAs,
 * written into the host buffer `image` (256-byte aligned, >= the stack's
 * workspace size) at its workspace offsets, its workspace pointers taken
 * relative to `image` itself; the rest of the image is zero.  The packed
 * factors and scales are not read.
 *   offsets[5] : byte offsets of the phase headers, jobs, split table, start
 *                table, and the end of the accumulator region
 *   counts[6]  : phases, jobs, the split/start table stride in CTAs, and the
 *                sizes in bytes of a phase header, a job and a start record
 * Same argument errors as lb_stack_prepare (grid < 1: LB_ERR_INVALID_ARG).
 */
lb_status lb_stack_plan_host(const lb_stack_desc *d, int grid, void *image, size_t image_bytes,
                             size_t *offsets, int *counts);

/*
 * lb_stack_forward — one token through a prepared stack.
 *   x : device bf16 [hidden];  y : device fp32 [hidden], overwritten.
 * One cooperative persistent kernel on `stream` (it zeroes each phase's
 * accumulators itself, one phase ahead).  Grid-wide waits inside the kernel
 * are bounded (about 2 s); if one gives up, the kernel returns early, y is
 * undefined and lb_workspace_status reports LB_ERR_TIMEOUT.  The error is
 * sticky: later calls on the workspace return at once, until lb_stack_prepare
 * runs on it again.
 */
lb_status lb_stack_forward(const lb_stack_desc *d, void *workspace, size_t ws_bytes,
                           const void *x, float *y, void *stream);

/*
 * lb_stack_forward_host — the same through host buffers: copies x (host bf16)
 * to the device, runs the stack, copies y (host fp32) back and synchronises
 * `stream`.  The device-side x and y live in the workspace.  Pinned host
 * memory gives asynchronous copies; pageable memory also works.
 */
lb_status lb_stack_forward_host(const lb_stack_desc *d, void *workspace, size_t ws_bytes,
                                const void *x_host, float *y_host, void *stream);

/* Synchronises `stream`, then reports whether the last stack or linear call
 * that used `workspace` finished its device-side waits: LB_OK or LB_ERR_TIMEOUT. */
lb_status lb_workspace_status(const void *workspace, void *stream);

/* Device fp32 output of linear `proj` (LB_Q ... LB_DOWN) of layer `layer` from
 * the last lb_stack_forward on this workspace (read it after the stream is
 * synchronised), or NULL for LB_O and LB_DOWN (those add straight into the
 * residual stream) and for bad arguments.  Lets callers check the q and k
 * projections, which feed nothing else in the stack. */
const float *lb_stack_output(const lb_stack_desc *d, const void *workspace, int layer,
                             int proj);

#ifdef __cplusplus
}
#endif
#endif /* LB_H */
