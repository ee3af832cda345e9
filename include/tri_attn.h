/*
 * tri_attn.h -- C ABI of the B200 (sm_100a) triangle-attention library
 * (libtriattn.so).  Plain pointers and sizes only; no framework types.
 *
 * What it computes.  Triangle attention around the starting node of an
 * AlphaFold3 / OpenFold3 Pairformer pair tensor: for batch b, pair row i,
 * head h and query j,
 *
 *   out[b,i,j,h,:] = sum_k softmax_k( scale * q[b,i,j,h,:].k[b,i,k,h,:]
 *                                     + bias[b,h,j,k] + mask[b,i,k] ) v[b,i,k,h,:]
 *
 * with ONE pair bias shared by all N rows i, so the work is cubic in the crop
 * size N and the bias gradient is a reduction over rows.  Pages this follows:
 *   (A) "16张H100，训练步提速1.73倍：TurboPairFormer为什么不是'装个包就能加速AlphaFold3'"
 *       (biocloudservice.com), sections "先看清'1.73倍'对应什么" (cubic cost) and
 *       "它优化了什么，而不是只'少存一点张量'" (the four gradients and the shared
 *       pair bias; the BF16 output-rounding residual with an FP32 correction);
 *   (B) "TurboPairFormer: более быстрое, стабильное и точное дообучение OpenFold3"
 *       (dev48.org), section "Как работает TurboPairFormer" (probabilities
 *       recomputed in the backward, residual compensation, fixed accumulation
 *       order giving bitwise-identical gradients).
 *
 * Ending-node orientation is the same operation on the transposed pair
 * tensor: pass every 5-D tensor (inputs AND outputs) with stride[1] and
 * stride[2] swapped.  bias and mask are always given in the attention's own
 * frame ((j,k) and (i,k)); the caller builds them from the transposed pair
 * representation, as AlphaFold does.
 *
 * Conventions (every entry point):
 *  - Ownership: the caller allocates and frees every buffer (inputs, outputs,
 *    saved forward state, workspace).  The library never allocates device or
 *    host memory for data, never frees, and never synchronises the stream.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Argument errors are detected on the host and
 *    returned before anything is enqueued; nothing is launched on error.
 *  - Device: the current CUDA device must be compute capability 10.0
 *    (B200, sm_100a); otherwise TRI_ATTN_ERR_ARCH.
 *  - Types: q, k, v, bias, dout, o, resid and all gradients are BF16; mask
 *    and lse are FP32.
 *  - Strides are in ELEMENTS.  The innermost (channel / key) stride must be 1;
 *    every other stride must be a non-negative multiple of 8 elements (16
 *    bytes) except the mask's, which may be anything (0 broadcasts).  Data
 *    pointers must be 16-byte aligned (mask: 4-byte).
 *  - Supported sizes: 1 <= B, 1 <= N <= 4096, 1 <= H, d in {32, 64}.
 *  - Rows whose every key is masked (all mask values <= -1e8) are outside
 *    the contract: their outputs are unspecified.
 *  - Determinism: for fixed inputs and shapes every output is bitwise
 *    identical from run to run (no floating-point atomics; every reduction
 *    has a fixed order independent of scheduling and SM count).
 *  - Thread safety: all entry points are reentrant.
 */
#ifndef TRI_ATTN_H
#define TRI_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TRI_ATTN_ABI_VERSION 1

/* A cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st *tri_attn_stream_t;

typedef enum {
    TRI_ATTN_OK = 0,
    TRI_ATTN_ERR_NULL = 1,           /* a required pointer is NULL                     */
    TRI_ATTN_ERR_SHAPE = 2,          /* B, N or H out of range                         */
    TRI_ATTN_ERR_STRIDE = 3,         /* innermost stride != 1, or a stride not a
                                        non-negative multiple of 8 elements          */
    TRI_ATTN_ERR_ALIGN = 4,          /* a data pointer is not 16-byte aligned          */
    TRI_ATTN_ERR_DTYPE = 5,          /* reserved for bindings: wrong element type      */
    TRI_ATTN_ERR_UNSUPPORTED = 6,    /* d not in {32, 64}, or N > 4096                 */
    TRI_ATTN_ERR_WORKSPACE = 7,      /* workspace NULL or smaller than required        */
    TRI_ATTN_ERR_ARCH = 8,           /* current device is not sm_100                   */
    TRI_ATTN_ERR_CUDA = 9,           /* a CUDA runtime/driver call failed              */
    TRI_ATTN_ERR_DEVICE_TIMEOUT = 10, /* a kernel's bounded wait expired (see
                                        tri_attn_device_error)                        */
    TRI_ATTN_ERR_SCRATCH_LIMIT = 11  /* the sizes need more scratch than
                                        TRI_ATTN_STATIC_SCRATCH_BYTES (only from
                                        tri_attn_bwd_static_scratch)                 */
} tri_attn_status;

/* BF16 pair tensor [B,N,N,H,d]; stride[] = element strides of (b,i,j,h,c), c-stride 1. */
typedef struct {
    void *ptr;
    int64_t stride[5];
} tri_attn_tensor5;

/* BF16 bias / bias gradient [B,H,N,N]; stride[] = element strides of (b,h,j,k), k-stride 1. */
typedef struct {
    void *ptr;
    int64_t stride[4];
} tri_attn_tensor4;

/* FP32 additive mask [B,N,N] indexed (b,i,k); ptr may be NULL (no mask); any strides. */
typedef struct {
    const float *ptr;
    int64_t stride[3];
} tri_attn_mask;

/*
 * Forward arguments.
 *   q, k, v, bias, mask : inputs (read only)
 *   o     : output, BF16 round-to-nearest-even of the FP32 result O32
 *   resid : output, BF16 RNE of (O32 - float(o)), the output-rounding residual
 *           (page A, section "它优化了什么": saved so that the backward's softmax
 *           correction can be formed in FP32 from o + resid)
 *   lse   : output, FP32 log-sum-exp of each softmax row (natural log), a
 *           contiguous [B,H,N,N] array indexed (b,h,i,j)
 *   scale : multiplies q.k only; 0 means 1/sqrt(d)
 */
typedef struct {
    int B, N, H, d;
    float scale;
    tri_attn_tensor5 q, k, v;
    tri_attn_tensor4 bias;
    tri_attn_mask mask;
    tri_attn_tensor5 o, resid;
    float *lse;
} tri_attn_fwd_args;

/* Backward flag: form the softmax correction D from o alone, ignoring resid
 * (the uncompensated variant, for measuring what the residual buys). */
#define TRI_ATTN_BWD_NO_RESIDUAL 1u

/*
 * Backward arguments.
 *   f     : the forward's inputs plus its saved state (o, resid, lse), all read only
 *   dout  : upstream gradient of o (read only)
 *   dq, dk, dv : outputs, BF16, same layout rules as q
 *   dbias : output, BF16 [B,H,N,N], the sum over rows i of the score gradient
 *   workspace, workspace_bytes : caller-owned device scratch of at least
 *           tri_attn_bwd_workspace_bytes(B,N,H,d) bytes, 256-byte aligned;
 *           contents on entry are ignored and on exit are unspecified
 *   flags : 0, or TRI_ATTN_BWD_NO_RESIDUAL
 * No gradient is produced for mask.
 */
typedef struct {
    tri_attn_fwd_args f;
    tri_attn_tensor5 dout;
    tri_attn_tensor5 dq, dk, dv;
    tri_attn_tensor4 dbias;
    void *workspace;
    size_t workspace_bytes;
    unsigned flags;
} tri_attn_bwd_args;

/* Enqueue the forward on `stream`.  Returns TRI_ATTN_OK or the first argument
 * error found (nothing enqueued), or TRI_ATTN_ERR_CUDA if a launch failed. */
tri_attn_status tri_attn_fwd(const tri_attn_fwd_args *args, tri_attn_stream_t stream);

/* Bytes of device workspace tri_attn_bwd needs for these sizes (a pure
 * function of the sizes; 0 for invalid sizes).  No device access. */
size_t tri_attn_bwd_workspace_bytes(int B, int N, int H, int d);

/* Enqueue the backward (dq, dk, dv, dbias) on `stream`.  Same error rules as
 * tri_attn_fwd, plus TRI_ATTN_ERR_WORKSPACE. */
tri_attn_status tri_attn_bwd(const tri_attn_bwd_args *args, tri_attn_stream_t stream);

/* tri_attn_bwd with timing markers: `markers` is NULL or an array of four
 * cudaEvent_t handles (as void*) that are recorded on `stream` before the
 * D pre-pass, before the dq/dk/dv kernel, before the dbias kernel(s) and
 * after the last kernel, so a caller can time each phase with the events it
 * owns.  Otherwise identical to tri_attn_bwd. */
tri_attn_status tri_attn_bwd_marked(const tri_attn_bwd_args *args, tri_attn_stream_t stream,
                                    void *const *markers);

/* ---------------------------------------------------------------------------
 * Row shards: a 1-D split of the rows i across devices, the row sharding of
 * the pair representation in "Design-CP: Context Parallelism for Design of
 * Protein Nanoparticles" (gist.science summary), section "方法论", item
 * "1. 推理策略" (1D row sharding).  The problems of
 * different rows i are independent except for dBias, the sum over i of the
 * score gradient: each shard returns its share of that sum in FP32, and
 * tri_attn_dbias_sum adds the shares of all shards in a fixed order.
 *
 * A shard call covers rows i0 .. i0+rows-1 of the full problem:
 *   args->N            : the full N (the j and k extent; bias is [B,H,N,N])
 *   q,k,v,o,resid,dout,dq,dk,dv : point at row i0 (strides unchanged)
 *   mask.ptr           : points at row i0 (if not NULL)
 *   lse                : this shard's own contiguous FP32 [B,H,rows,N] array
 *   1 <= rows <= N, else TRI_ATTN_ERR_SHAPE.
 * With rows = N and no offset, tri_attn_fwd_rows equals tri_attn_fwd bit for
 * bit, and so do the o, resid, lse, dq, dk, dv of a shard and of the whole.
 * --------------------------------------------------------------------------- */
tri_attn_status tri_attn_fwd_rows(const tri_attn_fwd_args *args, int rows, tri_attn_stream_t stream);

/* Workspace bytes of tri_attn_bwd_rows (pure function; 0 for invalid sizes). */
size_t tri_attn_bwd_rows_workspace_bytes(int B, int rows, int N, int H, int d);

/* Number P of FP32 dBias partial sums tri_attn_bwd_rows writes for these sizes
 * (pure function, the same for every shard of equal rows; 0 if invalid). */
int tri_attn_bwd_rows_dbias_parts(int B, int rows, int N, int H, int d);

/* Backward of one shard: dq, dk, dv of its rows as tri_attn_bwd does, and its
 * share of dBias as P contiguous FP32 [B,H,N,N] arrays in dbias_parts
 * (caller-owned, 16-byte aligned, P * B*H*N*N floats, overwritten); their sum
 * is the shard's sum over its rows of the score gradient.  args->dbias is not
 * used.  Workspace: tri_attn_bwd_rows_workspace_bytes. */
tri_attn_status tri_attn_bwd_rows(const tri_attn_bwd_args *args, int rows, float *dbias_parts,
                                  tri_attn_stream_t stream);

/* dbias = BF16 RNE of the sum of nparts contiguous FP32 [B,H,N,N] arrays,
 * added in ascending index order (the shards' partials gathered in rank
 * order: every device that calls this on the same gathered array gets the
 * same bits).  parts 16-byte aligned; dbias strides as in tri_attn_bwd. */
tri_attn_status tri_attn_dbias_sum(const float *parts, int nparts, int B, int H, int N, tri_attn_tensor4 dbias,
                                   tri_attn_stream_t stream);

/* Size of the static scratch area of tri_attn_bwd_static_scratch, per device:
 * 64 MiB, enough for every size whose tri_attn_bwd_workspace_bytes is at most
 * that (for example B=1, N=768, H=4 at d=32 or d=64). */
#define TRI_ATTN_STATIC_SCRATCH_BYTES (64ull << 20)

/*
 * The backward without any device allocation.  The method's pages have no
 * counterpart to this: it is a service of the library, for callers that must
 * not allocate device memory on the path where the backward runs (an
 * application whose allocator owns all device memory, or a latency-critical
 * loop where cudaMalloc / cudaFree, which can synchronise the device, are not
 * allowed).  It runs exactly the kernels of tri_attn_bwd and returns the same
 * results, but its scratch is a fixed array of TRI_ATTN_STATIC_SCRATCH_BYTES
 * in the library's own device memory, reserved when the library's module for
 * it is loaded onto a device; args->workspace and args->workspace_bytes are
 * ignored.
 *   - Order of checks: the argument errors of tri_attn_bwd first (on the
 *     host, before any CUDA call), then the limit: sizes whose
 *     tri_attn_bwd_workspace_bytes(B,N,H,d) exceeds
 *     TRI_ATTN_STATIC_SCRATCH_BYTES are rejected with
 *     TRI_ATTN_ERR_SCRATCH_LIMIT before anything is enqueued.
 *   - Set-up: the first call on each device (the current device at the call)
 *     looks up the array's device address, which loads the module there; call
 *     it once on each device before any stream capture begins, so that this
 *     set-up happens outside a capture.  The address is kept per device
 *     together with the CUDA context it belongs to; after a device reset (a
 *     new context) the next call looks it up again, so that call is a set-up
 *     call too.
 *   - Initial contents: nothing in the scratch has to start at zero; every
 *     word the kernels read is written earlier in the same call.
 *   - Races: all calls on one device share the one array.  Two calls whose
 *     work can overlap on the device (different streams without an ordering
 *     event between them, or several host threads) race on it and produce
 *     wrong gradients; order them, for example on one stream.
 * Otherwise the same arguments and error rules as tri_attn_bwd.
 */
tri_attn_status tri_attn_bwd_static_scratch(const tri_attn_bwd_args *args, tri_attn_stream_t stream);

/* ---------------------------------------------------------------------------
 * Triangle multiplicative update: the contraction step.
 *
 * The pages name the Triangle Multiplicative Update as the second operation
 * TurboPairFormer optimises beside triangle attention (page A, opening
 * paragraph; page B, the paragraph introducing TurboPairFormer) without a
 * formula; read the AlphaFold way, its only cubic step contracts two projected
 * pair tensors over the third residue k, for every batch b and channel c:
 *   outgoing edges (flags 0):            x[b,c,i,j] = sum_k a[b,c,i,k] b[b,c,j,k]
 *   incoming edges (TRI_MUL_INCOMING):   x[b,c,i,j] = sum_k a[b,c,k,i] b[b,c,k,j]
 * The projections, gates and LayerNorms around it are per-position work of the
 * model and are not part of this call.
 *   a, b, x : BF16 [B,C,N,N], channel-first (the caller permutes the
 *             channel-last pair representation), strides as tri_attn_tensor4
 *             with (b, c, row, col) in place of (b, h, j, k): innermost stride
 *             1, the others non-negative multiples of 8 elements, pointers
 *             16-byte aligned
 *   x       : output, BF16 round-to-nearest-even of the FP32 sum
 * Sizes: 1 <= B, 1 <= C, B*C <= 65535, 1 <= N <= 16384.  Same ownership,
 * asynchrony, error and determinism rules as the attention calls.
 */
#define TRI_MUL_INCOMING 1u

typedef struct {
    int B, C, N;
    tri_attn_tensor4 a, b;
    tri_attn_tensor4 x;
    unsigned flags; /* 0 (outgoing edges) or TRI_MUL_INCOMING */
} tri_mul_fwd_args;

/* Backward of the contraction: given dx (the upstream gradient of x), writes
 *   outgoing:  da[i,k] = sum_j dx[i,j] b[j,k]     db[j,k] = sum_i dx[i,j] a[i,k]
 *   incoming:  da[k,i] = sum_j dx[i,j] b[k,j]     db[k,j] = sum_i dx[i,j] a[k,i]
 * (BF16 outputs from FP32 sums).  f.a, f.b and f.flags as in the forward;
 * f.x is not used. */
typedef struct {
    tri_mul_fwd_args f;
    tri_attn_tensor4 dx;
    tri_attn_tensor4 da, db;
} tri_mul_bwd_args;

tri_attn_status tri_mul_fwd(const tri_mul_fwd_args *args, tri_attn_stream_t stream);
tri_attn_status tri_mul_bwd(const tri_mul_bwd_args *args, tri_attn_stream_t stream);

/* ---------------------------------------------------------------------------
 * Gated output projection around the attention (no counterpart on the pages,
 * which describe the attention itself; the AlphaFold-style steps on either
 * side of it, fused):  for every pair position r,
 *     g = sigmoid(z[r,:] Wg),   y[r,:] = (g * o[r,:]) Wo
 *   z  : BF16 [R, 128], the attention block's pair input (cz = 128)
 *   o  : BF16 [R, 128], the attention output with heads concatenated (H*d = 128)
 *   wg : BF16 [128, 128] row-major, wg[cz][co];  wo: BF16 [128, 128], wo[co][cz]
 *   y  : BF16 [R, 128] output (RNE of the FP32 result)
 * Row strides in elements (multiples of 8); pointers 16-byte aligned; R >= 1.
 * No biases.  Same ownership, asynchrony and error rules as the other calls.
 */
typedef struct {
    int R;
    const void *z;
    int64_t z_stride;
    const void *o;
    int64_t o_stride;
    const void *wg, *wo;
    void *y;
    int64_t y_stride;
} tri_gate_fwd_args;

tri_attn_status tri_gate_fwd(const tri_gate_fwd_args *args, tri_attn_stream_t stream);

/* Backward of tri_gate_fwd for the upstream gradient dy (a = g * o):
 *     dA = dy Wo^T,  do = dA * g,  dl = dA * o * g * (1 - g),
 *     dz = dl Wg^T,  dWo = sum_r a^T dy,  dWg = sum_r z^T dl
 *   f      : the forward's arguments (f.y is not used)
 *   dy     : BF16 [R, 128] upstream gradient
 *   dz, d_o: BF16 [R, 128] outputs (overwritten)
 *   dwg    : FP32 [128, 128] row-major, dwg[cz][co] (overwritten)
 *   dwo    : FP32 [128, 128] row-major, dwo[co][cz] (overwritten)
 *   workspace, workspace_bytes : caller-owned device scratch of at least
 *            tri_gate_bwd_workspace_bytes(R) bytes, 16-byte aligned (partial
 *            weight-gradient sums of each CTA).
 * The weight gradients are summed in a fixed order, so repeated calls with the
 * same inputs give bitwise-identical results.  Strides, alignment and errors
 * as for tri_gate_fwd; TRI_ATTN_ERR_WORKSPACE if the workspace is NULL or too
 * small. */
typedef struct {
    tri_gate_fwd_args f;
    const void *dy;
    int64_t dy_stride;
    void *dz;
    int64_t dz_stride;
    void *d_o;
    int64_t do_stride;
    float *dwg, *dwo;
    void *workspace;
    size_t workspace_bytes;
} tri_gate_bwd_args;

/* Bytes of workspace tri_gate_bwd needs for R pair positions (pure function;
 * 0 for R < 1). */
size_t tri_gate_bwd_workspace_bytes(int R);

tri_attn_status tri_gate_bwd(const tri_gate_bwd_args *args, tri_attn_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char *tri_attn_strerror(tri_attn_status status);

/* Reads (and, if clear != 0, resets) the library's device error word on the
 * current device.  Every spin-wait inside the kernels is bounded; a wait that
 * expires records its site there and the kernel returns early instead of
 * hanging.  While the word is set, every later launch of the library's
 * kernels returns at once without computing (outputs untouched), until the
 * word is cleared here.  Synchronises the device.  Returns TRI_ATTN_OK,
 * TRI_ATTN_ERR_DEVICE_TIMEOUT (and stores the raw word in *word if non-NULL),
 * or TRI_ATTN_ERR_CUDA. */
tri_attn_status tri_attn_device_error(int clear, uint32_t *word);

/* Sets the bound of every kernel spin-wait, in nanoseconds of GPU global
 * timer (default 2e9 = 2 s).  Affects launches enqueued afterwards. */
void tri_attn_set_wait_limit_ns(uint64_t ns);

/* Test hook for the timeout path: enqueues a one-CTA kernel whose bounded
 * wait is on a barrier that nothing ever completes, so the wait must expire
 * (after the current limit) and record TRI_ATTN_ERR_DEVICE_TIMEOUT in the
 * device error word.  Faults nothing; the context stays usable. */
tri_attn_status tri_attn_selftest_expire_wait(tri_attn_stream_t stream);

/* TRI_ATTN_ABI_VERSION of the loaded library. */
int tri_attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TRI_ATTN_H */
