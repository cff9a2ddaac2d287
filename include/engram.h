/*
 * engram.h - C ABI of the Engram conditional-memory hot path for NVIDIA B200
 * (sm_100a): the n-gram hash with its table-row gather, and the fused Engram
 * gate, forward and backward, with the weight-gradient reduction.
 *
 * The operations are the Engram kernels listed on the page "DeepSeek 开源
 * TileKernels：用 Python 写出逼近硬件极限的 GPU 内核" (zhichai.net/topic/177618722),
 * section "5. Engram — 条件记忆门控": engram_hash, engram_gate_fwd/bwd,
 * engram_fused_weight and engram_grad_w_reduce, with the gate formula
 *
 *     gate   = sigmoid(signed_sqrt(dot(RMSNorm(x, wh), RMSNorm(k, we)) * scalar))
 *     output = hidden_states + gate * v
 *     signed_sqrt(s) = sign(s) * sqrt(|s|),  scalar = 1 / sqrt(hidden_size).
 *
 * Conventions shared by every call:
 *   - Device pointers point to CUDA device memory of the current device.  The
 *     caller allocates every buffer and keeps ownership; the library allocates
 *     no device memory.  Per device it keeps, from the first call that needs
 *     them until the process exits, host-side launch settings of the gate
 *     calls and, for engram_gather_bwd, one stream and two events.
 *   - Every compute call is asynchronous on `stream` (NULL: the legacy default
 *     stream) and never synchronises.  Outputs are valid once the stream has
 *     reached the call.
 *   - "bf16" tensors are contiguous, row-major arrays of IEEE bfloat16.  The
 *     gate calls take any hidden size H in [1, 65536] and bf16 tensors on any
 *     2-byte boundary: when H is a multiple of 8 up to 8192 and every bf16
 *     tensor (and the fp32 partial rows) starts on a 16-byte boundary, the
 *     kernels tuned for the pages' sizes run (whole rows moved with 16-byte
 *     bulk copies); otherwise generic kernels compute the same formulas with
 *     plain loads, two passes over each token's rows.  The hash/gather calls
 *     keep their own alignment rules, stated below.
 *   - Errors: arguments are checked before anything is launched; a failing
 *     check returns ENGRAM_ERR_INVALID_ARG (bad pointer, size or alignment) or
 *     ENGRAM_ERR_UNSUPPORTED (a size this library does not handle) and launches
 *     nothing.  A failing CUDA runtime call returns ENGRAM_ERR_CUDA.  The
 *     message of the last failure on the calling thread is returned by
 *     engram_last_error().  Kernels never trap; a pipeline wait that exceeds
 *     its time limit records a code that engram_read_device_error() reports.
 */
#ifndef ENGRAM_H
#define ENGRAM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENGRAM_API __attribute__((visibility("default")))
#else
#define ENGRAM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
struct CUstream_st;
typedef struct CUstream_st *engram_stream_t;

typedef enum {
    ENGRAM_OK = 0,
    ENGRAM_ERR_INVALID_ARG = 1,
    ENGRAM_ERR_UNSUPPORTED = 2,
    ENGRAM_ERR_CUDA = 3
} engram_status_t;

/* Codes a kernel may record in the device error word. */
#define ENGRAM_DEVICE_ERR_PIPELINE_TIMEOUT 1u
#define ENGRAM_DEVICE_ERR_INDEX_RANGE 2u   /* engram_gather_bwd met an index outside its table */

/* Version of this ABI (incremented on any incompatible change). */
ENGRAM_API int engram_abi_version(void);

/* Static description of a status code.  Never NULL. */
ENGRAM_API const char *engram_status_string(engram_status_t status);

/* Message of the last failing call made by this thread ("" if none). */
ENGRAM_API const char *engram_last_error(void);

/*
 * engram_hash_gather - n-gram hash to embedding-table indices, then gather of
 * the indexed table rows ("engram_hash" on the page above; the hash combines
 * XOR and multiplication over the token sequence and maps it to indices of 8
 * embedding tables per n-gram layer, 2 layers, up to 3-grams).
 *
 * For token t = (b, s), layer l and table j:
 *     h      = XOR_{i=0}^{ngram_n[l]-1}  u64(tok(b, s-i)) * multipliers[l*n_max + i]
 *              (products wrap modulo 2^64; tok(b, s-i) = pad_id when s-i < 0,
 *              so the history never crosses into another sequence)
 *     idx    = h mod table_sizes[l*J + j]          (unsigned 64-bit remainder)
 *     row    = rows [idx] of table (l, j)
 *
 * tokens      device, int64 [B*S], row-major [B][S], 8-byte aligned.
 * B, S        >= 0 (B*S == 0 launches nothing).
 * multipliers HOST, uint64 [L*n_max]; copied into the launch, may be freed on
 *             return.  Entries beyond ngram_n[l] in a row are ignored.
 * ngram_n     HOST, int32 [L], each in [1, n_max].
 * L           number of n-gram layers, 1..4.     n_max  1..8.
 * table_sizes HOST, int64 [L*J], rows of table (l, j) at l*J+j, each >= 1.
 * J           tables per layer, 1..16.
 * tables      device, bf16, the L*J tables stored one after another in
 *             (l, j) order, each table_sizes[l*J+j] rows of D values;
 *             16-byte aligned.  Needed only when rows_out != NULL.
 * D           row width in bf16 values: a multiple of 8, 8..256.
 * pad_id      token id used for positions before the start of a sequence.
 * idx_out     device, int64 [B*S*L*J] laid out [t][l][j], 8-byte aligned,
 *             or NULL to skip writing indices.
 * rows_out    device, bf16 [B*S*L*J*D] laid out [t][l][j][D], 16-byte
 *             aligned, or NULL to skip the gather (idx_out and rows_out may
 *             not both be NULL when B*S > 0).  With rows_out the tables may
 *             hold at most 2^48 rows in total; without it table sizes may be
 *             any positive int64.
 */
ENGRAM_API engram_status_t engram_hash_gather(const int64_t *tokens, int64_t B, int64_t S,
                                   const uint64_t *multipliers, const int32_t *ngram_n,
                                   int32_t L, int32_t n_max, const int64_t *table_sizes,
                                   int32_t J, const void *tables, int32_t D, int64_t pad_id,
                                   int64_t *idx_out, void *rows_out, engram_stream_t stream);

/*
 * engram_gather_bwd_workspace_size - bytes of device workspace that
 * engram_gather_bwd needs for T tokens, L layers, J tables per layer, rows of
 * D values and total_rows rows in all tables together (the sum of
 * table_sizes).  About 32 bytes per entry plus 2 bits per table row.  Returns
 * -1 (with engram_last_error() set) for sizes that engram_gather_bwd rejects.
 * No device is queried.
 */
ENGRAM_API int64_t engram_gather_bwd_workspace_size(int64_t T, int32_t L, int32_t J, int32_t D,
                                                    int64_t total_rows);

/*
 * engram_gather_bwd - backward of the row gather of engram_hash_gather with
 * respect to the tables.  The page above lists only the gather; its gradient
 * is the transpose of a row copy: every gathered row's gradient is added to
 * the table row it was read from, so a row read by several tokens receives
 * the sum of their gradients:
 *     d_tables[row0(l,j) + idx[t][l][j]][c] += d_rows[t][l][j][c]
 * with row0(l,j) the first row of table (l, j) in the concatenated tables.
 * Rows that no token read are left untouched (d_tables accumulates, like a
 * parameter gradient: zero it before the first call of a step).
 *
 * The gradients of one row are summed in fp64 (bf16 values enter exactly) in
 * an order fixed by the positions of the entries, and the row is updated with
 * one rounding: d_tables[r] = fp32((double)d_tables[r] + sum).  The result is
 * bitwise reproducible.
 *
 * idx         device, int64 [T*L*J] laid out [t][l][j] (as written by
 *             engram_hash_gather), 8-byte aligned; each entry must lie in
 *             [0, table_sizes[l*J + j]).  An entry outside that range is
 *             skipped and the kernels record ENGRAM_DEVICE_ERR_INDEX_RANGE
 *             (see engram_read_device_error); nothing outside the buffers is
 *             touched.
 * T           >= 0 tokens (0 launches nothing; the pointers may then be NULL).
 * L, J        1..4 layers, 1..16 tables per layer; T*L*J <= 2^30.
 * table_sizes HOST, int64 [L*J], each >= 1, total rows R below 2^32 - 1.
 * d_rows      device, bf16 [T*L*J*D] laid out [t][l][j][D], 16-byte aligned:
 *             the gradient of the gathered rows.
 * D           row width: a multiple of 8, 8..256.
 * d_tables    device, fp32 [R*D], row-major, 16-byte aligned; accumulated.
 * workspace   device scratch of at least workspace_bytes >=
 *             engram_gather_bwd_workspace_size(T, L, J, D, R) bytes, 16-byte
 *             aligned, owned by the caller; its contents need not be
 *             initialised and are meaningless afterwards.  Calls in flight at
 *             the same time need separate workspaces.
 *
 * Streams: the kernels for the rows read more than once run on a stream of
 * the device's highest priority that the library creates on the first call
 * (one per device), forked from `stream` and joined back into it with two
 * events, so the call is ordered on `stream` like any other.  Calls from
 * several host threads take turns while they enqueue, and their side work
 * runs in the order they enqueued.  A call may be captured into a CUDA graph
 * once an earlier call has created the side stream; until that capture ends,
 * the side stream belongs to it, so no other thread may call
 * engram_gather_bwd on the same device meanwhile.
 */
ENGRAM_API engram_status_t engram_gather_bwd(const int64_t *idx, int64_t T, int32_t L, int32_t J,
                                  const int64_t *table_sizes, const void *d_rows, int32_t D,
                                  float *d_tables, void *workspace, size_t workspace_bytes,
                                  engram_stream_t stream);

/*
 * engram_gate_fwd - fused Engram gate forward ("engram_gate_fwd" on the page
 * above: RMSNorm, signed-sqrt activation and sigmoid gate fused), with the
 * fused weight w = wh * we ("engram_fused_weight") formed inside the kernel:
 *     rx   = (mean_j x_j^2 + eps)^(-1/2),  rk = (mean_j k_j^2 + eps)^(-1/2)
 *     s    = rx * rk * sum_j x_j k_j wh_j we_j * scalar
 *     gate = sigmoid(sign(s) sqrt(|s|)),   out = x + gate * v
 * Accumulation is fp32; out is rounded to bf16 (nearest even).
 *
 * x, k, v     device, bf16 [T*H], row-major [T][H], 2-byte aligned.
 * wh, we      device, bf16 [H], 2-byte aligned.
 * T           >= 0 tokens (0 launches nothing; the pointers may then be NULL).
 * H           hidden size, 1..65536 (see the conventions for which kernels run).
 * eps         >= 0, finite.   scalar  finite (normally 1/sqrt(H)).
 * out         device, bf16 [T*H], 2-byte aligned (may not alias the inputs).
 * gate        device, fp32 [T], 4-byte aligned, or NULL to skip it.
 */
ENGRAM_API engram_status_t engram_gate_fwd(const void *x, const void *k, const void *v, const void *wh,
                                const void *we, int64_t T, int32_t H, float eps, float scalar,
                                void *out, float *gate, engram_stream_t stream);

/*
 * engram_gate_bwd_num_partials - the recommended row count G of the
 * weight-gradient partial buffer of engram_gate_bwd on the current device
 * (one persistent CTA per partial row).  Returns a value >= 1, or -1 with
 * engram_last_error() set when no CUDA device can be queried.
 */
ENGRAM_API int64_t engram_gate_bwd_num_partials(int64_t T, int32_t H);

/*
 * engram_gate_bwd - backward of engram_gate_fwd with respect to x, k, v and,
 * in partial form, wh and we ("engram_gate_bwd").  The per-token statistics
 * are recomputed from x and k; nothing is saved from the forward.  With
 * g = grad_out, d = rx*rk*sum_j x_j k_j w_j, w = wh*we and
 *     du = (sum_j g_j v_j) * gate * (1 - gate)
 *     dd = du / (2 sqrt(max(|s|, 1e-6))) * scalar,    c = dd * rx * rk
 *     dx_j = g_j + c w_j k_j - dd d rx^2 x_j / H
 *     dk_j = c w_j x_j - dd d rk^2 k_j / H
 *     dv_j = gate * g_j
 *     w_partial[p][j] = sum over the tokens t of partial row p of c_t x_tj k_tj
 * CTA p of G handles tokens p, p+G, p+2G, ... in that order, so the partials
 * (and everything else) are bitwise reproducible for a given G.
 *
 * grad_out, x, k, v  device, bf16 [T*H], 2-byte aligned.
 * wh, we             device, bf16 [H], 2-byte aligned.
 * T >= 0, H as in engram_gate_fwd, eps/scalar as passed to the forward.
 * dx, dk, dv         device, bf16 [T*H], 2-byte aligned (no aliasing).
 * w_partial          device, fp32 [G*H], 4-byte aligned; fully overwritten
 *                    (rows of CTAs without tokens are written as zeros, so
 *                    T == 0 yields all-zero partials; the token tensors may
 *                    then be NULL).
 * G                  >= 1, at most 2^31 - 1 (engram_gate_bwd_num_partials()
 *                    gives the value that fills the GPU once).
 */
ENGRAM_API engram_status_t engram_gate_bwd(const void *grad_out, const void *x, const void *k,
                                const void *v, const void *wh, const void *we, int64_t T,
                                int32_t H, float eps, float scalar, void *dx, void *dk,
                                void *dv, float *w_partial, int64_t G, engram_stream_t stream);

/*
 * engram_grad_w_reduce - weight-gradient reduction ("engram_grad_w_reduce"):
 *     P_j   = sum_{p=0}^{G-1} w_partial[p][j]
 *     dwh_j = we_j * P_j,   dwe_j = wh_j * P_j
 * which are the gradients of sum over tokens of the forward's loss with
 * respect to wh and we.  The fp32 sum has an order fixed by G alone, so the
 * result is bitwise reproducible: the rows form consecutive groups of
 * size = max(ceil(sqrt(G)), ceil(G/32)) rows (the last group may be shorter),
 * each group is summed in row order starting from 0, and the group sums are
 * added in group order starting from 0.  engram_gate_bwd_fused uses the same
 * order, so both give the same bits.
 *
 * w_partial   device, fp32 [G*H] as written by engram_gate_bwd, 4-byte aligned.
 * G >= 1, H >= 1.
 * wh, we      device, bf16 [H], 2-byte aligned.
 * dwh, dwe    device, fp32 [H], 4-byte aligned; overwritten, not accumulated.
 */
ENGRAM_API engram_status_t engram_grad_w_reduce(const float *w_partial, int64_t G, int32_t H,
                                     const void *wh, const void *we, float *dwh, float *dwe,
                                     engram_stream_t stream);

/* Words of the ticket array engram_gate_bwd_fused takes. */
#define ENGRAM_GATE_BWD_TICKETS 64

/*
 * engram_gate_bwd_fused - engram_gate_bwd and engram_grad_w_reduce in one
 * launch (the page lists the two operators separately; here the reduction of
 * the partial rows runs in the tail of the backward kernel instead of a
 * second kernel).  Each CTA of the backward writes its partial row and takes
 * a ticket (an atomic count); the last CTAs to take one (at most half of the
 * CTAs the GPU holds at once, so that the others can always be scheduled)
 * wait until every CTA has, with a time limit, and then each reduces a slice
 * of the columns over all partial rows and writes that slice of dwh and dwe.
 * The order of every fp32 sum is the one engram_grad_w_reduce documents, so
 * dwh and dwe are bitwise those of engram_gate_bwd followed by
 * engram_grad_w_reduce with the same G.
 *
 * Arguments as in engram_gate_bwd, plus:
 * w_partial   device, fp32 [G*H], 4-byte aligned: scratch of the reduction
 *             (its contents on return are unspecified: group rows hold sums).
 * tickets     device, uint32 [ENGRAM_GATE_BWD_TICKETS], 4-byte aligned, all
 *             zero before the first call (e.g. cudaMemsetAsync once).  Every
 *             call sets them back to zero when it completes, so one array
 *             serves any number of calls in stream order; calls that may run
 *             at the same time on the GPU need separate arrays.  After a call
 *             that recorded ENGRAM_DEVICE_ERR_PIPELINE_TIMEOUT its gradients are
 *             invalid and the tickets must be zeroed again before the next call.
 * dwh, dwe    device, fp32 [H], 4-byte aligned; overwritten, not accumulated.
 * Shapes that the tuned kernels do not take (see the conventions) run the
 * generic backward and then the standalone reduction: two launches, same
 * results as those two calls, tickets untouched.
 */
ENGRAM_API engram_status_t engram_gate_bwd_fused(const void *grad_out, const void *x,
                                      const void *k, const void *v, const void *wh,
                                      const void *we, int64_t T, int32_t H, float eps,
                                      float scalar, void *dx, void *dk, void *dv,
                                      float *w_partial, int64_t G, uint32_t *tickets,
                                      float *dwh, float *dwe, engram_stream_t stream);

/*
 * engram_gate_bwd_noalloc - engram_gate_bwd followed by engram_grad_w_reduce,
 * allocating nothing, for callers that cannot allocate device memory (code
 * that may not call cudaMalloc or an allocating library, e.g. a runtime whose
 * memory policy forbids allocations outside its own pool, or one that only
 * owns the buffers it passes in).  The Engram section has no counterpart: it
 * is a packaging of the two calls above.
 *
 * Arguments as in engram_gate_bwd, except that the weight-gradient partial
 * rows are kept in a static device array of the library (8 MiB per GPU that
 * loads it, held until the process exits) instead of a caller buffer, and the
 * reduced gradients dwh, dwe (device, fp32 [H], 4-byte aligned, overwritten)
 * are written directly.  The partial row count G is the one
 * engram_gate_bwd_num_partials(T, H) recommends, lowered to floor(2^21 / H)
 * when G rows of H floats would not fit in the array (the backward's CTAs
 * loop over tokens, so any G gives the same gradients up to the order of the
 * fp32 sums).  H itself is limited to 65536 as everywhere, so one row always
 * fits; sizes outside the gate's limits return ENGRAM_ERR_UNSUPPORTED or
 * ENGRAM_ERR_INVALID_ARG and launch nothing.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current): make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents, so calls whose kernels overlap on the GPU (different streams
 * without ordering between them) race and give wrong gradients; calls in
 * stream order are fine.  Nothing in the array has to start at zero: every
 * value the reduction reads is written by the same call first.
 */
ENGRAM_API engram_status_t engram_gate_bwd_noalloc(const void *grad_out, const void *x,
                                        const void *k, const void *v, const void *wh,
                                        const void *we, int64_t T, int32_t H, float eps,
                                        float scalar, void *dx, void *dk, void *dv,
                                        float *dwh, float *dwe, engram_stream_t stream);

/*
 * engram_read_device_error - synchronises the current device, then reads (and
 * when `clear` is non-zero, resets) the device error word in which kernels
 * record a pipeline wait that ran past its time limit.  *code_out receives 0
 * or a bitwise OR of ENGRAM_DEVICE_ERR_* codes.  Diagnostic; not for hot paths.
 */
ENGRAM_API engram_status_t engram_read_device_error(uint32_t *code_out, int32_t clear);

#ifdef __cplusplus
}
#endif

#endif /* ENGRAM_H */
