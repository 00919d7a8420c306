/*
 * libaal — associative-algebra block projections on B200 (sm_100a).
 *
 * The operator comes from "Change the Product, Keep the Parameters:
 * Associative Algebra Layers for Transformers" (Koziev & Oseledets,
 * arXiv:2609.32814).  A projection Y = X W (X [tokens, din], W [din, dout],
 * agihunt.info digest, opening paragraph) is cut into q feature groups on
 * both sides, so W is a q x q grid of blocks W_ak of size (din/q) x (dout/q).
 * Instead of the row-by-column rule, output block (i, k) of X * W sums only
 * the products X_ia W_ak with a in S(i, k), where S is the multiplication
 * table of an associative algebra:
 *
 *   complete-graph law Q_q  (agihunt.info digest, multiplication-table
 *   paragraph): S(i, i) = {i}; S(i, k) = {i, k} for k != i — a diagonal
 *   block multiplies only its own group, an off-diagonal block is the source
 *   diagonal times the edge plus the edge times the target diagonal.
 *   2q^2 - q block products on the square, 2q - 1 per row.
 *
 *   tensor-square law Q2 (x) Q2 (agihunt.info digest, tensor-square
 *   paragraph): 4 groups indexed by pairs g = 2*g1 + g2,
 *   S((i1,i2),(k1,k2)) = S(i1,k1) x S(i2,k2) under Q_2.  36 block products on
 *   the square, 9 of 16 per row.
 *
 * Row typing (agihunt.info digest, paragraph on the Transformer mapping;
 * hotpaper.ai summary, "row-typed rectangular projections"): each token gets
 * a row type t from its absolute position and computes only row t of the
 * table: y_k = sum_{a in S(t, k)} x_a W_ak.  The type is position mod q.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Matrices are row-major with a leading dimension ``ld`` (elements, >=
 *   cols).  Every pointer in an aal_mat is DEVICE memory owned by the
 *   caller; the library never frees or keeps it.
 * - dtype: AAL_BF16 (bf16 inputs, fp32 accumulation, bf16 outputs) or
 *   AAL_F32 (fp32 throughout).  All matrices of one call share one dtype.
 * - The compute calls are asynchronous on ``stream`` (a cudaStream_t; NULL is
 *   the legacy default stream).  Host-side argument errors are returned
 *   before anything is launched.  Errors found on the device (an explicit
 *   row type outside [0, q), a wait that ran out) are recorded in a device
 *   status word that aal_get_device_status() reads.
 * - The tensor-core path needs 16-byte aligned base pointers and leading
 *   dimensions that are multiples of 8 (bf16); other shapes take the general
 *   CUDA path, which needs 4-byte (fp32) or 2-byte (bf16) alignment only.
 * - Nothing aborts; no call allocates device memory.
 */
#ifndef AAL_H_
#define AAL_H_

#include <stdint.h>

#if defined(__GNUC__)
#define AAL_API __attribute__((visibility("default")))
#else
#define AAL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum aal_status {
  AAL_OK = 0,
  AAL_ERR_INVALID_ARG = 1,    /* bad shape, null pointer, unknown enum value */
  AAL_ERR_UNSUPPORTED = 2,    /* valid request the library cannot serve      */
  AAL_ERR_ALIGNMENT = 3,      /* pointer / ld misaligned for a required path */
  AAL_ERR_CUDA = 4,           /* a CUDA runtime call failed                  */
  AAL_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out             */
  AAL_ERR_DEVICE_BOUNDS = 6,  /* a kernel met an out-of-range index (type)   */
  AAL_ERR_SCRATCH_LIMIT = 7   /* request larger than a fixed device scratch   */
} aal_status;

typedef enum aal_law {
  AAL_LAW_Q = 0,     /* complete-graph law Q_q, any q >= 1 */
  AAL_LAW_Q2XQ2 = 1  /* tensor square Q2 (x) Q2; q must be 4 */
} aal_law;

typedef enum aal_dtype { AAL_BF16 = 0, AAL_F32 = 1 } aal_dtype;

/* A row-major device matrix: element (r, c) at ((T*)ptr)[r * ld + c]. */
typedef struct aal_mat {
  void* ptr;
  int32_t dtype; /* aal_dtype */
  int64_t rows;
  int64_t cols;
  int64_t ld;
} aal_mat;

typedef enum aal_row_type_kind {
  /* Tokens are packed as back-to-back sequences of seq_len tokens; row r sits
   * at absolute position (r mod seq_len) + pos_offset and has type
   * position mod q. */
  AAL_TYPES_POSITION = 0,
  /* types[r] (device int32 array of length rows) gives row r's type. */
  AAL_TYPES_EXPLICIT = 1
} aal_row_type_kind;

typedef struct aal_row_type_rule {
  int32_t kind;          /* aal_row_type_kind */
  int64_t seq_len;       /* kind 0: > 0 */
  int64_t pos_offset;    /* kind 0: >= 0 */
  const int32_t* types;  /* kind 1: device pointer, not owned */
} aal_row_type_rule;

/* ---------------------------------------------------------------------- */
/* Compute calls                                                           */
/* ---------------------------------------------------------------------- */

/*
 * Row-typed projection Y = X * W (agihunt.info digest, multiplication-table
 * and Transformer-mapping paragraphs).
 *   X [M, din], W [din, dout], Y [M, dout]; din and dout divisible by q.
 *   Row r of type t: Y[r, group k] = sum_{a in S(t,k)} X[r, group a] W_ak.
 *   Y is overwritten.  M may be 0 (nothing is launched).
 */
AAL_API aal_status aal_project_fwd(int32_t law, int32_t q, aal_row_type_rule rule,
                           aal_mat X, aal_mat W, aal_mat Y, void* stream);

/*
 * SwiGLU feed-forward block with all three projections algebraic and the same
 * row types (agihunt.info digest: the pilot changes only the FFN
 * projections; the full SwiGLU forward is among the measured kernels):
 *   H = silu(X * Wg) . (X * Wu)   (elementwise; silu(z) = z / (1 + e^-z))
 *   Y = H * Wd
 *   X [M, D], Wg and Wu [D, F], Wd [F, D], H [M, F] (caller memory, written
 *   and kept, e.g. for a backward pass), Y [M, D].
 *   The SiLU and the product are applied to the fp32 accumulators before H is
 *   rounded to the call's dtype.
 */
AAL_API aal_status aal_swiglu_fwd(int32_t law, int32_t q, aal_row_type_rule rule,
                          aal_mat X, aal_mat Wg, aal_mat Wu, aal_mat Wd,
                          aal_mat H, aal_mat Y, void* stream);

/*
 * Backward of aal_project_fwd for L = <dY, X * W> (agihunt.info digest:
 * forward plus gradient on the narrow expert FFN shape).
 *   dX[r, group a] = sum over k with a in S(t_r, k) of dY[r, group k] W_ak^T
 *   dW_ak          = sum over rows r with a in S(t_r, k) of
 *                    X[r, group a]^T dY[r, group k]
 *   dX [M, din] may have ptr == NULL (not computed); likewise dW [din, dout].
 *   dX is overwritten; dW is overwritten, or added to when accumulate_dW != 0.
 */
AAL_API aal_status aal_project_bwd(int32_t law, int32_t q, aal_row_type_rule rule,
                           aal_mat X, aal_mat W, aal_mat dY,
                           aal_mat dX, aal_mat dW, int32_t accumulate_dW,
                           void* stream);

/*
 * Backward of aal_swiglu_fwd (agihunt.info digest, SwiGLU figures and the
 * kernel table's backward row; the composition of the projection backward
 * with the derivative of silu(g) u):
 *   G = X*Wg, U = X*Wu (recomputed), dH = dY through Wd's transposed table,
 *   dG = dH (.) U (.) silu'(G), dU = dH (.) silu(G),
 *   dX = dG through Wg's transposed table + dU through Wu's,
 *   dWg = X^T-typed dG, dWu = X^T-typed dU, dWd = H^T-typed dY,
 * with silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + e^-g), every product
 * row-typed with the same rule as the forward.
 *   X [M, D], Wg, Wu [D, F], Wd [F, D], H [M, F] (the forward's activation),
 *   dY [M, D]: inputs.  G, U, dG, dU [M, F]: caller's workspace, overwritten
 *   (on return they hold the pre-activations and their gradients).
 *   dX [M, D], dWg, dWu [D, F], dWd [F, D]: overwritten.
 * The SiLU' chain runs in the epilogue of the dH kernel on the tensor-core
 * path; the general path uses a separate elementwise kernel.  Errors:
 * AAL_ERR_INVALID_ARG for inconsistent shapes, AAL_ERR_UNSUPPORTED for mixed
 * dtypes.
 */
AAL_API aal_status aal_swiglu_bwd(int32_t law, int32_t q, aal_row_type_rule rule,
                          aal_mat X, aal_mat Wg, aal_mat Wu, aal_mat Wd, aal_mat H,
                          aal_mat dY, aal_mat G, aal_mat U, aal_mat dG, aal_mat dU,
                          aal_mat dX, aal_mat dWg, aal_mat dWu, aal_mat dWd, void* stream);

/*
 * Decode step: one new token per batch entry (agihunt.info digest: decoding
 * evaluates only the new position's row, as a matrix-vector product with its
 * own kernel).
 *   positions: device int64 array [B], absolute positions (>= 0); the row
 *   type of entry b is positions[b] mod q.
 *   x [B, din], W [din, dout], y [B, dout] (overwritten).
 */
AAL_API aal_status aal_decode_matvec(int32_t law, int32_t q, const int64_t* positions,
                             aal_mat x, aal_mat W, aal_mat y, void* stream);

/*
 * Decode step of a whole algebraic SwiGLU FFN: the three decode rows of its
 * projections with the activation between them (agihunt.info digest:
 * decoding evaluates only the new position's row; SwiGLU figures, gate, up
 * and down all algebraic with the same row types):
 *   h = silu(x * Wg) (.) (x * Wu),   y = h * Wd,   silu(z) = z / (1 + e^-z)
 * where each "*" is the row-typed product of entry b's row type
 * positions[b] mod q.
 *   positions: device int64 [B]; x [B, D]; Wg, Wu [D, F]; Wd [F, D];
 *   h [B, F] (caller's workspace, overwritten with the activation, bf16 or
 *   fp32 like the inputs); y [B, D] (overwritten).
 * Two launches: gate, up and the activation in one tensor-core decode
 * kernel (one launch per 128 entries), then the down decode; up to 16
 * entries the down decode is a programmatic dependent launch that fetches
 * its weights while the first kernel runs and waits for h on the device.
 * With AAL_FFN_DECODE_FUSED=1 in the environment the step is instead one
 * launch per 128 entries where the shape allows it (bf16, q <= 64, D / q and
 * F / q multiples of 16, 16-byte aligned rows, D / 16 below the SM count):
 * CTAs owning 16 columns of h run gate, up and the activation; CTAs owning 16
 * columns of y stage their columns of Wd meanwhile, wait in a grid barrier
 * (bounded; a wait that runs out records AAL_ERR_DEVICE_TIMEOUT) and finish
 * the down projection.  That barrier uses one of 64 slots of the library's
 * device memory, taken round robin per launch: at most 64 such launches may
 * run concurrently on one device (a launch captured into a CUDA graph keeps
 * its slot).  It is opt-in because on B200 it measured slower than the two
 * launches (12.9 against 8.4 us per step at one entry).
 * An entry with a negative position is skipped (its rows of h and y are not
 * written) and the device status reports AAL_ERR_DEVICE_BOUNDS.
 * Errors: AAL_ERR_INVALID_ARG for inconsistent shapes or a missing
 * positions array, AAL_ERR_UNSUPPORTED for mixed dtypes.
 */
AAL_API aal_status aal_swiglu_decode(int32_t law, int32_t q, const int64_t* positions,
                             aal_mat x, aal_mat Wg, aal_mat Wu, aal_mat Wd, aal_mat h,
                             aal_mat y, void* stream);

/*
 * aal_swiglu_decode without the caller's activation buffer.  The paper has no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory, for example a plug-in inside a host application that owns
 * every device allocation through its own pool and forbids direct cudaMalloc,
 * or a real-time decode loop in which cudaMalloc's implicit device-wide
 * synchronisation is not allowed.
 *   Arguments, results and errors are those of aal_swiglu_decode without h:
 *   positions device int64 [B]; x [B, D]; Wg, Wu [D, F]; Wd [F, D];
 *   y [B, D] (overwritten).  The activation h [B, F] is kept instead in one
 *   fixed array of the library's own device memory, 4 MiB on every device
 *   that loads the library, held until the process exits.
 * Limit: B * F * (2 for bf16, 4 for fp32) <= 4,194,304 bytes (for example
 * B <= 1365 at F = 1536 in bf16); a larger request returns
 * AAL_ERR_SCRATCH_LIMIT before anything is launched.
 * The call allocates nothing and frees nothing.  Its first call on a device
 * looks up the array's device address once (cudaGetSymbolAddress with that
 * device current); make that first call before any stream capture.
 * Every call shares the one array, which keeps the last call's contents;
 * nothing in it has to start at zero (each call writes the rows of h it reads
 * first).  Calls whose work overlaps on the GPU (different streams without
 * an ordering between them) race on the array and give wrong results: order
 * them on one stream or with events.
 */
AAL_API aal_status aal_swiglu_decode_noalloc(int32_t law, int32_t q, const int64_t* positions,
                                     aal_mat x, aal_mat Wg, aal_mat Wu, aal_mat Wd,
                                     aal_mat y, void* stream);

/*
 * Full (not row-typed) product of square block matrices, Z = X * W
 * (agihunt.info digest: fixed-block square product, and the quadratic
 * arithmetic when the block size stays fixed while q grows).
 *   X, W, Z [n, n], n divisible by q, block size b = n / q:
 *   Z_ik = sum_{a in S(i,k)} X_ia W_ak.  Z is overwritten and must not alias
 *   X or W.
 */
AAL_API aal_status aal_square_product(int32_t law, int32_t q, aal_mat X, aal_mat W,
                              aal_mat Z, void* stream);

/* ---------------------------------------------------------------------- */
/* Workspace for explicit and ragged row types                             */
/* ---------------------------------------------------------------------- */

/*
 * The tensor-core path reads the rows of one type through a strided view,
 * which needs position-derived types with seq_len and the row count both
 * multiples of q.  For explicit types, or sequences that do not line up
 * (agihunt.info digest, Transformer-mapping paragraph: the type follows the
 * absolute position, so any packing is legal), aal_project_fwd and
 * aal_swiglu_fwd first sort the rows by type on the device into a caller
 * workspace and then run the tensor-core path on the sorted rows, writing
 * every output row back to its place.  Without a large enough workspace
 * those calls take the general CUDA path (AAL_PATH_TENSOR: they fail with
 * AAL_ERR_UNSUPPORTED).  The backward calls always take the general path for
 * such rules.
 *
 * The backward calls use a workspace differently: under Q_q a few tiles are
 * far longer than the rest (the diagonal blocks of dW sum over every token;
 * the dX blocks a == t sum over every output group), and with a large enough
 * workspace aal_project_bwd and aal_swiglu_bwd cut those tiles into K pieces
 * that run on separate SMs, keep the pieces' fp32 partial sums in the
 * workspace and add them in a short reduction kernel.  The result is the
 * same sum in another association order.  The dH step of aal_swiglu_bwd
 * (its SiLU' chain needs the whole sum) is never split.
 *
 * Small backward problems (rows * d_in * d_hidden up to about 8.6e9) also
 * run launches side by side: aal_project_bwd puts dW on a second stream of
 * the calling host thread beside dX, and aal_swiglu_bwd puts dWd and dWg
 * there beside dX and dWu, each launch on half of the SMs.  The second stream
 * is forked from and joined back to the call's stream by event records and
 * stream waits (so the call also captures into a CUDA graph), and the call's
 * stream orders everything as before.  The second stream and its two events
 * are created by a thread's first such call on a device outside a graph
 * capture and kept for the thread's lifetime; a call captured before that
 * keeps every launch on the call's stream.  The second stream's partial sums sit
 * after the first stream's in the workspace, and aal_workspace_size covers
 * that layout.
 *
 * aal_workspace_size: bytes the call needs for ``rows`` rows; call is
 * AAL_CALL_PROJECT_FWD (d_in = din, d_hidden unused), AAL_CALL_SWIGLU_FWD
 * (d_in = D, d_hidden = F), AAL_CALL_PROJECT_BWD (d_in = din, d_hidden =
 * dout) or AAL_CALL_SWIGLU_BWD (d_in = D, d_hidden = F).  0 when the call
 * uses none, -1 for invalid arguments.  Forward: roughly rows * (d_in
 * [+ d_hidden]) * 2 + rows * 4 bytes; backward: the heavy tiles' partial
 * sums (e.g. 17 MB for M = 2048, din = 2048, dout = 768, q = 16).
 *
 * aal_set_workspace: device memory the following calls of this host thread
 * may use (NULL or 0 bytes: none).  The pointer must be 256-byte aligned
 * (AAL_ERR_ALIGNMENT otherwise); the library does not own it, and the
 * caller keeps it alive and unused by other work until the calls using it
 * have completed on their streams.  Calls that overlap on the GPU must not
 * share a workspace.  Supported: bf16, q <= 256, 16-byte aligned rows,
 * din / q and dout / q multiples of 16.
 */
enum { AAL_CALL_PROJECT_FWD = 1, AAL_CALL_SWIGLU_FWD = 2, AAL_CALL_PROJECT_BWD = 3,
       AAL_CALL_SWIGLU_BWD = 4 };
AAL_API int64_t aal_workspace_size(int32_t call, int32_t law, int32_t q, aal_row_type_rule rule,
                           int64_t rows, int64_t d_in, int64_t d_hidden);
AAL_API aal_status aal_set_workspace(void* device_ptr, uint64_t bytes);

/* ---------------------------------------------------------------------- */
/* Host-side table queries (integer, no GPU needed)                        */
/* ---------------------------------------------------------------------- */

/*
 * The multiplication table as the kernels use it: S is HOST memory of q*q*q
 * bytes, written as S[(i*q + k)*q + a] = 1 if a is in S(i, k), else 0.
 */
AAL_API aal_status aal_block_table(int32_t law, int32_t q, uint8_t* S);

/*
 * Number of block products: row_typed != 0 -> per row type (2q - 1 for Q_q,
 * 9 for Q2xQ2); row_typed == 0 -> whole square product (2q^2 - q, 36)
 * (author's post and agihunt.info digest: 6 at q = 2 against 8 dense).
 * Returns -1 for an invalid law / q.
 */
AAL_API int64_t aal_block_product_count(int32_t law, int32_t q, int32_t row_typed);

/* ---------------------------------------------------------------------- */
/* Status, paths, version                                                  */
/* ---------------------------------------------------------------------- */

/*
 * Synchronizes ``stream``, then reads and clears the device status word of
 * the current device: AAL_OK, AAL_ERR_DEVICE_TIMEOUT or
 * AAL_ERR_DEVICE_BOUNDS (or AAL_ERR_CUDA if the synchronization failed).
 * The word is one per device, shared by every stream and thread: the first
 * error a kernel records wins until the word is read, and reading clears it.
 * Only ``stream`` is synchronized, so a kernel still running on another
 * stream may record an error after the read (it then shows up on a later
 * read), and one caller's read consumes an error another stream's kernel
 * recorded.  Synchronize the device, or every stream in use, before reading
 * when the answer must cover all of them.
 */
AAL_API aal_status aal_get_device_status(void* stream);

/* Static English description of a status code (never NULL). */
AAL_API const char* aal_status_string(int32_t status);

/*
 * Kernel-path policy for the following calls on this host thread:
 *   AAL_PATH_AUTO (0): the tensor-core path where the shape allows it, else
 *   the general CUDA path; AAL_PATH_TENSOR (1): the tensor-core path or
 *   AAL_ERR_UNSUPPORTED; AAL_PATH_GENERAL (2): always the general CUDA path.
 * aal_last_path() returns the path the last successful compute call on this
 * thread launched (1 tensor-core, 2 general, 3 decode kernel, 0 none).
 */
enum { AAL_PATH_AUTO = 0, AAL_PATH_TENSOR = 1, AAL_PATH_GENERAL = 2, AAL_PATH_DECODE = 3 };
AAL_API aal_status aal_set_path_policy(int32_t policy);
AAL_API int32_t aal_last_path(void);

/*
 * Optional timing hook for one kernel kind, for the next launch of that kind
 * on this host thread only: the library records the CUDA event ``before``
 * (a cudaEvent_t) on the call's stream just before that launch and ``after``
 * just after it, then forgets both.  Passing NULL events clears the hook.
 * During CUDA-graph capture the records become event-record nodes of the
 * graph, so the events time the launch on every replay.
 * Kinds: AAL_KERNEL_PROJECT (1, also the down projection inside
 * aal_swiglu_fwd), AAL_KERNEL_GATE_UP (2, the fused gate/up/SiLU kernel of
 * aal_swiglu_fwd), AAL_KERNEL_BWD_DX (3), AAL_KERNEL_BWD_DW (4),
 * AAL_KERNEL_SQUARE (5), AAL_KERNEL_DECODE (6, also the down decode inside
 * aal_swiglu_decode), AAL_KERNEL_DECODE_GATE_UP (7, the gate/up/SiLU decode
 * kernel of aal_swiglu_decode), AAL_KERNEL_SWIGLU_BWD (8, the dH kernel of
 * aal_swiglu_bwd with the SiLU' chain; aal_swiglu_bwd's other launches use
 * the PROJECT, BWD_DX and BWD_DW kinds), AAL_KERNEL_FFN_DECODE (9, the
 * one-launch FFN decode kernel of aal_swiglu_decode; with more than 128
 * entries the pair brackets all of the call's launches).
 */
enum { AAL_KERNEL_PROJECT = 1, AAL_KERNEL_GATE_UP = 2, AAL_KERNEL_BWD_DX = 3,
       AAL_KERNEL_BWD_DW = 4, AAL_KERNEL_SQUARE = 5, AAL_KERNEL_DECODE = 6,
       AAL_KERNEL_DECODE_GATE_UP = 7, AAL_KERNEL_SWIGLU_BWD = 8, AAL_KERNEL_FFN_DECODE = 9 };
AAL_API aal_status aal_set_timing_events(int32_t kernel, void* before, void* after);

/* Number of kernels launched by compute calls on this thread since the last
 * reset (for launch accounting). */
AAL_API int64_t aal_launch_count(int32_t reset);

/* Library version as major*10000 + minor*100 + patch. */
AAL_API int32_t aal_version(void);

/*
 * Environment switches (read once per process, except AAL_TEST_STALL).  The
 * defaults are the measured-fastest choices; the alternatives compute the
 * same products and stay available for comparison and testing.
 *   AAL_TC_PAIR=1            CTA pairs (tcgen05 cta_group::2, M = 256) for the
 *                            unswapped forward (default off: measured slower).
 *   AAL_TC_CLASS_GROUPS=0|2|4  most row types a tile of the swapped forward
 *                            holds (default 4; wider than 128 columns is never
 *                            chosen); 0 keeps one type per tile.
 *   AAL_TC_GROUP_PAIRS=0     one output group per tile on the unswapped Q_q
 *                            projection and square product (default: pairs).
 *   AAL_TC_CLASS_PAIRS=0     one row type per tile on the unswapped Q_q
 *                            projection when a type has at most 64 rows
 *                            (default: two types share a tile).
 *   AAL_DECODE_MMA=0         SIMT decode kernels instead of the tensor-core one.
 *   AAL_DECODE_TYPED=0       the cluster decode kernel for single-type batches.
 *   AAL_FFN_DECODE_FUSED=1   the one-launch FFN decode (default off: slower).
 *   AAL_TC_SIDE_BY_SIDE=0    the backward calls keep every launch on the call's
 *                            stream (default: small problems run their weight
 *                            gradients on a second stream, see above).
 *   AAL_TEST_STALL=1         test hook: the tcgen05 kernel's MMA thread waits on
 *                            a barrier nothing arrives on until the bounded
 *                            wait runs out (AAL_ERR_DEVICE_TIMEOUT); read at
 *                            every launch.
 */

#ifdef __cplusplus
}
#endif

#endif /* AAL_H_ */
