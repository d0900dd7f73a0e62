/*
 * ckda.h -- C ABI of the B200 (sm_100a) gated delta-rule library.
 *
 * The recurrence, per sequence and head, token t:
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t
 *
 * transition from "Complex KDA: Understanding and Enhancing the Expressivity of
 * Kimi Delta Attention" (paper review page), section "Diagonal-plus-rank-one
 * (DPR1) transition"; the write term is the gated delta rule (CyFA blog,
 * section 2.2, with gate and strength); state S in R^{dk x dv}, row = key
 * channel, read S^T q ("Dual DeltaNet" abstract).  There is no 1/sqrt(dk)
 * scale: callers pre-scale q.
 *
 * Gate forms (signed_gate):
 *   0  KDA   alpha = sigma(a) in (0,1)^dk,    beta = sigma(b) in (0,1)
 *   1  CKDA  alpha = 2 sigma(a) - 1 in [-1,1], beta = 2 sigma(b) in [0,2]
 *            (CKDA review, "Method steps", step 1: both ranges widen together)
 *   2  raw   a holds alpha and b holds beta directly (tests and special cases)
 *   3  gate range only:      alpha = 2 sigma(a) - 1,  beta = sigma(b)
 *   4  strength range only:  alpha = sigma(a),        beta = 2 sigma(b)
 *            (3 and 4: the single-range variants of the CKDA review, "Experimental
 *            results", Figure 6)
 * Logits of +-inf are legal and exact: alpha = 0, +-1 and beta = 0, 1, 2.
 * Flags, OR-ed into signed_gate:
 *   CKDA_GATE_PER_HEAD  one gate logit per token and head: a is [B, T, H] ([B, H] for
 *            decode) and the gate alpha_t = alpha_t * 1 is shared by all key channels, the
 *            scalar (GDN-style) gate the CKDA review sets against KDA's channel-wise one
 *            (section "Scalar vs channel-wise gating").
 *   CKDA_QK_L2NORM      q and k arrive as raw projections and are divided by their L2 norm
 *            over the key channels inside the kernel (a zero vector stays zero), the fused
 *            normalisation of the review's Triton path (section "Reproducibility").
 *   CKDA_DELTA_PRODUCT2 DeltaProduct2, the review's other route to plane rotations (sections
 *            "Research motivation", "Experimental results" (5)): each token carries two keys,
 *            values and strengths, k [B, T, 2, H, dk], v [B, T, 2, H, dv], b [B, T, 2, H]
 *            (decode: [B, 2, H, .]); the gate is applied once, then the two delta-rule updates
 *            in order, then the read-out:
 *              S <- Diag(alpha_t) S;  S <- S + beta_tj k_tj (v_tj - S^T k_tj)^T, j = 1, 2;
 *              o_t = S^T q_t.
 *            Runs on the exact CUDA-core kernel; not available to ckda_chunk_bwd.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, dense and row-major.  Alignment
 *     (CKDA_ERR_ALIGN otherwise): states (S0, S_T, S) 16 bytes; b and
 *     cu_seqlens 4 bytes; ckda_chunk_fwd's q, k, v, a, o 16 bytes;
 *     ckda_decode_step's q, k, v, a, o their element size.  The caller allocates and
 *     owns every buffer, workspace included; the library never allocates,
 *     never frees and never synchronises.  Work is enqueued on `stream`
 *     (a cudaStream_t; NULL = legacy default stream) and runs asynchronously:
 *     a return of CKDA_OK means "validated and enqueued".
 *   - io_dtype (q, k, v, a) and o_dtype (o) are CKDA_F32 or CKDA_BF16.
 *     b is always float32; states are always float32.
 *   - dk, dv in {16, 32, 64, 128}.
 *   - Errors: a negative CKDA_ERR_* code, nothing enqueued, no output written.
 *     No entry point aborts, throws or traps; device-side checks (offsets in
 *     cu_seqlens, bounded waits) set a status word in the workspace that
 *     ckda_workspace_status() reads back.
 *   - NaN or Inf in q, k, v, and NaN in a or b, give undefined values but no fault.
 */
#ifndef CKDA_H
#define CKDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CKDA_OK 0
#define CKDA_ERR_NULL (-1)      /* a required pointer is NULL                      */
#define CKDA_ERR_DIM (-2)       /* dk/dv not in {16,32,64,128}, or bad B/T/H/n_seqs */
#define CKDA_ERR_CHUNK (-3)     /* chunk not in {16,32,64}                          */
#define CKDA_ERR_DTYPE (-4)     /* io_dtype / o_dtype / signed_gate out of range    */
#define CKDA_ERR_ALIGN (-5)     /* a pointer misaligned for its argument            */
#define CKDA_ERR_SEQLENS (-6)   /* cu_seqlens offsets invalid (device-detected)     */
#define CKDA_ERR_WORKSPACE (-7) /* workspace NULL or smaller than required          */
#define CKDA_ERR_TIMEOUT (-8)   /* a bounded device wait gave up                    */
#define CKDA_ERR_CUDA (-9)      /* a CUDA runtime call or kernel launch failed      */
#define CKDA_ERR_DEVICE (-10)   /* current device is not sm_100 (B200 class)        */

#define CKDA_F32 0
#define CKDA_BF16 1

#define CKDA_GATE_PER_HEAD 16  /* flag: one gate per token and head (a is [B, T, H])  */
#define CKDA_QK_L2NORM 32      /* flag: q and k are L2-normalised inside the kernel   */
#define CKDA_DELTA_PRODUCT2 64 /* flag: two rank-one delta updates per token          */

/*
 * Chunkwise (WY / UT-transform) parallel forward, "prefill".
 *
 * The CKDA review states that the DPR1 transition keeps WY chunk-wise
 * parallel training (section "Diagonal-plus-rank-one (DPR1) transition");
 * tokens are processed `chunk` at a time, the state is carried between
 * chunks, and the result equals the token-by-token recurrence.
 *
 *   q, k, a : [B, T, H, dk]  io_dtype       v : [B, T, H, dv]  io_dtype
 *            (a : [B, T, H] with CKDA_GATE_PER_HEAD)
 *   b       : [B, T, H]      float32        o : [B, T, H, dv]  o_dtype (NULL: not written)
 *   S0      : [N, H, dk, dv] float32, NULL = zero initial state
 *   S_T     : [N, H, dk, dv] float32, NULL = not written; may alias S0
 *   cu_seqlens : NULL, or int32 [n_seqs + 1] device offsets into the T axis
 *            (packed variable-length batch): B must be 1, N = n_seqs,
 *            offsets must start at 0, be non-decreasing and end at T.
 *            Without it N = B and every batch row is one sequence of T tokens.
 *            Offsets are checked on the device: a bad sequence is skipped
 *            and CKDA_ERR_SEQLENS is recorded in the workspace status word.
 *            B * T must not exceed 2^31 - 1 (token rows are addressed with
 *            32-bit coordinates); larger calls return CKDA_ERR_DIM.
 *   chunk   : 16, 32 or 64 tokens per chunk (a ragged last chunk is fine;
 *            chunks never span two sequences).
 *   workspace : device scratch, 256-byte aligned, of at least 256 bytes (the
 *            status header); owned by the caller, reused freely between calls
 *            on the same stream, never shared by two calls in flight at once.
 *            With ckda_chunk_fwd_workspace_size() bytes, the tensor-core path
 *            (1) hands a (sequence, head) whose gates decay faster than its range
 *            (a chunk product below 2^-100 in some channel) to a second launch
 *            that carries per-channel references and stays on the tensor
 *            cores; with less, such chunks run token by token (exact, slower);
 *            (2) cuts the one or two longest sequences of a batch into
 *            segments when their serial chunk walk would bound the call (a
 *            packed batch with one long document, a short batch of long
 *            sequences): the segments run in parallel from a zero and an
 *            identity state, their affine state maps are chained on the
 *            device, and the segments run again from their true states (the
 *            DPR1 transition of the CKDA review is linear in the state).  The
 *            result is the same recurrence; with less workspace nothing is cut.
 *   stream  : cudaStream_t.
 * Returns CKDA_OK or a negative CKDA_ERR_* code.
 */
int ckda_chunk_fwd(const void *q, const void *k, const void *v, const void *a, const float *b,
                   const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                   int dk, int dv, int chunk, int signed_gate, int io_dtype, int o_dtype,
                   void *o, float *S_T, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace ckda_chunk_fwd uses in full for these sizes (same
 * meaning as there; n_seqs > 0 means a packed batch of n_seqs sequences, else
 * B sequences of T tokens): 256 for the exact path; for dk = dv = 128 and
 * chunk 64 also a 16-byte queue entry and a 64 KB saved state per unit of
 * one launch for the hand-off above, and, where sequences may be cut (every
 * packed batch of at most 1024 sequences; an unpacked batch whose walk the cut
 * shortens on a 148-SM B200), the unit lists and 26 state slots per head.
 * Pure host arithmetic, no CUDA call.
 */
size_t ckda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk,
                                     int n_seqs);

/*
 * Chunkwise backward of ckda_chunk_fwd: the gradients of
 *   L = sum dO . o + sum dS_T . S_T
 * with respect to q, k, v, the gate logits a, the strength logits b and S0.
 * The CKDA review measures its kernels forward plus backward ("Experimental
 * results", Figure 5: CKDA at 96-97 % of KDA's throughput); it gives no
 * backward formulas, so this is the chain rule of the forward above (the
 * chunkwise UT form walked in reverse), exact fp32 arithmetic on CUDA cores,
 * including exact zero gates (an exact zero gate's gradient is the derivative
 * of L at that gate, which L, affine in each gate, has everywhere).
 *
 *   q, k, v, a, b, S0, cu_seqlens, n_seqs, B, T, H, dk, dv, signed_gate,
 *   io_dtype : as ckda_chunk_fwd (the chunk size is the library's own).
 *   dO    : [B, T, H, dv] in do_dtype (CKDA_F32 or CKDA_BF16); NULL = zero.
 *   dS_T  : [N, H, dk, dv] float32; NULL = zero.
 *   dq, dk_out, da : [B, T, H, dk] float32     dv_out : [B, T, H, dv] float32
 *            (da : [B, T, H] with CKDA_GATE_PER_HEAD; with CKDA_QK_L2NORM dq and dk_out
 *            are the gradients with respect to the raw, un-normalised q and k)
 *   db    : [B, T, H] float32                   (all required, every row written)
 *   dS0   : [N, H, dk, dv] float32, or NULL (not written)
 *   workspace : device scratch of ckda_chunk_bwd_workspace_size() bytes (it holds
 *            the state and the state gradient at every chunk boundary and each chunk's
 *            state-independent factors), 256-byte
 *            aligned, owned by the caller; its status word is read with
 *            ckda_workspace_status (bad cu_seqlens: the sequence's gradients are
 *            not written).
 * Returns CKDA_OK or a negative CKDA_ERR_* code; arguments are checked as by
 * ckda_chunk_fwd (B * T <= 2^31 - 1, 16-byte alignment of every tensor).
 */
int ckda_chunk_bwd(const void *q, const void *k, const void *v, const void *a, const float *b,
                   const float *S0, const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                   int dk, int dv, int signed_gate, int io_dtype, const void *dO, int do_dtype,
                   const float *dS_T, float *dq, float *dk_out, float *dv_out, float *da,
                   float *db, float *dS0, void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace ckda_chunk_bwd needs (host arithmetic, no CUDA call). */
size_t ckda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs);

/*
 * One recurrent decode step for B x H heads: the recurrence above for a
 * single token, applied to the state in place.  The CKDA review notes the
 * extended ranges add no per-token inference cost (section "Research
 * motivation"); the step reads and writes each head's fp32 state once.
 *
 *   q, k, a : [B, H, dk] io_dtype     v : [B, H, dv] io_dtype     b : [B, H] float32
 *            (a : [B, H] with CKDA_GATE_PER_HEAD)
 *   S       : [B, H, dk, dv] float32, updated in place (S_{t-1} -> S_t)
 *   o       : [B, H, dv] o_dtype, o = S_t^T q (NULL: not written)
 * Returns CKDA_OK or a negative CKDA_ERR_* code.
 */
int ckda_decode_step(const void *q, const void *k, const void *v, const void *a, const float *b,
                     float *S, int B, int H, int dk, int dv, int signed_gate, int io_dtype,
                     int o_dtype, void *o, void *stream);

/*
 * ckda_chunk_fwd without a caller-provided workspace.  The pages describe no
 * such call; it exists for callers that cannot allocate device memory at all,
 * for example a serving runtime that plans all device memory at start-up and
 * forbids later allocations, or plain C code that links only this library
 * and has no device allocator.  Arguments, layouts and results are those of
 * ckda_chunk_fwd; the workspace is replaced by a fixed 4096-byte scratch array
 * compiled into the library (every GPU that loads the library holds it until
 * the process exits).  The scratch holds the status header only, so chunks
 * whose gates decay past the tensor-core kernel's range run token by token
 * (no hand-off) and no sequence is cut into segments.  Neither this call nor
 * the library calls cudaMalloc or cudaFree.
 *   - Every call looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with the caller's device current, so the address
 *     is never stale.  The first call on a device may load the library's
 *     device code there; make that first call before any stream capture.
 *   - Every call on a device shares the same scratch, and it keeps what the
 *     last call left there; the status header is cleared on `stream` at the
 *     start of each call.  Calls whose work overlaps on the GPU (different
 *     streams without ordering) race on the scratch: serialise them.
 *   - The device status word (bad cu_seqlens, timeouts) of the last call is
 *     read back with ckda_noalloc_status().
 * Returns CKDA_OK or a negative CKDA_ERR_* code.
 */
int ckda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *a,
                           const float *b, const float *S0, const int32_t *cu_seqlens, int n_seqs,
                           int B, int T, int H, int dk, int dv, int chunk, int signed_gate,
                           int io_dtype, int o_dtype, void *o, float *S_T, void *stream);

/*
 * The device status word of the last ckda_chunk_fwd_noalloc call on the current
 * device (CKDA_OK, CKDA_ERR_SEQLENS or CKDA_ERR_TIMEOUT), read from the
 * library's scratch array into *status.  Like ckda_chunk_fwd_noalloc this has no
 * counterpart on the pages.  It SYNCHRONISES `stream` (a 4-byte copy to the
 * host) and allocates nothing.  Returns CKDA_OK or CKDA_ERR_NULL / CKDA_ERR_CUDA.
 */
int ckda_noalloc_status(int *status, void *stream);

/*
 * Reads the device status word that ckda_chunk_fwd records in `workspace`
 * (CKDA_OK, CKDA_ERR_SEQLENS or CKDA_ERR_TIMEOUT) into *status.  This call
 * SYNCHRONISES `stream` (it copies 4 bytes to the host).  Returns CKDA_OK or
 * CKDA_ERR_NULL / CKDA_ERR_CUDA.
 */
int ckda_workspace_status(const void *workspace, int *status, void *stream);

/*
 * TEST HOOK for the failure path of the bounded device waits; not needed in
 * normal use.  After ckda_debug_wait_injection(chunk_index, wait_ns) with
 * chunk_index >= 0, every later ckda_chunk_fwd call that runs on the
 * tensor-core kernel (bf16 inputs, dk = dv = 128, chunk 64) adds, in every
 * (sequence, head) unit that reaches chunk number `chunk_index`, one wait at
 * the start of that chunk on a barrier that nothing ever arrives on, bounded
 * by `wait_ns` nanoseconds (0 = the normal 2 s bound).  The wait runs out, the
 * unit abandons its work (outputs of that unit are left unwritten or partial),
 * lets every copy and product it started finish, releases its tensor memory
 * and records CKDA_ERR_TIMEOUT in the status word.  chunk_index < 0 switches
 * the hook off (the default).  Process-wide; takes effect at the next launch.
 */
void ckda_debug_wait_injection(int chunk_index, unsigned long long wait_ns);

/*
 * TEST HOOK for the segment cut of ckda_chunk_fwd (workspace item (2));
 * not needed in normal use.  After ckda_debug_segment_split(n_split,
 * n_segments) with 1 <= n_split <= 2 and 3 <= n_segments <= 8, every later
 * packed ckda_chunk_fwd call on the tensor-core kernel whose workspace has
 * ckda_chunk_fwd_workspace_size() bytes cuts its n_split longest sequences
 * into n_segments segments (fewer when a sequence has fewer chunks; a
 * sequence of under three chunks is not cut) whatever the cost model says.
 * Other arguments switch the hook off (the default: the cost model decides).
 * Process-wide; takes effect at the next launch.
 */
void ckda_debug_segment_split(int n_split, int n_segments);

/*
 * TEST HOOK: what the segment cut's cost model decides for a packed batch of
 * n_seqs sequences of lengths[0 .. n_seqs) tokens with H heads on sm_count
 * SMs (host arithmetic, no CUDA call; the device planner evaluates the same
 * model).  *n_cut receives the number of sequences cut (0, 1 or 2: the
 * longest ones), segments[0..1] how many segments each (0 past *n_cut).
 * Returns CKDA_OK, CKDA_ERR_NULL or CKDA_ERR_DIM (n_seqs outside
 * [0, 1024], H or sm_count not positive, a negative length).
 */
int ckda_debug_segment_choice(const int32_t *lengths, int n_seqs, int H, int sm_count,
                              int *n_cut, int *segments);

/* Static, human-readable text for a status code (never NULL). */
const char *ckda_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int ckda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CKDA_H */
