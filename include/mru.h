/*
 * mru.h -- C-ABI of libmru.so, the B200 (sm_100a) Matrix Recurrent Unit
 * prefix-product scan.
 *
 * The operation ("MRU Update: An independent developer's alternative to
 * Attention is now running successfully", section "What MRU Actually Does"):
 * every token's embedding slice is lifted to an n x n input state matrix X_t,
 * and the states are the cumulative products along the sequence,
 *
 *     S_t = S_{t-1} . X_t,     S_0 = I (or a caller-given S0),
 *
 * computed as a parallel scan because matrix multiplication is associative.
 * Construction modes ("Improving Matrix Recurrent Units as an Attention
 * Alternative", "Key Points" / "Technical Deep Dive"):
 *   RESHAPE  Xr = add_identity*I + alpha*M, X = Xr;
 *   DETNORM  X = Xr / |det Xr|^(1/n)   (determinant-correcting scalar; the
 *            sign of det Xr is kept; det Xr = 0 or not finite is an error);
 *   LDU      X = L D U, L = I + ldu_offdiag*strict_lower(M),
 *            U = I + ldu_offdiag*strict_upper(M),
 *            D = diag(exp(ldu_diag*tanh(M_ii)));
 *   CAYLEY   X = (I - A)^-1 (I + A), and
 *   EXPM     X = exp(A), with A = alpha (M - M^T) / 2, the skew-symmetric
 *            part of alpha M (the orthogonal constructions the pages report
 *            tried, "Key Points"); X is orthogonal with det X = 1.
 *            add_identity is not used.  These two run on the generic fp32
 *            kernels for every n.
 * M is the head's slice x[b, t, h*n*n : (h+1)*n*n] viewed row-major as n x n.
 *
 * Layouts (all row-major, contiguous, C order):
 *   x        [B, L, H*n*n]   float32 or bfloat16 (per x_dtype)      device
 *   X, F     [B, L, H, n, n] float32                                 device
 *   S0       [B, H, n, n]    float32, or NULL for the identity       device
 *   S_out    [B, L, H, n, n] float32; memory position t holds S_{t+1} device
 *   u        [n, q], or [H, n, q] with u_per_head: the readout's query
 *            columns U (q = 1: one vector u), float32                device
 *   o_out    [B, L, H, n, q] float32, o_t = S_t . U (the head's U)    device
 *   snapshots [B, L/every, H, n, n] float32, S_t at 1-based t = k*every device
 *
 * Ownership and execution: the caller owns every buffer (the library never
 * allocates or frees device memory); calls are asynchronous on `stream`
 * (a cudaStream_t passed as void*; NULL is the legacy default stream).
 * Buffers must be 16-byte aligned and x/X must not alias any output.
 *
 * Errors: argument problems are returned synchronously and nothing is
 * launched.  Conditions found on the device (a singular matrix in DETNORM
 * mode) are recorded in a status word inside the workspace and read with
 * mru_last_device_status(), which synchronises the stream.  Nothing throws
 * across this boundary.
 */
#ifndef MRU_H_
#define MRU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MRU_OK = 0,
    MRU_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned buffer, bad enum */
    MRU_ERR_UNSUPPORTED = 2,  /* n not in {4, 8, 16, 32, 64}, or an unsupported combination */
    MRU_ERR_WORKSPACE = 3,    /* workspace smaller than mru_workspace_size() */
    MRU_ERR_CUDA = 4,         /* a CUDA launch or copy failed */
    MRU_ERR_SINGULAR = 5,     /* DETNORM met det = 0 or a non-finite determinant */
    MRU_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up (recorded in the status word) */
} mru_status;

typedef enum {
    MRU_MODE_RESHAPE = 0, MRU_MODE_DETNORM = 1, MRU_MODE_LDU = 2,
    MRU_MODE_CAYLEY = 3,  /* X = (I - A)^-1 (I + A), A = alpha (M - M^T) / 2 */
    MRU_MODE_EXPM = 4     /* X = exp(A),             A = alpha (M - M^T) / 2 */
} mru_mode;
typedef enum { MRU_F32 = 0, MRU_BF16 = 1 } mru_dtype;
typedef enum {
    MRU_MATH_AUTO = 0,    /* library choice per n and dtype (fp32-accurate) */
    MRU_MATH_FP32 = 1,    /* fp32 FMA throughout (the generic kernels) */
    MRU_MATH_TF32 = 2,    /* tensor-core products with tf32 operands, fp32 accumulate */
    MRU_MATH_TF32X3 = 3,  /* split-tf32 (hi/lo, three products), fp32 accumulate */
    MRU_MATH_BF16X3 = 4   /* split-bf16 (hi/lo, three products), fp32 accumulate */
    /* A mode without a specialised kernel for the problem's n and dtype runs
     * the fp32 kernels, which are at least as accurate. */
} mru_math;

typedef struct {
    int64_t B, H, L;            /* batch, heads, sequence length (>= 0) */
    int32_t n;                  /* matrix side: 4, 8, 16, 32 or 64 */
    int32_t x_dtype;            /* mru_dtype of x */
    int32_t mode;               /* mru_mode */
    int32_t math;               /* mru_math */
    float alpha;                /* RESHAPE / DETNORM: Xr = add_identity*I + alpha*M */
    int32_t add_identity;       /* 0 or 1 */
    float ldu_offdiag;          /* LDU: off-diagonal scale of L and U */
    float ldu_diag;             /* LDU: D_ii = exp(ldu_diag * tanh(M_ii)) */
    int32_t store_minus_identity; /* mru_build_states writes F = X - I; mru_scan reads F */
    int32_t chunk;              /* tokens per scan chunk; 0 = library choice, else >= 1 */
} mru_problem;

/* The readout ("dimension reduction": the state matrix turned back into a
 * vector, "MRU Update: An independent developer's alternative to Attention
 * is now running successfully", section "What MRU Actually Does").  The
 * pages leave its form open; here it is a set of q query columns,
 * o_t = S_t U (n x q per token and head), one U for all heads or one per
 * head.  q = 1 is the single readout vector o_t = S_t u. */
typedef struct {
    const float* u;             /* [n, q], or [H, n, q] with u_per_head: query columns U (device) */
    int64_t snapshot_every;     /* 0: no snapshots; else > 0, floor(L/every) snapshots per (b, h) */
    float* snapshots;           /* [B, L/every, H, n, n] (device), ignored when every == 0 */
    int32_t q;                  /* query columns, 1 <= q <= n; 0 is read as 1 */
    int32_t u_per_head;         /* 0: one U shared by every head; 1: U[h] for head h */
} mru_readout;

/* Bytes of device workspace a call on this problem needs (>= 256: the first
 * 256 bytes hold the device status word).  Returns 0 for an invalid problem. */
size_t mru_workspace_size(const mru_problem* p);

/* Lift only: X_out[b,t,h] = X_t (or F = X_t - I when store_minus_identity).
 * Construction as listed above.  ws: at least mru_workspace_size(p) bytes. */
mru_status mru_build_states(const mru_problem* p, const void* x, float* X_out,
                            void* ws, size_t ws_bytes, void* stream);

/* Scan only: S_out[b,t,h] = S0[b,h] . X_1 ... X_{t+1} from given matrices X
 * (or F = X - I when store_minus_identity; the identity-split form keeps the
 * product accurate for near-identity inputs).  x_dtype/mode are ignored. */
mru_status mru_scan(const mru_problem* p, const float* X, const float* S0, float* S_out,
                    void* ws, size_t ws_bytes, void* stream);

/* Lift + scan fused: construction from x happens inside the scan.  With
 * ro == NULL every state is written to S_out (o_out unused, may be NULL).
 * With ro != NULL the states are reduced instead: o_out[b,t,h] = S_t . U
 * ([n, q] per token and head), and S_t is stored to ro->snapshots at
 * t = every, 2*every, ... (S_out unused).  q outside [0, n] or u_per_head
 * outside {0, 1} is MRU_ERR_INVALID_ARG.
 * With MRU_N64_TCGEN05=1 in the environment (read at each call) the n = 64
 * readout path runs its chunk phase on the fifth-generation tensor cores
 * (tcgen05.mma into tensor memory) instead of mma.sync: the same results
 * within the tf32 gate, slower on B200, so not the default. */
mru_status mru_scan_fused(const mru_problem* p, const void* x, const float* S0,
                          const mru_readout* ro, float* S_out, float* o_out,
                          void* ws, size_t ws_bytes, void* stream);

/* mru_scan_fused from and to HOST buffers, the upload, the scan and the
 * download pipelined: the problem is cut into `pieces` parts (0: the
 * library's choice, 8), along the batch when B >= 2, else along the sequence
 * in whole chunks (each part started from the previous part's last state;
 * with the readout and B = 1 there is one part).  Part i's upload runs on
 * h2d_stream while part i - 1 is scanned on compute_stream and part i - 2
 * downloads on d2h_stream, so that the two copy directions and the kernels
 * overlap.  Work queued on compute_stream before the call finishes before the
 * first copy starts, and the call is complete (outputs in host memory) when
 * compute_stream reaches its end: synchronise that stream before reading.
 *   x_host     [B, L, H*n*n] host (pinned memory for full speed), as x
 *   out_host   [B, L, H, n, n] (ro == NULL) or [B, L, H, n, q] (ro) host
 *   snaps_host [B, L/every, H, n, n] host when ro->snapshot_every > 0,
 *              downloaded from ro->snapshots (device staging), else unused
 *   x_dev      device staging of x's size; out_dev device staging of
 *              out_host's size (16-byte aligned, distinct)
 *   S0, ro->u  device, as in mru_scan_fused
 * The three streams may be the same (no overlap then).  Events are created
 * and released inside the call; no memory is allocated.  Results are
 * bit-identical to mru_scan_fused when the cut is along the batch; along the
 * sequence the parts' boundaries round the state to fp32 once more. */
mru_status mru_scan_fused_host(const mru_problem* p, const void* x_host, const float* S0, const mru_readout* ro,
                               float* out_host, float* snaps_host, void* x_dev, float* out_dev, void* ws,
                               size_t ws_bytes, int32_t pieces, void* compute_stream, void* h2d_stream,
                               void* d2h_stream);

/* Backward (vector-Jacobian product) of mru_scan_fused without the readout.
 * The pages train the MRU but print no gradient: this is the chain rule of
 * the forward definition ("MRU Update: An independent developer's
 * alternative to Attention is now running successfully", section "What MRU
 * Actually Does": S_t = S_{t-1} X_t; construction variants from "Improving
 * Matrix Recurrent Units as an Attention Alternative", "Technical Deep
 * Dive").  With G_t = dL/dS_t (later states included):
 *   G_L = dS_L,  G_{t-1} = dS_{t-1} + G_t X_t^T,
 *   dL/dX_t = S_{t-1}^T G_t,  dL/dS0 = G_1 X_1^T,
 * then through the construction of X_t from the embedding slice M:
 *   reshape: alpha dX;  determinant-corrected (X = c Xr):
 *   alpha c (dX - <dX, Xr> Xr^-T / n);  LDU: through L, D and U;
 *   Cayley: dA = 2 W^-T dX W^-T (W = I - A);  exponential: dA = L(A^T, dX),
 *   the Frechet derivative of exp at A^T;  then dM = alpha (dA - dA^T) / 2.
 *   x      [B, L, H*n*n] the forward's embeddings (f32 or bf16)
 *   S0     [B, H, n, n] fp32 or NULL (identity), as in the forward
 *   S_fwd  [B, L, H, n, n] fp32, the forward's states (mru_scan_fused output)
 *   dS     [B, L, H, n, n] fp32 upstream gradients of every S_t
 *   dx     [B, L, H*n*n] fp32 out: gradient with respect to the (widened)
 *          embedding values
 *   dS0    [B, H, n, n] fp32 out, or NULL
 * Every pointer 16-byte aligned; dx and dS0 alias no input.  The workspace
 * holds mru_backward_workspace_size(p) bytes.  fp32-accurate arithmetic for
 * every n and mode unless tf32 is asked for: fp32 on the generic kernels,
 * split tf32 on the tensor cores for n = 16 (fp32 embeddings, reshape,
 * corrected with the identity, or the Cayley map), three-term split bf16 for n = 32 LDU (bf16
 * embeddings, exact in bf16).  n = 64 with p->math = MRU_MATH_TF32 (fp32
 * embeddings, reshape or determinant-corrected): tf32 products on the
 * tensor cores, the forward's tf32 arithmetic (chunks of 64 tokens by
 * default).  fp64 for the right-to-left scan of the chunk gradients.  A
 * singular matrix sets MRU_ERR_SINGULAR in the workspace status word. */
size_t mru_backward_workspace_size(const mru_problem* p);
mru_status mru_scan_backward(const mru_problem* p, const void* x, const float* S0, const float* S_fwd,
                             const float* dS, float* dx, float* dS0, void* ws, size_t ws_bytes,
                             void* stream);

/* Backward of mru_scan_fused WITH the readout: the gradient with respect to
 * the embeddings (and S0) of a loss of the readout's outputs, given their
 * gradients, without any state stored by the caller.  The readout maps the
 * state back to vectors ("MRU Update: An independent developer's alternative
 * to Attention is now running successfully", section "What MRU Actually
 * Does", step 3); its chain rule, o_t = S_t U, gives every state the upstream
 * gradient
 *   dL/dS_t = do_t U^T  (+ dP_k at 1-based t = k * every),
 * and the scan's backward (mru_scan_backward) takes it from there.  The
 * call recomputes the states with the forward scan into the workspace, forms
 * those gradients there, and runs the backward.
 *   x      [B, L, H*n*n] the forward's embeddings (f32 or bf16)
 *   S0     [B, H, n, n] fp32 or NULL (identity), as in the forward
 *   ro     the forward's readout: u, q, u_per_head, snapshot_every
 *          (ro->snapshots is not used)
 *   d_o    [B, L, H, n, q] fp32 gradients of the readout outputs o_t
 *   d_snaps [B, L/every, H, n, n] fp32 gradients of the snapshots, or NULL
 *          (no snapshot term; ignored when ro->snapshot_every == 0)
 *   dx     [B, L, H*n*n] fp32 out;  dS0 [B, H, n, n] fp32 out, or NULL
 * Every pointer 16-byte aligned; dx and dS0 alias no input.  The workspace
 * holds mru_backward_readout_workspace_size(p) bytes (twice the states'
 * size plus the backward's own); the status word is at its start, as for
 * every other call.  Arithmetic as mru_scan_backward's. */
size_t mru_backward_readout_workspace_size(const mru_problem* p);
mru_status mru_scan_backward_readout(const mru_problem* p, const void* x, const float* S0, const mru_readout* ro,
                                     const float* d_o, const float* d_snaps, float* dx, float* dS0, void* ws,
                                     size_t ws_bytes, void* stream);

/* Synchronises `stream` and returns the device-detected status of the last
 * call that used this workspace: MRU_OK, MRU_ERR_SINGULAR, or
 * MRU_ERR_TIMEOUT when a bounded wait of one of the opt-in kernels gave up
 * (the single-read n = 16 kernel's carry waits, the n = 64 tcgen05 kernel's
 * tensor-core waits; outputs are then unspecified, the CUDA context stays
 * usable). */
mru_status mru_last_device_status(const void* ws, void* stream);

/* Testing hook for the bounded waits of the single-read n = 16 kernel.  With
 * MRU_N16_FUSED=1 in the environment (read at each call), mru_scan_fused for
 * n = 16, fp32, reshape / DETNORM / CAYLEY / EXPM and more than one chunk per
 * sequence runs one persistent kernel that reads x from HBM once instead of
 * the three passes (it is correct but, on B200, still slower; the passes
 * stay the default).  Its warps wait on one another in two
 * places only: a group of chunks looking back for the aggregates of the
 * groups before it, and an apply item waiting for its group's carry; every
 * wait gives up after a time limit (2 s), records MRU_ERR_TIMEOUT in the
 * status word and makes the launch end early.  After this call, the next
 * such launch in the process never publishes the carry of its first group
 * and uses a limit of `ms` milliseconds (> 0), so that it ends with
 * MRU_ERR_TIMEOUT without any fault; ms <= 0 cancels a pending request. */
void mru_debug_stall_next_fused(int32_t ms);

/* Static string for a status code. */
const char* mru_status_string(mru_status s);

/* The mru_math the kernels chosen for this problem compute in
 * (MRU_MATH_FP32 for the generic fp32 kernels, MRU_MATH_TF32X3 or
 * MRU_MATH_BF16X3 for the tensor-core kernels); -1 if p is invalid. */
int32_t mru_effective_math(const mru_problem* p, int32_t readout);

/* Chunk length the library would use for this problem, with the readout
 * (readout != 0) or with every state written (0 if p is invalid). */
int32_t mru_chosen_chunk(const mru_problem* p, int32_t readout);

/* Number of kernel launches one call of mru_scan_fused makes for p. */
int32_t mru_launch_count(const mru_problem* p, int32_t readout);

/* Name of the i-th kernel one call of mru_scan_fused launches for p (with the
 * readout when readout != 0); "" when i is out of range or p is invalid. */
const char* mru_kernel_name(const mru_problem* p, int32_t readout, int32_t i);

/* Benchmark hook.  With count > 0, every later mru_scan / mru_scan_fused call
 * records events[2*i] just before and events[2*i+1] just after its i-th
 * kernel launch (for i < count/2), on the call's stream, so that the caller
 * can time each kernel with cudaEventElapsedTime.  The cudaEvent_t handles
 * are created and owned by the caller; count <= 64.  events == NULL or
 * count == 0 switches the hook off.  Process-wide; not thread-safe. */
mru_status mru_set_profile_events(void* const* events, int32_t count);

/* Size of the fixed device scratch that mru_scan_fused_noalloc uses (16 MiB). */
#define MRU_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* mru_scan_fused without a workspace argument, for callers that may not
 * allocate device memory at all: a plugin inside a host framework that owns
 * every device allocation, or a service that reserves its whole memory budget
 * at start-up and forbids allocation afterwards.  The method's pages have no
 * counterpart to this entry point; it exists for such callers only.
 *
 * Arguments and results are those of mru_scan_fused; the caller still owns
 * x, S0, the readout buffers, S_out and o_out.  The scratch is one
 * file-scope device array of MRU_NOALLOC_SCRATCH_BYTES, held by every GPU
 * whose context loads this library until the process exits.  The call
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library call).
 *
 *   - Size limit: with p->chunk == 0 the chunk is the library's choice,
 *     doubled until the workspace this call needs (its output form and
 *     readout layout; at most mru_workspace_size) fits the scratch; a
 *     problem that does not fit even then, or whose explicit p->chunk does not
 *     fit, is rejected with MRU_ERR_WORKSPACE before anything is launched.
 *   - Set-up: every call looks up the scratch's device address on the
 *     current device (cudaGetSymbolAddress; nothing is cached, so the lookup
 *     stays right after a device reset); the first call on a device also
 *     loads the module there, so make it before any stream capture.
 *   - Sharing: every call on a device uses the same scratch, which keeps the
 *     last call's contents; the call clears what must start at zero itself.
 *     Calls whose executions overlap on the GPU (on different streams, or
 *     from different host threads) race on the scratch: serialise them.
 *   - Status: when status_out (a device pointer to one uint32, 4-byte
 *     aligned) is not NULL, the device status word is copied there on the
 *     stream after the scan: 0 ok, bit 0 singular matrix, bit 1 timeout.
 */
mru_status mru_scan_fused_noalloc(const mru_problem* p, const void* x, const float* S0,
                                  const mru_readout* ro, float* S_out, float* o_out,
                                  uint32_t* status_out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MRU_H_ */
