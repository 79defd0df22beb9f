/*
 * ckda.h - C ABI of the CKDA (Complex Kimi Delta Attention) library for NVIDIA B200
 * (sm_100a): chunked forward, decode step, backward pass, and the affine maps and
 * prefix of context parallelism over the sequence.
 *
 * The operation (Complex KDA: Understanding and Enhancing the Expressivity of Kimi
 * Delta Attention, as summarised by the blog post "One update, one quarter-turn",
 * section "The mirror", and by the ai.info summary, "What This Paper Is About"):
 * for every (batch b, head h) a d_k x d_v state S evolves token by token as
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                   (read after the update, no 1/sqrt(d) scale)
 *
 * with a signed per-channel gate alpha_t in [-1,1]^{d_k}, a step beta_t in [0,2]
 * and a unit key ||k_t|| = 1 (ai.info summary, "Key Contributions", Theorem 1).
 * Those ranges are preconditions on device data and are NOT checked; values outside
 * them (beta > 2, |alpha| > 1) are computed as given.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All pointers are DEVICE pointers owned by the caller. The library allocates no
 *   device memory and keeps no per-call state; the only global state is one device
 *   error word per GPU (see ckda_get_device_error), kernel attributes cached per GPU,
 *   and the fixed scratch array of ckda_chunk_fwd_noalloc (part of the module's
 *   device image).
 * - Layout is contiguous row-major, head-interleaved:
 *       q, k, alpha : [B, T, H, d_k]     v, o : [B, T, H, d_v]     beta : [B, T, H]
 *       S0, S_T, S  : [B, H, d_k, d_v]   (d_v fastest)
 *   q, k, v have the dtype named by `dt`; alpha, beta, states and o are fp32.
 * - Every base pointer must be 16-byte aligned (CKDA_ERR_MISALIGNED otherwise).
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   Calls are asynchronous on that stream and never synchronise the host, except
 *   ckda_get_device_error.
 * - Argument errors return before anything is launched. A failed launch returns
 *   CKDA_ERR_CUDA. Device-side failures (a bounded wait that ran out) are recorded
 *   in the device error word and reported by ckda_get_device_error.
 * - 1 <= d_k, d_v <= 128. T >= 0 (T = 0 writes S_T = S0 and no o).
 *
 * This header needs no CUDA or torch header.
 */
#ifndef CKDA_H_
#define CKDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CKDA_API __attribute__((visibility("default")))
#else
#define CKDA_API
#endif

#define CKDA_MAX_D 128
#define CKDA_ABI_VERSION 9

typedef enum {
    CKDA_OK = 0,
    CKDA_ERR_INVALID_ARG = 1,   /* null required pointer, bad size, bad dtype        */
    CKDA_ERR_UNSUPPORTED = 2,   /* valid request the library cannot serve            */
    CKDA_ERR_MISALIGNED = 3,    /* a base pointer is not 16-byte aligned             */
    CKDA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed              */
    CKDA_ERR_TIMEOUT = 5,       /* a device-side bounded wait ran out                */
    CKDA_ERR_WORKSPACE = 6      /* workspace missing or smaller than required        */
} ckda_status_t;

typedef enum {
    CKDA_F32 = 0,               /* q, k, v are float32                               */
    CKDA_BF16 = 1               /* q, k, v are bfloat16                              */
} ckda_dtype_t;

/* Which kernel family ckda_chunk_fwd selects for a problem. */
typedef enum {
    CKDA_PATH_RECURRENT = 0,    /* fp32 SIMT token-by-token kernel (any d <= 128)    */
    CKDA_PATH_CHUNK_TC = 1      /* chunked WY/UT kernel on tcgen05 tensor cores      */
} ckda_path_t;

/* How the gate argument of the _ex forward calls is given. */
typedef enum {
    CKDA_GATE_SIGNED = 0,       /* alpha in [-1,1]^dk: the CKDA gate, sign and magnitude   */
    CKDA_GATE_LOG = 1           /* g = ln(alpha) <= 0 of a non-negative gate (the KDA form) */
} ckda_gate_t;

/*
 * The `mode` argument of the *_ex calls and of ckda_bwd is a ckda_gate_t value,
 * optionally OR-ed with option bits:
 *   CKDA_OPT_NORMALIZE_QK: q and k are divided by their L2 norms per token and head,
 *     x / max(||x||_2, 1e-12), before the recurrence (the layer step before the path: the
 *     keys of the transition are unit vectors, ai.info summary of the Complex KDA paper,
 *     "Methodology"; the floor is torch.nn.functional.normalize's default). The
 *     normalisation is fused: the normalised values are never written to memory.
 * Unknown bits return CKDA_ERR_INVALID_ARG.
 */
#define CKDA_OPT_NORMALIZE_QK 0x100

/* Version of this ABI (CKDA_ABI_VERSION). */
CKDA_API int ckda_abi_version(void);

/* Human-readable name of a status code; never NULL, static storage. */
CKDA_API const char* ckda_status_string(ckda_status_t status);

/*
 * Bytes of device workspace ckda_chunk_fwd needs for this problem on the current
 * device (may be 0). Nonzero when the tensor-core path splits each sequence into
 * segments (few (b, h) pairs, long T): the segments' entering states and transition
 * products, B*H*nseg*dk*(dv+dk) fp32. Invalid sizes return 0; ckda_chunk_fwd then
 * rejects them.
 */
CKDA_API size_t ckda_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, ckda_dtype_t dt);

/* The path ckda_chunk_fwd takes for these sizes (for tests and reporting). */
CKDA_API ckda_path_t ckda_chunk_fwd_path(int B, int T, int H, int dk, int dv, ckda_dtype_t dt);

/*
 * Segments per sequence the tensor-core path runs side by side for these sizes on
 * the current device (1 = one pass, no workspace; for tests and reporting). A
 * segment of tokens acts on the state as the affine map S -> M S + N (the
 * recurrence's step composed over the segment); the path builds every segment's
 * M and N at once, chains the entering states, then evaluates the segments again
 * from those states. Not a step the pages describe: a scheduling choice for
 * sequences too few to fill the GPU. Returns 1 for shapes on the recurrent path.
 */
CKDA_API int ckda_chunk_fwd_segments(int B, int T, int H, int dk, int dv, ckda_dtype_t dt);

/*
 * Chunked forward (prefill / training forward without gradients).
 * Evaluates the recurrence above for all T tokens of every (b, h) and writes every
 * o_t and, if S_T != NULL, the final state. The tensor-core path splits the sequence
 * into chunks of 64 tokens and evaluates each chunk in the WY/UT form (the
 * "Chunk-WY" kernels named on the thelatestinai card) with the signed gate carried
 * as sign parity plus log-magnitude (ai.info summary, "Methodology": sign separated
 * from the log-space gate magnitude); other shapes take the recurrent path. Both
 * compute the same map; results agree with the sequential fp64 definition within
 * rounding.
 *   q, k     [B,T,H,dk] dt        v      [B,T,H,dv] dt
 *   alpha    [B,T,H,dk] fp32      beta   [B,T,H]    fp32
 *   S0       [B,H,dk,dv] fp32 or NULL (zero initial state)
 *   o        [B,T,H,dv] fp32 out
 *   S_T      [B,H,dk,dv] fp32 out or NULL; may equal S0 (in-place update)
 *   workspace: device buffer of at least ckda_chunk_fwd_workspace_bytes(...) bytes,
 *              owned by the caller (NULL allowed when that size is 0).
 * o must not overlap any input. Returns CKDA_OK or an error status (nothing launched
 * on argument errors).
 */
CKDA_API ckda_status_t ckda_chunk_fwd(const void* q, const void* k, const void* v,
                             const float* alpha, const float* beta, const float* S0,
                             float* o, float* S_T,
                             int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * ckda_chunk_fwd with the gate in the form `mode` selects. CKDA_GATE_SIGNED is
 * ckda_chunk_fwd itself. CKDA_GATE_LOG reads g = ln(alpha), fp32, in alpha's
 * [B,T,H,dk] layout, for a gate that never changes sign: the parameterisation of KDA,
 * whose gate CKDA extends from [0,1] to [-1,1] (ai.info summary of the Complex KDA paper,
 * "What This Paper Is About"). The map is the same recurrence with alpha = e^g
 * (g = -inf gives alpha = 0). It runs on the same kernels, so that CKDA's cost over KDA
 * can be measured (ai.info summary, "Main Findings": the throughput cost of the signed
 * gate). CKDA_OPT_NORMALIZE_QK may be OR-ed in (see above). An unknown mode returns
 * CKDA_ERR_INVALID_ARG.
 */
CKDA_API ckda_status_t ckda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                                const float* gate, const float* beta, const float* S0,
                                float* o, float* S_T,
                                int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                                int mode,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Capacity of the fixed device scratch ckda_chunk_fwd_noalloc uses: 20 MiB per device.
 * It is sized for a 148-SM GPU (B200), where the long-context forward (B=1, T=65536, H=16,
 * d=128) needs exactly this; the segment plan depends on the SM count, so on a GPU with
 * more SMs the same problem may need more and is then rejected. */
#define CKDA_NOALLOC_SCRATCH_BYTES ((size_t)20 << 20)

/* CKDA_NOALLOC_SCRATCH_BYTES as compiled into this library (for bindings that cannot read
 * the macro). */
CKDA_API size_t ckda_noalloc_scratch_bytes(void);

/*
 * ckda_chunk_fwd_ex without a caller-supplied workspace and without any allocation.
 * The paper has no counterpart to this call: it is a deployment variant of the
 * segmented long-sequence path. Where that path needs scratch (see
 * ckda_chunk_fwd_workspace_bytes), it uses a fixed array of
 * CKDA_NOALLOC_SCRATCH_BYTES that lives in the library's device image (allocated by
 * the CUDA runtime when the module loads on a device, never by this call); its
 * address is looked up once per device. Arguments, layouts and results are those of
 * ckda_chunk_fwd_ex; o, S_T and every input stay caller-owned.
 * Errors: CKDA_ERR_WORKSPACE, with nothing launched, when the problem needs more
 * scratch than the capacity (B*H*nseg*dk*(dv+dk)*4 > 20 MiB); otherwise as
 * ckda_chunk_fwd_ex. The scratch is one per device: calls that need it must be
 * ordered (e.g. issued on one stream); concurrent calls on unordered streams race.
 */
CKDA_API ckda_status_t ckda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                const float* gate, const float* beta, const float* S0,
                                float* o, float* S_T,
                                int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                                int mode, void* stream);

/*
 * Context parallelism over T (a sequence split over ranks in token order; the ai.info
 * summary of the Complex KDA paper, "Why This Matters", names long-context models with
 * a fixed-size recurrent state as the use). The pages describe no multi-GPU scheme:
 * this is the plainest one the recurrence allows. A slice of tokens acts on the state
 * entering it as an affine map, S_out = M S_in + N, with M (d_k x d_k) the product of
 * the slice's transitions (I - beta k k^T) Diag(alpha), last token leftmost, and N
 * (d_k x d_v) the state the slice builds from S_in = 0. Each rank after the first
 * builds its slice's map (ckda_chunk_fwd_maps), the first runs its slice directly
 * from S0; the ranks exchange (M, N) once (an all-gather: B*H*d_k*(d_k+d_v) floats per
 * rank); ckda_cp_prefix chains the maps into every rank's entering state; each rank
 * after the first then runs its slice from that state (ckda_chunk_fwd_ex) for o.
 */

/* Bytes of workspace ckda_chunk_fwd_maps needs (0 when it builds the maps in one pass):
 * few (b, h) pairs split the slice into sub-slices built side by side, which need
 * B*H*(nsub+1)*dk*(dk+dv) fp32. Invalid sizes return 0. */
CKDA_API size_t ckda_chunk_fwd_maps_workspace_bytes(int B, int T, int H, int dk, int dv, ckda_dtype_t dt);

/*
 * The affine map S_T = M S_0 + N of every (b, h) sequence of T tokens, for the gate
 * form and options in `mode` (as ckda_chunk_fwd_ex).
 *   q, k, gate [B,T,H,dk]; v [B,T,H,dv] (dtype dt); beta [B,T,H] fp32
 *   M  [B,H,dk,dk] fp32 out: the product of the transitions (T = 0: the identity)
 *   N  [B,H,dk,dv] fp32 out: the final state from a zero initial state (T = 0: zero)
 *   workspace: at least ckda_chunk_fwd_maps_workspace_bytes(...) bytes, caller-owned.
 * Tensor-core shapes (bf16, d_k, d_v in {64, 128}) run the chunk kernel with v = 0 and
 * an identity initial state for M; other shapes run the recurrent kernel the same way.
 * M and N must not overlap each other or any input. Errors as ckda_chunk_fwd_ex
 * (CKDA_ERR_INVALID_ARG for a NULL M or N).
 */
CKDA_API ckda_status_t ckda_chunk_fwd_maps(const void* q, const void* k, const void* v,
                                const float* gate, const float* beta, float* M, float* N,
                                int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                                int mode, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The exchange step's prefix, in place on the gathered maps of R ranks in token order.
 * `blocks` holds R consecutive blocks of B*H*dk*(dk+dv) fp32, block r = rank r's
 * [B,H,dk,dk] M followed by its [B,H,dk,dv] N. Block 0's N is the first rank's final
 * state (its M is not read). On return the N part of block r holds the state after
 * rank r's tokens: rank r + 1's entering state, and for r = R - 1 the sequence's final
 * state. fp32, S_{r} = M_r S_{r-1} + N_r in rank order. R = 1 is a no-op.
 * Errors: CKDA_ERR_INVALID_ARG (R < 1, bad sizes, NULL blocks), CKDA_ERR_MISALIGNED,
 * CKDA_ERR_UNSUPPORTED when dk is not a multiple of 4.
 */
CKDA_API ckda_status_t ckda_cp_prefix(float* blocks, int R, int B, int H, int dk, int dv, void* stream);

/*
 * Token-by-token forward on CUDA cores in fp32 (the recurrent path of
 * ckda_chunk_fwd, callable directly). Same arguments and semantics as
 * ckda_chunk_fwd, no workspace. Each thread keeps one state column resident in
 * registers; the state is read once and written once.
 */
CKDA_API ckda_status_t ckda_recurrent_fwd(const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta, const float* S0,
                                 float* o, float* S_T,
                                 int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                                 void* stream);

/* ckda_recurrent_fwd with the gate and options `mode` selects (see ckda_chunk_fwd_ex). */
CKDA_API ckda_status_t ckda_recurrent_fwd_ex(const void* q, const void* k, const void* v,
                                    const float* gate, const float* beta, const float* S0,
                                    float* o, float* S_T,
                                    int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                                    int mode, void* stream);

/*
 * One recurrent decode step for N independent sequences (blog post "One update,
 * one quarter-turn", section "The whiteboard": each token erases a little and writes
 * a little into a fixed-size state). Updates S in place and writes o:
 *     S <- (I - beta k k^T) Diag(alpha) S + beta k v^T,   o = S^T q   (new S)
 *   q, k   [N,H,dk] dt      v [N,H,dv] dt      alpha [N,H,dk] fp32   beta [N,H] fp32
 *   S      [N,H,dk,dv] fp32, read and written exactly once per element
 *   o      [N,H,dv] fp32 out (must not overlap S)
 */
CKDA_API ckda_status_t ckda_decode_step(const void* q, const void* k, const void* v,
                               const float* alpha, const float* beta,
                               float* S, float* o,
                               int N, int H, int dk, int dv, ckda_dtype_t dt, void* stream);

/* Which kernels ckda_bwd runs for a problem. */
typedef enum {
    CKDA_BWD_RECURRENT = 0,     /* token by token on CUDA cores, fp32 (any d <= 128, fp32 or bf16)  */
    CKDA_BWD_CHUNK_TC = 1       /* chunked on tcgen05 tensor cores (bf16, d_k and d_v in {64, 128},
                                   no CKDA_OPT_NORMALIZE_QK)                                          */
} ckda_bwd_path_t;

/* The kernels ckda_bwd runs for these sizes, dtype and mode (for tests and reporting). */
CKDA_API ckda_bwd_path_t ckda_bwd_path(int B, int T, int H, int dk, int dv, ckda_dtype_t dt, int mode);

/*
 * Bytes of device workspace ckda_bwd needs for the mode it is called with (0 for empty
 * problems or an invalid mode), all fp32.
 * CKDA_BWD_CHUNK_TC: the state entering every 64-token chunk and the cotangent of the state
 *   leaving it (2 * B*H*ceil(T/64)*dk*dv), the chunks' dWx = (I + A)^{-T} dU
 *   (B*H*ceil(T/64)*64*dv), plus the forward's segment workspace when few sequences split
 *   (ckda_chunk_fwd_workspace_bytes), each part 256-byte aligned.
 * CKDA_BWD_RECURRENT: the forward state at every 8th token (B*H*ceil(T/8)*dk*dv), recomputed
 *   states (128 KiB per (b, h) and 32-column slab of the state) and per-slab partial sums of
 *   the row gradients (slabs*B*T*H*(3*dk + 1)), where slabs = ceil(dv / 32).
 */
CKDA_API size_t ckda_bwd_workspace_bytes_ex(int B, int T, int H, int dk, int dv, ckda_dtype_t dt, int mode);

/* ckda_bwd_workspace_bytes_ex for mode CKDA_GATE_SIGNED. */
CKDA_API size_t ckda_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, ckda_dtype_t dt);

/*
 * Backward pass: the gradients of the forward map of ckda_chunk_fwd_ex for the loss
 *     L = sum_t <grad_o_t, o_t> + <grad_S_T, S_T>
 * (the vector-Jacobian product with cotangents grad_o and grad_S_T). The pages measure
 * the forward and backward passes together and mention a sign-aware backward kernel
 * (ai.info summary of the Complex KDA paper, "Main Findings"); they print no backward
 * formulas, so this is the derivative of the recurrence itself. Two implementations
 * (ckda_bwd_path): for bf16 q/k/v with d_k, d_v in {64, 128} and no q/k normalisation, the
 * chunked form on tensor cores (a forward pass that keeps every chunk's entering state, the
 * state cotangent chunk by chunk in reverse, then every chunk's gradients side by side; the
 * products split into bf16 terms as in the forward, so its error is of the bf16 forward's
 * order, not of fp32); otherwise token by token in reverse on CUDA cores in fp32 from states
 * recomputed out of checkpoints.
 *   q, k, v, gate, beta, S0, B..dv, dt, mode: as for ckda_chunk_fwd_ex (S0 may
 *              be NULL: zero initial state; any dk, dv <= 128; fp32 or bf16 q, k, v)
 *   grad_o     [B,T,H,dv] fp32 cotangent of o (required when B*T*H > 0)
 *   grad_S_T   [B,H,dk,dv] fp32 cotangent of the final state, or NULL (zero)
 *   grad_q, grad_k [B,T,H,dk] fp32 out   grad_v [B,T,H,dv] fp32 out
 *   grad_gate  [B,T,H,dk] fp32 out: dL/dalpha (CKDA_GATE_SIGNED) or dL/dg (CKDA_GATE_LOG)
 *   grad_beta  [B,T,H] fp32 out          grad_S0 [B,H,dk,dv] fp32 out, or NULL (not written)
 *   workspace  device buffer of at least ckda_bwd_workspace_bytes(...) bytes, owned by
 *              the caller.
 * Every pointer is 16-byte aligned; outputs must not overlap inputs. Returns CKDA_OK or
 * an error status (nothing launched on argument errors).
 */
CKDA_API ckda_status_t ckda_bwd(const void* q, const void* k, const void* v, const float* gate,
                                const float* beta, const float* S0, const float* grad_o,
                                const float* grad_S_T, float* grad_q, float* grad_k, float* grad_v,
                                float* grad_gate, float* grad_beta, float* grad_S0,
                                int B, int T, int H, int dk, int dv, ckda_dtype_t dt,
                                int mode, void* workspace, size_t workspace_bytes,
                                void* stream);

/* ckda_decode_step with the gate form and options `mode` selects (see ckda_chunk_fwd_ex):
 * gate holds alpha (CKDA_GATE_SIGNED) or g = ln(alpha) (CKDA_GATE_LOG), and
 * CKDA_OPT_NORMALIZE_QK divides q and k by their L2 norms inside the step. */
CKDA_API ckda_status_t ckda_decode_step_ex(const void* q, const void* k, const void* v,
                               const float* gate, const float* beta,
                               float* S, float* o,
                               int N, int H, int dk, int dv, ckda_dtype_t dt, int mode, void* stream);

/*
 * Synchronises `stream`, then reads and clears this GPU's device error word.
 * Returns CKDA_OK, CKDA_ERR_TIMEOUT (a bounded device wait ran out; the kernel
 * returned early and its outputs are invalid) or CKDA_ERR_CUDA (a sticky CUDA error;
 * the context is unusable).
 */
CKDA_API ckda_status_t ckda_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CKDA_H_ */
