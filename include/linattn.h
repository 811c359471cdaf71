/*
 * linattn: linear attention with the feature map phi(x) = elu(x) + 1 on NVIDIA B200
 * (sm_100a).  C ABI; every entry point is asynchronous on the caller's CUDA stream.
 *
 * The method (page "Efficient Transformers: Linear Attention and Flash Attention",
 * section "Linear attention: reordering the matmuls, not shrinking them", the kernelised
 * attention formula):
 *
 *     out_i = phi(q_i) S / (phi(q_i) . z),   S = sum_j phi(k_j) v_j^T (D x d),
 *                                            z = sum_j phi(k_j)       (D)
 *
 * computed in the associativity-reordered order, so the n x n matrix is never formed.
 * Causal attention sums over j <= i, the current token included, as in the same page's
 * section "The recurrent view: attention as an RNN" (S_t = S_{t-1} + phi(k_t) v_t^T and
 * the output at t reads S_t).  phi(x) = x + 1 for x > 0 and exp(x) for x <= 0.
 * There is no 1/sqrt(d) scale and no epsilon inside the method: callers pre-scale
 * their inputs if they want one, and phi > 0 keeps the denominator positive.
 *
 * Dimensions: the feature dimension D equals the head dimension d (phi is elementwise)
 * and the value dimension equals d.  Supported d: 64 and 128.
 *
 * Memory: every pointer is caller-owned DEVICE memory, 16-byte aligned.  The library
 * keeps no pointer after a call returns.  Outputs must not alias inputs.  Temporary
 * workspace is taken from a library-owned stream-ordered pool on the caller's stream
 * and released on the same stream.
 *
 * Errors: every argument is checked before anything is launched; a failed check
 * returns LINATTN_ERR_INVALID_ARG or LINATTN_ERR_UNSUPPORTED and launches nothing.
 * A CUDA error at launch returns LINATTN_ERR_CUDA.  Kernels never trap: a bounded wait
 * that gives up sets a per-device error flag, which linattn_device_error() reports as
 * LINATTN_ERR_TIMEOUT after synchronising the stream.
 */
#ifndef LINATTN_H
#define LINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's stream handle type (cudaStream_t is a typedef of this pointer). */
struct CUstream_st;
typedef struct CUstream_st *linattn_stream_t;

typedef enum {
    LINATTN_OK = 0,
    LINATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, size <= 0, bad flag or dtype */
    LINATTN_ERR_UNSUPPORTED = 2, /* d outside {64, 128} */
    LINATTN_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    LINATTN_ERR_TIMEOUT = 4      /* a kernel's bounded wait gave up (see linattn_device_error) */
} linattn_status;

typedef enum {
    LINATTN_F32 = 0, /* float32 I/O: computed in fp32 on the CUDA cores */
    LINATTN_BF16 = 1 /* bfloat16 I/O: the forward runs bf16 tensor-core products with fp32
                        accumulation and state; the backward runs on the CUDA cores in fp32 */
} linattn_dtype;

/*
 * Forward pass over B*H independent heads.
 *   q, k, v : [B][H][n][d] row-major, element type `dtype`, read only.
 *   out     : [B][H][n][d] row-major, element type `dtype`, written.
 *   causal  : 0 = every query sees every key (the formula above);
 *             1 = query i sees keys j <= i (the recurrent view's running state).
 * Any n >= 1 is accepted.  Accumulation is fp32; the output is rounded once to `dtype`
 * (bf16: round to nearest even).  The causal mode runs as chunked prefix sums of (S, z):
 * per-segment aggregates, their exclusive scan, then the outputs of every segment from its
 * prefix.  Returns LINATTN_OK after enqueuing the work on `stream`.
 */
linattn_status linattn_forward(const void *q, const void *k, const void *v, void *out,
                               int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                               linattn_dtype dtype, linattn_stream_t stream);

/*
 * One recurrent decode step for Bseq*H independent states (the recurrent view):
 *   S' = S + phi(k) v^T,  z' = z + phi(k),  out = phi(q) S' / (phi(q) . z').
 * The output reads the UPDATED state (the current token is included).
 *   state_S : [Bseq][H][D][d] float32, row r = feature index, column c = value index;
 *             read and written in place.
 *   state_z : [Bseq][H][D] float32, read and written in place.
 *   q, k, v : [Bseq][H][d] bfloat16, read only.   out : [Bseq][H][d] bfloat16, written.
 * The state is the caller's: keeping the two buffers is all a pause/resume needs.
 */
linattn_status linattn_decode_step(float *state_S, float *state_z, const void *q,
                                   const void *k, const void *v, void *out, int64_t Bseq,
                                   int64_t H, int64_t d, linattn_stream_t stream);

/*
 * The state a causal pass leaves after its last token, per head:
 *   state_S[b][h] = sum_j phi(k_j) v_j^T  ([D][d] float32),
 *   state_z[b][h] = sum_j phi(k_j)        ([D] float32),
 * with k, v : [B][H][n][d] of type `dtype`.  This is the prefill that hands a sequence
 * over to linattn_decode_step (the recurrent view's S_n, z_n).  Overwrites both outputs.
 */
linattn_status linattn_forward_state(const void *k, const void *v, float *state_S,
                                     float *state_z, int64_t B, int64_t H, int64_t n,
                                     int64_t d, linattn_dtype dtype, linattn_stream_t stream);

/*
 * linattn_forward continued from a given state: the pass over tokens [0, n) of each head
 * starts from (state_S[b][h] [D][d], state_z[b][h] [D], float32, device memory, read only).
 *   causal = 1: the state is that of the tokens before this block (the recurrent view's
 *     S_t, z_t at the block's start), so out_i = phi(q_i)(S0 + sum_{j<=i} phi(k_j) v_j^T) /
 *     phi(q_i).(z0 + sum_{j<=i} phi(k_j)).  With state 0 this is linattn_forward.
 *   causal = 0: the state is what the rest of the sequence contributes, so
 *     out_i = phi(q_i)(S0 + sum_j phi(k_j) v_j^T) / phi(q_i).(z0 + sum_j phi(k_j)).
 * This splits one sequence over several calls or devices: each block's state comes from
 * linattn_forward_state of the other blocks, summed with linattn_sum_states.  Other
 * arguments, layouts and errors as in linattn_forward; state_S and state_z must be 16-byte
 * aligned.  (Pages: "Efficient Transformers: Linear Attention and Flash Attention", section
 * "The recurrent view: attention as an RNN" — the state carries everything earlier tokens
 * contribute.)
 */
linattn_status linattn_forward_init(const void *q, const void *k, const void *v, void *out,
                                    const float *state_S, const float *state_z, int64_t B,
                                    int64_t H, int64_t n, int64_t d, int causal,
                                    linattn_dtype dtype, linattn_stream_t stream);

/*
 * The two calls of a sequence-sharded block that read its k, v once: linattn_forward_state_keep
 * is linattn_forward_state that also leaves the block's aggregates in `aggregates` (caller-
 * owned device memory of linattn_block_aggregates_bytes(B, H, n, d, dtype) bytes, 16-byte
 * aligned); linattn_forward_init_from is linattn_forward_init that takes them from there
 * instead of recomputing them from k, v.  The pair must see the same B, H, n, d, dtype and
 * device, with nothing between them writing k, v or the buffer; linattn_forward_init_from
 * overwrites the buffer (causal: its exclusive prefixes).  linattn_block_aggregates_bytes
 * returns 0 for arguments linattn_forward_state would reject.  Other arguments, layouts and
 * errors as in linattn_forward_state and linattn_forward_init.  (Pages: "Efficient
 * Transformers: Linear Attention and Flash Attention", section "The recurrent view: attention
 * as an RNN": a block's state is the sum of its tokens' contributions, so the sums the state
 * needs are the ones the block's own pass starts from.)
 */
size_t linattn_block_aggregates_bytes(int64_t B, int64_t H, int64_t n, int64_t d,
                                      linattn_dtype dtype);
linattn_status linattn_forward_state_keep(const void *k, const void *v, float *state_S,
                                          float *state_z, float *aggregates, int64_t B,
                                          int64_t H, int64_t n, int64_t d, linattn_dtype dtype,
                                          linattn_stream_t stream);
linattn_status linattn_forward_init_from(const void *q, const void *k, const void *v,
                                         void *out, const float *state_S, const float *state_z,
                                         float *aggregates, int64_t B, int64_t H, int64_t n,
                                         int64_t d, int causal, linattn_dtype dtype,
                                         linattn_stream_t stream);

/*
 * Performer's FAVOR+ positive random features (named on the page "Efficient Transformers:
 * Linear Attention and Flash Attention", section "Linear attention: reordering the matmuls,
 * not shrinking them", as features whose dot products approximate the softmax kernel
 * exp(q . k); the page gives no formula, this is the positive-feature form):
 *     out[t][i] = exp(W[i] . x[t] - |x[t]|^2 / 2) / sqrt(m),   i < m features,
 * so that E_W[phi(q) . phi(k)] = exp(q . k) for W with i.i.d. N(0, 1) entries.
 *   x   : [rows][d] of type `dtype` (for attention: q or k, already scaled as wanted).
 *   W   : [m][d] float32, the random projection (row i = w_i), drawn by the caller.
 *   out : [rows][m] of type `dtype`, written.
 * d, m in {64, 128}; rows < 2^31.  bf16: the product X W^T runs on the tensor cores with W
 * split into two bf16 parts (about 2^-16 relative); fp32: CUDA cores.  Feed the features of q
 * and k to linattn_forward_features.
 */
linattn_status linattn_favor_features(const void *x, const float *W, void *out, int64_t rows,
                                      int64_t d, int64_t m, linattn_dtype dtype,
                                      linattn_stream_t stream);

/*
 * linattn_forward on features the caller has computed: phi_q and phi_k ([B][H][n][m], type
 * `dtype`) are used as phi(q) and phi(k) directly, with no feature map applied, and v, out are
 * [B][H][n][d]:
 *     out_i = phi_q_i S / phi_q_i . z,   S = sum_j phi_k_j v_j^T (m x d),   z = sum_j phi_k_j.
 * The features must be non-negative with positive denominators (FAVOR+ features are).
 * m, d in {64, 128}; m != d needs bf16 I/O (the fp32 CUDA-core kernels keep m = d, else
 * LINATTN_ERR_UNSUPPORTED).  Other arguments, layouts and errors as in linattn_forward.
 */
linattn_status linattn_forward_features(const void *phi_q, const void *phi_k, const void *v,
                                        void *out, int64_t B, int64_t H, int64_t n, int64_t m,
                                        int64_t d, int causal, linattn_dtype dtype,
                                        linattn_stream_t stream);

/*
 * Backward pass: the gradients of a loss L with respect to q, k and v, given
 * dout = dL/dout for out = linattn_forward(q, k, v, causal).  All seven tensors are
 * [B][H][n][d] of type `dtype` (dq, dk, dv written in that type).  bf16: the products run
 * on the tensor cores (bf16 operands, float32 accumulation), the rank-one terms on the CUDA
 * cores in float32; float32: everything on the CUDA cores in float32.  The pages define the
 * forward only ("Linear Attention > Memory Efficiency" notes that training keeps the forward's
 * tensors for backpropagation); this is its chain rule: with
 * w_ij = phi(q_i).phi(k_j), den_i = sum_j w_ij and a_i = dout_i / den_i,
 * b_i = -(dout_i . out_i) / den_i,
 *     dL/dphi(q_i) = sum_j (v_j . a_i + b_i) phi(k_j),
 *     dL/dphi(k_j) = sum_i (v_j . a_i + b_i) phi(q_i),
 *     dL/dv_j      = sum_i w_ij a_i,
 * then through phi'(x) = 1 (x > 0), exp(x) (x <= 0); sums over j <= i (causal) or all.
 * Asynchronous on `stream`; takes a stream-ordered workspace: per head, bf16: two records
 * (d^2 + 3d + 4 floats) per segment of up to 4096 tokens plus about n (2.1 d + 3.2) floats;
 * float32:
 * 2 (n/64) (d^2 + d) + n (d + 1) floats.  Errors as in linattn_forward; a bounded wait that
 * gave up is reported by linattn_device_error.
 */
linattn_status linattn_backward(const void *q, const void *k, const void *v, const void *dout,
                                void *dq, void *dk, void *dv, int64_t B, int64_t H, int64_t n,
                                int64_t d, int causal, linattn_dtype dtype,
                                linattn_stream_t stream);

/*
 * linattn_backward with a chosen segment length for bf16 (the tokens of one work item of
 * the two chunked walks: a multiple of 64; 0 picks the default; ignored for float32).  The
 * result does not depend on it beyond rounding order; tests use it to move the segment
 * boundaries.  Other arguments as in linattn_backward.
 */
linattn_status linattn_backward_ex(const void *q, const void *k, const void *v,
                                   const void *dout, void *dq, void *dk, void *dv, int64_t B,
                                   int64_t H, int64_t n, int64_t d, int causal,
                                   linattn_dtype dtype, int64_t segment_len,
                                   linattn_stream_t stream);

/*
 * Per-head sum of gathered states.  states: float32 device memory laid out
 * [count][B][H][D*d + D] (each state: S row-major [D][d], then z [D]; this is what an
 * all-gather of every rank's linattn_forward_state output, packed that way, produces).
 * Writes state_S[b][h] = sum over i in [0, count), i != skip, of the S part of
 * states[i][b][h] (added in order of i), and state_z likewise; zero when nothing is summed
 * (count = 0).  skip = -1 sums every state.  All pointers 16-byte aligned; states may be
 * null when count = 0.  d in {64, 128}.
 */
linattn_status linattn_sum_states(const float *states, int64_t count, int64_t skip, int64_t B,
                                  int64_t H, int64_t d, float *state_S, float *state_z,
                                  linattn_stream_t stream);

/*
 * linattn_forward with a chosen segment length: the number of tokens one work item of
 * the chunked causal pass covers (a multiple of 128 tokens; 0 picks the default).
 * The result does not depend on it beyond rounding order; tests use it to move the
 * segment boundaries.  Other arguments as in linattn_forward.
 */
linattn_status linattn_forward_ex(const void *q, const void *k, const void *v, void *out,
                                  int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                  linattn_dtype dtype, int64_t segment_len,
                                  linattn_stream_t stream);

/*
 * linattn_forward with q, k, v and out in HOST memory: the same result as copying q, k, v to
 * the device, calling linattn_forward and copying out back.  The heads run in groups (about
 * eight, each at most 1 GiB of the four tensors) on three internal streams, so the copies of
 * one group overlap the copies and kernels of the others.  Page-locked (pinned) buffers let
 * the copies run asynchronously and concurrently; pageable ones are accepted and copied by the
 * runtime's staging.  The groups start after the work already enqueued on `stream`, and
 * `stream` waits for all of them: once it is synchronised, `out` holds the result and the
 * inputs may be reused.  Device memory: the pool holds three groups' buffers (and their
 * workspaces) while the call runs.  Returns after enqueuing; LINATTN_ERR_INVALID_ARG for a
 * null pointer or a bad shape (as linattn_forward; no alignment is required of host
 * buffers), LINATTN_ERR_CUDA if a copy, an allocation or a launch fails.
 */
linattn_status linattn_forward_host(const void *q, const void *k, const void *v, void *out,
                                    int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                    linattn_dtype dtype, linattn_stream_t stream);

/* Bytes of one head's state, D*d*4 + D*4 (fp32 S and z), independent of n
 * (page "Linear Attention > Memory Efficiency": 16,640 bytes at d = D = 64). */
size_t linattn_state_bytes(int64_t d);

/* Static text for a status code. */
const char *linattn_status_string(linattn_status status);

/* Synchronises `stream`, then reports and clears the current device's kernel error flags:
 * LINATTN_ERR_TIMEOUT if a bounded wait gave up since the last call, else LINATTN_OK
 * (or LINATTN_ERR_CUDA if synchronising or reading a flag failed).  It covers every entry
 * point, linattn_forward_noalloc included, and allocates nothing itself. */
linattn_status linattn_device_error(linattn_stream_t stream);

/* Self-test of the failure path: launches one thread that waits, with the kernels' bounded
 * wait, on a barrier nothing ever completes.  It gives up after the wait limit (2 s) without
 * trapping; the next linattn_device_error() then returns LINATTN_ERR_TIMEOUT (and clears it),
 * and the context stays usable. */
linattn_status linattn_selftest_wait_timeout(linattn_stream_t stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int linattn_version(void);

/* Number of kernels (and device memsets) this library has enqueued in this process, on
 * every device.  Benchmarks read it before and after a timed region. */
uint64_t linattn_launch_count(void);

/*
 * Measurement aid: while `count` > 0, every kernel (and device memset) this library
 * enqueues on the calling thread is followed by cudaEventRecord(events[i], stream) with
 * i = 0, 1, ... (up to count - 1), so the caller can time each launch of a multi-kernel call with
 * cudaEventElapsedTime.  `events` holds cudaEvent_t handles created by the caller; the
 * library keeps the pointer until the next call with count = 0.
 */
linattn_status linattn_profile_events(void *const *events, int count);

/* Size of the fixed device scratch block behind linattn_forward_noalloc (32 MiB). */
#define LINATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * linattn_forward for callers that cannot allocate memory: hosts that reserve all device
 * memory up front, and runtimes that own the device allocator and forbid libraries from
 * calling it.  The pages have no counterpart; this is a deployment variant, not part of the
 * method.  Same arguments, checks, layouts, results and dtypes as linattn_forward, through
 * the same kernels; it calls no cudaMalloc, cudaFree or other allocating routine.  Its
 * temporary state lives in one fixed block of LINATTN_NOALLOC_SCRATCH_BYTES of device memory
 * that the library declares statically; every GPU that loads the library holds that block
 * until the process exits.
 *   - Work that needs more temporary state than the block holds is rejected with
 *     LINATTN_ERR_INVALID_ARG before anything is launched (the bf16 path first lengthens
 *     its segments to fit; it needs 66,048 B per head and segment at d = 128, 16,640 B at
 *     d = 64; the fp32 path needs that per 64-token chunk).
 *   - All calls on a device share the block and leave their contents in it; nothing in it
 *     needs to start at zero.  Calls that overlap on the GPU race on it: issue them on one
 *     stream or otherwise order them.
 *   - The first call on each device looks up the block's device address with that device
 *     current; make that first call before any stream capture.  A failed look-up returns
 *     LINATTN_ERR_CUDA and is retried by the next call.
 *   - A kernel wait that gives up is recorded in the block's status word; linattn_device_error()
 *     reports it (and clears it) like any other.
 */
linattn_status linattn_forward_noalloc(const void *q, const void *k, const void *v, void *out,
                                       int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                                       linattn_dtype dtype, linattn_stream_t stream);

/* Self-test of linattn_forward_noalloc's failure report: the same bounded wait as
 * linattn_selftest_wait_timeout, recording its give-up in the static block's status word.
 * The next linattn_device_error() returns LINATTN_ERR_TIMEOUT (and clears it).  Allocates
 * nothing. */
linattn_status linattn_selftest_noalloc_wait_timeout(linattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LINATTN_H */
