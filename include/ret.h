/*
 * ret.h - C ABI of the B200 (sm_100a) retention library, libret.so.
 *
 * Retention is the sequence mixer of RetNet. Sources for the operations:
 *   [RM] aiqz.cc, "RetNet retention mechanism" tutorial page: sections
 *        保留机制初识 (first look, R_n = sum_{m<=n} gamma^(n-m) (Q_n K_m^T) V_m),
 *        衰减矩阵 (decay matrix D_nm = gamma^(n-m) for n >= m, else 0),
 *        并行训练 (parallel form R = (Q K^T (.) D) V),
 *        递归推理 (recurrent form S_n = gamma S_{n-1} + K_n^T V_n, R_n = Q_n S_n),
 *        块级循环 (chunkwise recurrent form: parallel inside a chunk, state
 *        passed between chunks).
 *   [RN] 171host.com, "Retentive Network (RetNet) 详解": section 3.1 (the three
 *        equivalent forms) and 3.2 (multi-scale retention: one gamma per head,
 *        plus a gate and a normalisation).
 *   [GR] pwwt.cn, "unilm RetNet 技术指南 ... Gated RetNet 的源码解析": the gated
 *        form with a per-token, per-head log-decay g (parallel_gate_retention,
 *        chunk_gate_retention = cross_chunk + inner_chunk,
 *        recurrent_gate_retention), and the GateRetention module (subln, an
 *        RMSNorm over the head dimension; g_proj feeding a swish gate).
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers owned by the caller, except in the *_host
 *     calls, whose tensors are in host memory. The library never frees caller
 *     memory and keeps no pointer after the call returns.
 *   - Tensors are contiguous row-major, heads leading:
 *       q, k [B, H, N, dk]   v, o [B, H, N, dv]   state [B, H, dk, dv] (fp32)
 *       gamma [H] (fp32)     g [B, H, N] (fp32, natural-log decay, normally <= 0)
 *   - dt selects the element type of q, k, v and o (RET_F32 or RET_BF16).
 *     gamma, g and state are always fp32. Arithmetic accumulates in fp32.
 *   - No 1/sqrt(dk) scale is applied: callers pass pre-scaled q or k.
 *   - Calls are asynchronous on `stream` (a cudaStream_t cast to void*;
 *     NULL = the legacy default stream). Arguments are validated on the host
 *     before anything is launched: a validation status (RET_ERR_NULL, _SHAPE,
 *     _DTYPE, _UNSUPPORTED, _ALIGN, _SCRATCH) means nothing ran. RET_ERR_CUDA
 *     from a call that launches several kernels may follow some of them; the
 *     outputs are then undefined.
 *   - Errors are returned, never raised: no exit(), no device trap.
 *   - Calls keep no per-call state (the library holds only per-device helpers
 *     it creates once: the no-allocation scratch buffer, five streams with their
 *     events for the backward and two for the *_host calls) and are safe from
 *     several host threads,
 *     except ret_chunkwise_noalloc, whose calls all share one scratch buffer:
 *     calls of it that overlap on the GPU race (see its declaration).
 *   - N == 0 is a valid empty problem: nothing is launched, state_out (if
 *     given) receives state_in (or zeros).
 */
#ifndef RET_H_
#define RET_H_

#if defined(__GNUC__)
#define RET_API __attribute__((visibility("default")))
#else
#define RET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RET_OK = 0,
    RET_ERR_NULL = 1,        /* a required pointer is NULL */
    RET_ERR_SHAPE = 2,       /* a size is negative or zero where it must be positive */
    RET_ERR_DTYPE = 3,       /* dt is not a ret_dtype value */
    RET_ERR_UNSUPPORTED = 4, /* sizes outside what the kernels support (see each call) */
    RET_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
    RET_ERR_TIMEOUT = 6,     /* a kernel's bounded wait ran out (device error word set) */
    RET_ERR_ALIGN = 7,       /* a pointer is not 16-byte aligned */
    RET_ERR_SCRATCH = 8      /* ret_chunkwise_noalloc: the problem needs more scratch than its fixed buffer */
} ret_status;

typedef enum { RET_F32 = 0, RET_BF16 = 1 } ret_dtype;

/*
 * Parallel form, [RM] 并行训练 / [RN] 3.1: O = (Q K^T (.) D) V with
 * D_nm = gamma_h^(n-m) for n >= m and 0 above the diagonal ([RM] 衰减矩阵).
 * O(N^2) work; meant for short sequences and as a cross-check of the other
 * forms. Requires dk <= 1024, dv >= 1.
 */
RET_API ret_status ret_parallel(const void* q, const void* k, const void* v, const float* gamma,
                        void* o, int B, int H, int N, int dk, int dv,
                        ret_dtype dt, void* stream);

/*
 * Chunkwise recurrent form, [RM] 块级循环 / [RN] 3.1 and 4.3. The sequence is
 * split into chunks of `chunk` tokens (the last may be shorter and behaves as
 * zero padding). For chunk i of length L, local rows j, m = 0..L-1:
 *   O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + diag(gamma^(j+1)) Q_[i] S_[i-1]
 *   S_[i] = gamma^L S_[i-1] + sum_m gamma^(L-1-m) K_m^T V_m
 * state_in : initial state [B, H, dk, dv] fp32, or NULL for zeros.
 * state_out: final state [B, H, dk, dv] fp32, or NULL. May equal state_in.
 * The result does not depend on `chunk` beyond rounding: the tensor-core path
 * computes on tiles of 64 or (gamma_h >= 2^-0.75, dk >= 128) 128 tokens.
 * Requires chunk >= 1, dk <= 256, dv >= 1. The tensor-core path (bf16,
 * dk in {64, 128, 256}, dv a multiple of 128, chunk a multiple of 64) also
 * needs 16-byte aligned q, k, v, o; other shapes use a CUDA-core path.
 * May allocate stream-ordered scratch (cudaMallocAsync) for long sequences
 * with few heads; it is freed on the same stream before the call returns.
 */
RET_API ret_status ret_chunkwise(const void* q, const void* k, const void* v, const float* gamma,
                         void* o, const float* state_in, float* state_out,
                         int B, int H, int N, int dk, int dv, int chunk,
                         ret_dtype dt, void* stream);

/*
 * One recurrent (decode) step, [RM] 递归推理:
 *   S <- gamma_h S + k^T v   (in place),   o = q S   (the updated state).
 * q, k [B, H, dk]; v, o [B, H, dv] of type dt; state [B, H, dk, dv] fp32.
 * The state is read and written once: the step is bound by HBM bandwidth.
 * Requires dk <= 4096; state must be 16-byte aligned and dv a multiple of 4
 * for the vectorised path (otherwise a scalar path runs).
 */
RET_API ret_status ret_recurrent_step(const void* q, const void* k, const void* v, const float* gamma,
                              float* state, void* o, int B, int H, int dk, int dv,
                              ret_dtype dt, void* stream);

/*
 * One gated recurrent (decode) step, [GR] recurrent_gate_retention:
 *   S <- exp(g_bh) S + k^T v   (in place),   o = q S   (the updated state).
 * g [B, H] fp32: this step's natural-log decay per (batch, head), normally <= 0
 * (the decode counterpart of gated_ret_chunkwise's g[:, :, n]). Other tensors,
 * layouts and requirements as ret_recurrent_step.
 */
RET_API ret_status gated_ret_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                                    float* state, void* o, int B, int H, int dk, int dv,
                                    ret_dtype dt, void* stream);

/*
 * Gated chunkwise form, [GR] chunk_gate_retention: the per-token log-decay g
 * replaces log(gamma). With Gl the inclusive cumulative sum of g restarted at
 * each chunk:
 *   inner: (Q K^T) * exp(Gl_j - Gl_m) for j >= m, times V
 *   cross: exp(Gl_j) (Q_[i] S_[i-1])_j
 *   state: S_[i] = exp(Gl_{L-1}) S_[i-1] + sum_m exp(Gl_{L-1} - Gl_m) K_m^T V_m
 * Only in-chunk differences of the cumulative sum are exponentiated, so long
 * sequences cannot underflow. Same shapes, state handling, limits and paths as
 * ret_chunkwise.
 */
RET_API ret_status gated_ret_chunkwise(const void* q, const void* k, const void* v, const float* g,
                               void* o, const float* state_in, float* state_out,
                               int B, int H, int N, int dk, int dv, int chunk,
                               ret_dtype dt, void* stream);

/*
 * ret_chunkwise / gated_ret_chunkwise from HOST memory: q, k, v, gamma (or g) and
 * o are host pointers with the layouts above; no initial or final state. The
 * call copies the inputs to stream-ordered device buffers, computes and copies o
 * back, pipelined over groups of heads (at most 8: whole batches when B >= 8,
 * else runs of heads inside one batch): the copies in of later groups overlap
 * the forward and the copy out of earlier ones, on `stream` and two library
 * streams of the *_host calls, forked from it and joined back. It returns once everything is
 * enqueued: o is complete when `stream` is. Host buffers should be page-locked
 * (cudaHostAlloc, cudaHostRegister); pageable buffers still give the right
 * result, but the driver then stages each copy and nothing overlaps. Each
 * group's result is that of ret_chunkwise on the group alone: heads are
 * independent, but the group's plan (the sequence segments that fill the SMs)
 * can differ from the whole batch's, and with it the rounding. Limits and paths as
 * ret_chunkwise; the device buffers are freed on `stream` before the call
 * returns. Not in the pages: the host side of serving a layer whose activations
 * live in host memory.
 */
RET_API ret_status ret_chunkwise_host(const void* q, const void* k, const void* v, const float* gamma,
                              void* o, int B, int H, int N, int dk, int dv, int chunk,
                              ret_dtype dt, void* stream);
RET_API ret_status gated_ret_chunkwise_host(const void* q, const void* k, const void* v, const float* g,
                                    void* o, int B, int H, int N, int dk, int dv, int chunk,
                                    ret_dtype dt, void* stream);

/* Static description of a status code. Never NULL. */
RET_API const char* ret_status_str(ret_status s);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word, which a kernel sets when one of its bounded waits runs out.
 * Returns RET_ERR_TIMEOUT if it was set, RET_ERR_CUDA if the stream reports
 * an error, RET_OK otherwise.
 */
RET_API ret_status ret_last_device_error(void* stream);

/*
 * Backward pass of ret_chunkwise / gated_ret_chunkwise from a zero initial
 * state: gradients of L = sum_n dout_n . o_n, differentiating [RM] 保留机制初识's
 * sum (o_n = sum_{m<=n} w_nm (q_n . k_m) v_m, w_nm = gamma^(n-m), or
 * exp(G_n - G_m) with G the cumulative sum of g, [GR] parallel_gate_retention):
 *   dq_n = sum_{m<=n} w_nm (dout_n . v_m) k_m,  dk_m = sum_{n>=m} w_nm (dout_n . v_m) q_n,
 *   dv_m = sum_{n>=m} w_nm (q_n . k_m) dout_n,
 *   dgamma_h (optional, [H] fp32) = d L / d gamma_h  (not defined for gamma_h = 0),
 *   dg (optional, [B, H, N] fp32) = d L / d g.
 * dout has v's layout; dq, dk, dv have q's, k's, v's (dtype dt). Computed with the
 * forward kernels (dq directly, dk and dv on the time-reversed sequence, a dv wider
 * than 256 contracted in pieces) and small kernels of this library; takes
 * stream-ordered scratch (freed on the same stream). On the tensor-core path the
 * pieces are read in place, and the steps that do not depend on each other run
 * side by side on five library-owned streams of the current device (four of the
 * device's greatest priority for the dq and dk pieces, one of its least for dv),
 * forked from and joined back to `stream` with events: all work stays ordered on
 * `stream` (and can be captured in a graph). Concurrent calls from several host
 * threads serialise while they enqueue.
 * bf16 needs 16-byte aligned tensors. Requires dk <= 256.
 */
RET_API ret_status ret_chunkwise_backward(const void* q, const void* k, const void* v, const float* gamma,
                                  const void* dout, void* dq, void* dk, void* dv, float* dgamma,
                                  int B, int H, int N, int dk_dim, int dv_dim, int chunk,
                                  ret_dtype dt, void* stream);
RET_API ret_status gated_ret_chunkwise_backward(const void* q, const void* k, const void* v, const float* g,
                                        const void* dout, void* dq, void* dk, void* dv, float* dg,
                                        int B, int H, int N, int dk_dim, int dv_dim, int chunk,
                                        ret_dtype dt, void* stream);

/*
 * ret_chunkwise_backward / gated_ret_chunkwise_backward from HOST memory: every
 * tensor (q, k, v, gamma or g, dout, dq, dk, dv, dgamma or dg) is a host pointer
 * with the layouts above; dgamma / dg may be NULL. The heads are cut into the
 * groups of ret_chunkwise_host and pipelined the same way: the copies in of later
 * groups overlap the backward and the copies out of earlier ones. Each group runs
 * the device-buffer backward on its heads; dgamma, which sums over batches, is
 * gathered per group on the device and added there once every group is done.
 * Returns once everything is enqueued: the outputs are complete when `stream` is.
 * Host buffers should be page-locked for the copies to overlap. Device buffers
 * come from the stream-ordered pool and are freed on `stream` before the call
 * returns. Limits as ret_chunkwise_backward. Not in the pages.
 */
RET_API ret_status ret_chunkwise_backward_host(const void* q, const void* k, const void* v, const float* gamma,
                                       const void* dout, void* dq, void* dk, void* dv, float* dgamma,
                                       int B, int H, int N, int dk_dim, int dv_dim, int chunk,
                                       ret_dtype dt, void* stream);
RET_API ret_status gated_ret_chunkwise_backward_host(const void* q, const void* k, const void* v, const float* g,
                                             const void* dout, void* dq, void* dk, void* dv, float* dg,
                                             int B, int H, int N, int dk_dim, int dv_dim, int chunk,
                                             ret_dtype dt, void* stream);

/*
 * Sequence split into consecutive segments computed separately (for example
 * one per GPU, then one exchange of states), [RM] 块级循环 / [GR] cross_chunk:
 * the chunkwise recurrence composes over segments as
 *   S_in(0) = state_in,   S_in(r + 1) = D_r S_in(r) + U_r,
 * where U_r is segment r's end state from a zero start and D_r its total decay
 * (gamma_h^{N_r}, or exp of the sum of its gates). Running ret_chunkwise (or
 * gated_ret_chunkwise) on segment r from S_in(r) then gives exactly that
 * segment's outputs of the whole sequence, and S_in(R) is the final state.
 *
 * ret_chunkwise_state / gated_ret_chunkwise_state: U and log2 D of one segment
 * (k, v, gamma or g as in the chunkwise calls; no q, no outputs).
 *   state_out  [B, H, dk, dv] fp32: U (from a zero start).
 *   log2_decay [B, H] fp32: log2 D per (b, h) (-inf where gamma_h = 0).
 * Same size rules and tensor-core path conditions as ret_chunkwise; may take
 * stream-ordered scratch (freed on the same stream before returning).
 */
RET_API ret_status ret_chunkwise_state(const void* k, const void* v, const float* gamma, float* state_out,
                               float* log2_decay, int B, int H, int N, int dk, int dv, int chunk,
                               ret_dtype dt, void* stream);
RET_API ret_status gated_ret_chunkwise_state(const void* k, const void* v, const float* g, float* state_out,
                                     float* log2_decay, int B, int H, int N, int dk, int dv, int chunk,
                                     ret_dtype dt, void* stream);

/* Kernels one ret_chunkwise_state / gated_ret_chunkwise_state call launches (0 for
 * an empty segment, -1 if the arguments would be rejected). Host function. */
RET_API int ret_chunkwise_state_launches(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt);

/*
 * Multi-scale retention output epilogue ("Retentive Network (RetNet) 详解",
 * section 3.2: a gate and a normalisation on retention's output; the Gated
 * RetNet page's GateRetention module: subln, an RMSNorm over each head's
 * dimension without affine weights, and a swish gate fed by g_proj):
 *   y[b, n, h, :] = swish(gate[b, n, h, :]) * o[b, h, n, :] / sqrt(mean_c o[b, h, n, c]^2 + eps),
 *   swish(x) = x / (1 + exp(-x)).
 * o: the retention output [B, H, N, dv] (as ret_chunkwise writes it); gate and y:
 * token-major [B, N, H, dv], the layout of the module's projections. All three
 * have dtype dt; sums and the scale are fp32. eps >= 0 (the pages' norm default
 * is 1e-5). One pass: each element of o and gate is read once and y written once.
 * y may be the gate buffer itself (in place); any other overlap of y with o or
 * gate is rejected with RET_ERR_UNSUPPORTED. Errors: RET_ERR_SHAPE for invalid
 * sizes or eps, RET_ERR_NULL for a missing pointer (N > 0), RET_ERR_DTYPE.
 * Any dv and alignment; whole 16-byte rows with 16-byte aligned pointers take
 * the vector kernel.
 */
RET_API ret_status ret_msr_norm_gate(const void* o, const void* gate, void* y, int B, int H, int N, int dv, float eps,
                                     ret_dtype dt, void* stream);

/* Kernels one ret_chunkwise_backward (gated = 0) or gated_ret_chunkwise_backward
 * (gated = 1) call launches with these arguments, ddecay non-zero when the decay
 * gradient is requested (0 for an empty sequence, -1 if the arguments would be
 * rejected). The cudaMemsetAsync that zeroes dgamma is not counted. */
RET_API int ret_chunkwise_backward_launches(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt, int gated,
                                            int ddecay);

/*
 * Start states of R consecutive segments from their end states and decays:
 *   seg_states [R, B, H, dk, dv] fp32 (U_0 .. U_{R-1}), seg_log2_decay [R, B, H],
 *   state_in [B, H, dk, dv] or NULL (zeros),
 *   start_states [R, B, H, dk, dv] receives S_in(0 .. R-1),
 *   end_state [B, H, dk, dv] or NULL receives S_in(R) (the state after all R).
 * start_states and end_state must not overlap the inputs. Errors: RET_ERR_SHAPE
 * for non-positive sizes, RET_ERR_NULL for a missing required pointer.
 */
RET_API ret_status ret_state_prefix(const float* seg_states, const float* seg_log2_decay,
                            const float* state_in, float* start_states, float* end_state,
                            int R, int B, int H, int dk, int dv, void* stream);

/*
 * Self-test of the failure path (the pages have no counterpart; a diagnostic).
 * Launches one CTA on `stream` that takes tensor memory as the tensor-core
 * kernels do, waits on an mbarrier that nothing completes with the kernels'
 * bounded wait limited to limit_us microseconds (1 .. 1,000,000), sets the
 * device error word when the wait runs out, releases the tensor memory and
 * returns. Nothing faults or hangs; afterwards ret_last_device_error reports
 * RET_ERR_TIMEOUT once and the device stays usable. Returns RET_ERR_SHAPE for
 * a limit out of range, RET_ERR_UNSUPPORTED without an sm_100 device,
 * RET_ERR_CUDA if the launch fails, RET_OK otherwise.
 */
RET_API ret_status ret_selftest_wait_timeout(unsigned int limit_us, void* stream);

/*
 * Which kernel family ret_chunkwise / gated_ret_chunkwise would run for these
 * arguments: 1 = tcgen05 tensor-core path, 0 = CUDA-core path, -1 = rejected.
 * Pure host function; nothing is launched.
 */
RET_API int ret_chunkwise_path(int dk, int dv, int chunk, ret_dtype dt);

/*
 * Number of kernels one ret_chunkwise / gated_ret_chunkwise call with these
 * arguments launches (0 for an empty sequence, -1 if the arguments would be
 * rejected). Pure host function; nothing is launched.
 */
RET_API int ret_chunkwise_launches(int B, int H, int N, int dk, int dv, int chunk, ret_dtype dt);

/*
 * ret_chunkwise without any device allocation. The pages have no counterpart for
 * this entry point: it is an interface for callers, not part of the method.
 *
 * ret_chunkwise may take stream-ordered scratch from the device's default
 * memory pool when it splits a long sequence of few heads into segments. Some
 * callers cannot let a library allocate: a framework whose own allocator has
 * reserved the device memory up front, a serving loop that forbids allocations
 * after start-up, or code that must not touch the default pool. This entry
 * point computes exactly what ret_chunkwise computes, with the same arguments
 * and the same kernels, but takes its scratch from a fixed buffer compiled into
 * the library: a file-scope device array of RET_NOALLOC_SCRATCH_BYTES (16 MiB)
 * that every GPU which loads the library holds until the process exits.
 *
 *  - The first call on a device, with that device current, looks up the
 *    buffer's device address (cudaGetSymbolAddress) and caches it. Make that
 *    first call before any stream capture. The cached address belongs to the
 *    device's current context: after cudaDeviceReset (or any reset of the
 *    primary context) in the same process it is stale, so do not call this
 *    entry point again in that process after such a reset.
 *  - A problem whose scratch would exceed the buffer is rejected on the host
 *    with RET_ERR_SCRATCH before anything is launched. Passing state_in and
 *    state_out as the same buffer needs an extra copy of the state in scratch.
 *    Where ret_chunkwise would cut its state-only pass finer than its segments
 *    and that does not fit, this entry point keeps one piece per segment (the
 *    same result up to rounding order).
 *  - All calls share the one buffer, which keeps the previous call's contents;
 *    every scratch byte a call reads is written earlier in that same call, so
 *    nothing has to be cleared. Calls that overlap on the GPU (for example on
 *    two streams) race on the buffer: serialise them.
 *  - Neither cudaMalloc, cudaMallocAsync, cudaFree nor any other allocating
 *    routine is called.
 */
#define RET_NOALLOC_SCRATCH_BYTES (16u << 20)
RET_API ret_status ret_chunkwise_noalloc(const void* q, const void* k, const void* v, const float* gamma,
                                 void* o, const float* state_in, float* state_out,
                                 int B, int H, int N, int dk, int dv, int chunk,
                                 ret_dtype dt, void* stream);

/*
 * Scratch bytes of the fixed buffer that ret_chunkwise_noalloc would use for these
 * sizes (in_place != 0: state_in and state_out are one buffer), 0 when the call needs
 * none, -1 for sizes the call rejects as invalid. A value above
 * RET_NOALLOC_SCRATCH_BYTES means the call returns RET_ERR_SCRATCH. The figure depends
 * on the current device's SM count (the plan splits long sequences of few heads into
 * segments to fill the SMs). Host-only: launches nothing. No counterpart on the pages.
 */
RET_API long long ret_chunkwise_noalloc_scratch_bytes(int B, int H, int N, int dk, int dv, int chunk,
                                              ret_dtype dt, int in_place);

/* Library version, "major.minor.patch". */
RET_API const char* ret_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RET_H_ */
