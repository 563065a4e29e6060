/*
 * gdn.h -- C ABI of libgdn.so, the B200 (sm_100a) Gated DeltaNet (GDN) token mixer.
 *
 * The mixer (defined in the "Qwen3.8-Flash-Next" technical report, Fig. 2, and the
 * "Qwen3-Next 80B-A3B" field guide, §02 "Gated DeltaNet state update"):
 *   1. width-4 depthwise causal conv over the q, k and v streams, then SiLU;
 *   2. L2 normalisation of q and k per head;
 *   3. decay gate g = -exp(A_log) * softplus(a + dt_bias) (the decay-gate note of the
 *      "Qwen3.8-Flash-Next" model notes) and write gate beta = sigmoid(b);
 *   4. the gated delta rule on one d_v x d_k fp32 state per value head (field guide,
 *      §02, steps 1-6):  S' = e^g S;  e = v - S'k;  S'' = S' + beta e k^T;  y = S'' q;
 *   5. RMS normalisation of y per value head, times norm_w, gated by SiLU(z).
 * Value head h reads QK head h / (h_v / h_qk) (16 QK heads shared by 32 value heads in
 * the pages' model).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or synchronises on the hot path.  Work is enqueued on `stream`
 *     and runs asynchronously.
 *   - Tensors are contiguous, row-major, in the layouts given below, with 16-byte aligned
 *     base pointers.
 *   - Return value: GDN_OK (0) or a negative GDN_ERR_* code.  Arguments are validated on
 *     the host before any launch; on an error nothing is launched and no output is
 *     touched.
 *   - State layout: S[n][h][i][j], i in [0, d_v) the value component, j in [0, d_k) the
 *     key component (column-vector convention: S maps a key to a value).
 *   - Conv weights conv_w[C_conv][4], C_conv = 2*h_qk*d_k + h_v*d_v, channel order
 *     q (h_qk*d_k) | k (h_qk*d_k) | v (h_v*d_v); tap 3 multiplies the current token,
 *     tap 0 the token three back.  No conv bias.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gdn_stream_t; /* identical to cudaStream_t */

/* return codes */
#define GDN_OK 0
#define GDN_ERR_NULL (-1)           /* a required pointer is NULL */
#define GDN_ERR_SHAPE (-2)          /* unsupported or inconsistent dimensions */
#define GDN_ERR_DTYPE (-3)          /* unsupported dtype code */
#define GDN_ERR_ALIGN (-4)          /* a base pointer is not 16-byte aligned */
#define GDN_ERR_WORKSPACE (-5)      /* workspace missing or smaller than required */
#define GDN_ERR_CUDA (-6)           /* a CUDA launch or runtime call failed */
#define GDN_ERR_DEVICE_TIMEOUT (-7) /* a bounded device-side wait ran out (device status) */
#define GDN_ERR_INDEX (-8)          /* a device-side index was out of range (device status) */

/* dtype codes */
#define GDN_DTYPE_F32 0
#define GDN_DTYPE_BF16 1

typedef struct gdn_dims {
  int32_t n_seqs;       /* N >= 1 sequences */
  int32_t total_tokens; /* T_tot >= 0 packed tokens (decode: must equal n_seqs) */
  int32_t h_qk, h_v;    /* QK heads, value heads; h_v % h_qk == 0 */
  int32_t d_k, d_v;     /* head widths; only 128 x 128 is supported */
  int32_t in_dtype;     /* GDN_DTYPE_BF16 | GDN_DTYPE_F32: q, k, v, z (and decode conv_state) */
  int32_t out_dtype;    /* GDN_DTYPE_BF16 | GDN_DTYPE_F32: y */
  float q_scale;        /* multiplies the normalised query; 1.0 gives the pages' y = S'' q */
  float l2_eps;         /* q, k L2 norm: x / sqrt(sum x^2 + l2_eps); 1e-6 */
  float rms_eps;        /* output norm: y / sqrt(mean y^2 + rms_eps); 1e-6 */
} gdn_dims_t;

/*
 * Bytes of device workspace gdn_prefill needs for these dimensions (0 if the dims are
 * invalid).  Depends only on the dims, never on cu_seqlens' contents.
 */
size_t gdn_prefill_workspace_size(const gdn_dims_t* d);

/*
 * Prefill over packed variable-length sequences (the whole mixer, steps 1-5 above).
 *
 *   q, k        [T_tot][h_qk][d_k]   in_dtype
 *   v, z        [T_tot][h_v][d_v]    in_dtype
 *   a, b        [T_tot][h_v]         fp32 (gate pre-activations)
 *   A_log, dt_bias [h_v]             fp32
 *   conv_w      [C_conv][4]          fp32
 *   norm_w      [d_v]                fp32 (shared by all value heads)
 *   init_state  [N][h_v][d_v][d_k]   fp32, or NULL for zero initial states
 *   cu_seqlens  [N+1]                int32 DEVICE array of sequence offsets
 *                                    (cu[0] = 0, non-decreasing, cu[N] = T_tot), or NULL
 *                                    when N == 1 (one sequence of T_tot tokens)
 *   y           [T_tot][h_v][d_v]    out_dtype (written)
 *   final_state [N][h_v][d_v][d_k]   fp32 (written); may alias init_state
 *   workspace   device scratch of at least gdn_prefill_workspace_size(d) bytes
 *
 * Each sequence starts with a zero conv history and with its init_state.  Empty
 * sequences copy init_state (or zeros) to final_state.  T_tot == 0 writes final_state
 * only.  cu_seqlens' contents are not validated on the host (they stay on the device).
 * bf16 inputs run on the tensor-core path, which needs T_tot / 64 + N + 1 <= 65535
 * (about 4.19M packed tokens per call); larger calls return GDN_ERR_SHAPE.
 */
int gdn_prefill(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
                const float* a, const float* b, const float* A_log, const float* dt_bias,
                const float* conv_w, const float* norm_w, const float* init_state,
                const int32_t* cu_seqlens, void* y, float* final_state, void* workspace,
                size_t workspace_bytes, gdn_stream_t stream);

/*
 * One decode step: one new token for each of N sequences, on resident state
 * (field guide, §02: the state size stays fixed as the sequence grows).
 *
 *   q, k        [N][h_qk][d_k]       in_dtype
 *   v, z        [N][h_v][d_v]        in_dtype
 *   a, b        [N][h_v]             fp32
 *   A_log, dt_bias, conv_w, norm_w   as in gdn_prefill
 *   conv_state  [N][3][C_conv]       in_dtype, in/out: raw (pre-conv) x_{t-3}, x_{t-2},
 *                                    x_{t-1}; replaced by x_{t-2}, x_{t-1}, x_t (bit-exact)
 *   state       [N][h_v][d_v][d_k]   fp32, in/out, updated in place to S''
 *   y           [N][h_v][d_v]        out_dtype (written)
 * d->total_tokens must equal d->n_seqs.
 */
int gdn_decode(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
               const float* a, const float* b, const float* A_log, const float* dt_bias,
               const float* conv_w, const float* norm_w, void* conv_state, float* state,
               void* y, gdn_stream_t stream);

/*
 * Prefill -> decode hand-off, part 1: the decode conv history each sequence has after a
 * prefill over the same packed inputs.  The width-4 causal conv of step 1 ("Qwen3.8-Flash-Next"
 * technical report, Fig. 2) needs the three raw rows before each new token; the decode step
 * keeps them beside the fixed-size state (field guide, §02).  Writes, per sequence n, the raw (pre-conv) q | k | v
 * channels of its last three tokens: conv_state[n][r] = x_{te-3+r}, te = cu_seqlens[n+1], in
 * gdn_decode's conv_state layout.  Rows before the sequence's first token are zeros (every
 * prefill sequence starts with a zero conv history), so a sequence of fewer than three tokens
 * gets leading zero rows.  The copy is bit-exact.
 *
 *   q, k        [T_tot][h_qk][d_k]   in_dtype
 *   v           [T_tot][h_v][d_v]    in_dtype
 *   cu_seqlens  [N+1] int32 device array, or NULL when N == 1
 *   conv_state  [N][3][C_conv]       in_dtype (written)
 * Only the dims' shape fields and in_dtype are used.  A cu_seqlens entry outside
 * [0, T_tot] or below its predecessor makes that sequence's rows zeros and sets the device
 * status to GDN_ERR_INDEX.
 */
int gdn_prefill_conv_state(const gdn_dims_t* d, const void* q, const void* k, const void* v,
                           const int32_t* cu_seqlens, void* conv_state, gdn_stream_t stream);

/*
 * Prefill -> decode hand-off, part 2: gdn_decode on resident pools, the way a serving loop
 * keeps one state and one conv history per live request (field guide, §02: the state stays
 * the same size however long the sequence grows, so it can live in a fixed slot).  Same arguments and results as
 * gdn_decode, except that sequence n reads and updates pool slot slot_ids[n]:
 *
 *   conv_state_pool [n_slots][3][C_conv]       in_dtype, in/out
 *   state_pool      [n_slots][h_v][d_v][d_k]   fp32, in/out
 *   slot_ids        [N] int32 device array
 *
 * A negative slot id marks a padding entry: nothing is read or written for it (its y rows
 * are left as they were).  A slot id >= n_slots is skipped the same way and sets the device
 * status to GDN_ERR_INDEX.  Two entries naming the same slot race on it: the caller keeps the
 * ids of one call distinct.  Returns GDN_ERR_NULL (slot_ids NULL), GDN_ERR_SHAPE
 * (n_slots < 1) or what gdn_decode returns.
 */
int gdn_decode_slots(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
                     const float* a, const float* b, const float* A_log, const float* dt_bias,
                     const float* conv_w, const float* norm_w, void* conv_state_pool, float* state_pool,
                     int32_t n_slots, const int32_t* slot_ids, void* y, gdn_stream_t stream);

/*
 * Several decode tokens per sequence in one call (1 <= n_tokens <= 8), e.g. to verify drafted
 * tokens: the same per-token rule as gdn_decode (field guide, §02, steps 1-6, then the gated
 * RMSNorm) applied to n_tokens consecutive tokens of each sequence, reading and writing each
 * state row once per call instead of once per token.
 *
 *   q, k        [N][n_tokens][h_qk][d_k]   in_dtype
 *   v, z        [N][n_tokens][h_v][d_v]    in_dtype
 *   a, b        [N][n_tokens][h_v]         fp32
 *   conv_state  [N][3][C_conv]             in/out: replaced by the last three raw rows
 *   state       [N][h_v][d_v][d_k]         fp32, in/out: the state after the last token
 *   y           [N][n_tokens][h_v][d_v]    out_dtype (written)
 * d->total_tokens must equal d->n_seqs * n_tokens.  Returns GDN_ERR_SHAPE for n_tokens
 * outside 1..8, otherwise what gdn_decode returns.  n_tokens = 1 is exactly a gdn_decode
 * call (same kernel, identical results).
 */
int gdn_decode_multi(const gdn_dims_t* d, int32_t n_tokens, const void* q, const void* k, const void* v,
                     const void* z, const float* a, const float* b, const float* A_log, const float* dt_bias,
                     const float* conv_w, const float* norm_w, void* conv_state, float* state, void* y,
                     gdn_stream_t stream);

/*
 * Input projection of the mixer ("Qwen3.8-Flash-Next" technical report, Fig. 2: the query, key
 * and value streams are projections of the block input, as are the gate inputs a, b and the
 * output gate z).  One GEMM on the tensor cores, for every token t:
 *   [q | k | v | z | a | b][t] = W_in x[t]       (fp32 accumulation over `hidden`)
 *   x      [T][hidden]                  bf16, T = d->total_tokens
 *   w_in   [N_in][hidden]               bf16, row-major (the nn.Linear layout), rows in the order
 *                                       q | k | v | z | a | b: N_in = 2 h_qk d_k + 2 h_v d_v + 2 h_v
 * Outputs, written in the layouts gdn_prefill and gdn_decode take:
 *   q, k   [T][h_qk][d_k]               bf16 (round to nearest even)
 *   v, z   [T][h_v][d_v]                bf16
 *   a, b   [T][h_v]                     fp32
 * d->in_dtype must be GDN_DTYPE_BF16 and hidden a positive multiple of 64.  The pages print no
 * weights; tests and benchmarks use synthetic ones.  Asynchronous on `stream`; allocates nothing.
 * Returns GDN_OK, GDN_ERR_NULL, GDN_ERR_SHAPE, GDN_ERR_DTYPE, GDN_ERR_ALIGN or GDN_ERR_CUDA.
 */
int gdn_in_proj(const gdn_dims_t* d, int32_t hidden, const void* x, const void* w_in, void* q, void* k,
                void* v, void* z, float* a, float* b, gdn_stream_t stream);

/*
 * Output projection (field guide §02: the gated, RMS-normalised mixer output goes through the
 * output projection): out[t] = W_out y[t].
 *   y      [T][h_v d_v]                 bf16 (gdn_prefill's or gdn_decode's y)
 *   w_out  [hidden][h_v d_v]            bf16, row-major
 *   out    [T][hidden]                  bf16 (fp32 accumulation, round to nearest even)
 * d->out_dtype must be GDN_DTYPE_BF16 and hidden a positive multiple of 32.  Same conventions
 * and return codes as gdn_in_proj.
 */
int gdn_out_proj(const gdn_dims_t* d, int32_t hidden, const void* y, const void* w_out, void* out,
                 gdn_stream_t stream);

/*
 * Backward pass of the recurrence core (training).  The forward is the field guide's §02 rule
 * (steps 1-6) on already convolved and normalised streams, per (sequence, value head h) with QK
 * head j = h / (h_v / h_qk) and alpha_t = e^{g_t}:
 *   S'_t = alpha_t S_{t-1};  e_t = v_t - S'_t k_t;  S_t = S'_t + beta_t e_t k_t^T;  y_t = S_t q_t
 * (the query enters as given: d->q_scale is not applied).  Given dL/dy_t and dL/dS_T, this
 * call returns dL/dq, dL/dk (summed over the value heads sharing a QK head), dL/dv, dL/dg,
 * dL/dbeta and dL/dS_0, all fp32:
 *   qh, kh, dq, dk        [T][h_qk][d_k]
 *   v, dy, dv             [T][h_v][d_v]        (dy: the gradient of y before the output norm)
 *   g, beta, dg, dbeta    [T][h_v]             (g: the log-decay, so that alpha = e^g)
 *   init_state, dS_final, dS_init   [N][h_v][d_v][d_k]   (init_state, dS_final may be NULL: 0)
 *   cu_seqlens            [N + 1] device int32, or NULL for one sequence
 * d->in_dtype and d->out_dtype are not read (fp32 throughout).  The workspace holds a state
 * checkpoint per chunk and value head (64 KiB each) and, per token and value head, the partial
 * sums of dq, dk, dbeta and dg of each of the 4 row slices (4 x 1032 bytes):
 * gdn_recurrence_backward_workspace_size(d) bytes.  Asynchronous on
 * `stream`.  Returns GDN_OK, GDN_ERR_NULL, GDN_ERR_SHAPE, GDN_ERR_ALIGN, GDN_ERR_WORKSPACE or
 * GDN_ERR_CUDA.
 */
size_t gdn_recurrence_backward_workspace_size(const gdn_dims_t* d);
int gdn_recurrence_backward(const gdn_dims_t* d, const float* qh, const float* kh, const float* v,
                            const float* g, const float* beta, const float* init_state,
                            const int32_t* cu_seqlens, const float* dy, const float* dS_final, float* dq,
                            float* dk, float* dv, float* dg, float* dbeta, float* dS_init, void* workspace,
                            size_t workspace_bytes, gdn_stream_t stream);

/* Static, NUL-terminated name of a return code ("GDN_OK", "GDN_ERR_SHAPE", ...). */
const char* gdn_status_string(int code);

/*
 * Synchronises `stream`, then returns and clears the library's device status word for
 * the current device: GDN_OK, GDN_ERR_DEVICE_TIMEOUT if a bounded device-side wait gave up
 * since the last read, GDN_ERR_INDEX if a slot id or a cu_seqlens entry was out of range
 * (see gdn_decode_slots, gdn_prefill_conv_state), or GDN_ERR_CUDA if a kernel found its
 * launch shape inconsistent and did nothing.  Returns GDN_ERR_CUDA also if the
 * synchronisation fails.
 */
int gdn_read_device_status(gdn_stream_t stream);

/*
 * Optional per-kernel timing, for benchmarks.  While enabled, every kernel launch of later
 * gdn_prefill / gdn_decode calls is bracketed by CUDA events recorded on the call's stream
 * (the first 8192 launches after the last read are kept; later ones are dropped).  Host state
 * is process-wide and not thread-safe.  Returns GDN_OK or GDN_ERR_CUDA.
 */
int gdn_profile_enable(int on);

typedef struct gdn_kernel_time {
  const char* name;  /* static kernel name */
  int launches;      /* launches recorded */
  double total_ms;   /* summed event-to-event time of those launches */
} gdn_kernel_time_t;

/*
 * Waits for the recorded events, sums the time per kernel name into `out` (at most
 * max_entries entries) and clears the record.  Returns the number of entries written, or
 * GDN_ERR_NULL / GDN_ERR_CUDA.
 */
int gdn_profile_read(gdn_kernel_time_t* out, int max_entries);

/*
 * Size of the library's built-in prefill scratch used by gdn_prefill_noalloc: 64 MiB of
 * device memory per GPU that loads the library, held until the process exits.
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * gdn_prefill without a caller-provided workspace, for callers that cannot allocate
 * device memory at call time: code whose device memory is entirely owned by another
 * allocator (a serving framework's pre-reserved pool), or code that must not trigger the
 * device-wide synchronisation that cudaMalloc / cudaFree can cause inside a
 * latency-critical loop.  The pages define no such call; it exists only for such callers.
 *
 * Same arguments, layouts and results as gdn_prefill, minus workspace and its size.  The
 * scratch is a fixed array inside the library (GDN_NOALLOC_SCRATCH_BYTES); this call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - Returns GDN_ERR_WORKSPACE, launching nothing, when gdn_prefill_workspace_size(d)
 *     exceeds GDN_NOALLOC_SCRATCH_BYTES (at the pages' model shape, 16 QK / 32 value
 *     heads, one sequence: up to 960 packed tokens with bf16 inputs, 740 with fp32).
 *   - The first call on a device looks up that device's address of the scratch array
 *     (with that device current); make that first call before any stream capture.  The
 *     address is cached for the life of the process: it assumes the device's primary
 *     context is never torn down (no cudaDeviceReset between calls).
 *   - Every call on a device shares the one array, which keeps the previous call's
 *     contents; the prefill writes every scratch byte before reading it, so nothing needs
 *     clearing.  Calls whose work overlaps on the GPU (two streams, or two host threads)
 *     race on the array and corrupt each other's results: serialise them.
 */
int gdn_prefill_noalloc(const gdn_dims_t* d, const void* q, const void* k, const void* v,
                        const void* z, const float* a, const float* b, const float* A_log,
                        const float* dt_bias, const float* conv_w, const float* norm_w,
                        const float* init_state, const int32_t* cu_seqlens, void* y,
                        float* final_state, gdn_stream_t stream);

/*
 * Diagnostic: runs one tcgen05 operand-layout case of the bf16 tensor-core path on fixed
 * synthetic tiles (case 0: K-major A and B, 128x64x128; 1: K-major A, MN-major B, 128x32x128;
 * 2: K-major A, MN-major B, 128x32x64; 3: MN-major A and B, 128x32x64; 4: as 1 with A copied
 * into tensor memory and read from there; 5: 64x32x128 from the lower half of a 128-row A
 * tile), each product in
 * three bf16 hi/lo terms, and compares with the same products on CUDA cores.  Writes
 * out2[0] = max |difference|, out2[1] = max |reference| (host memory).  Synchronous;
 * allocates nothing.  Returns GDN_OK, GDN_ERR_NULL, GDN_ERR_SHAPE (bad case) or GDN_ERR_CUDA.
 */
int gdn_selftest_tc(int case_id, float* out2);

/*
 * Path options, process-wide (all devices, all threads).  The default, 0, is the fast path
 * of every call; each bit selects a slower alternative that computes the same result, for
 * comparisons and diagnostics:
 *   GDN_OPT_FORCE_FP32_PATH   bf16-input prefills take the fp32 FFMA path
 *   GDN_OPT_SEPARATE_NORM     the bf16 path's output norm runs in its own kernel
 *   GDN_OPT_NO_PDL            plain stream order between the prefill's kernels
 * The initial value is read once per process from the environment (GDN_FORCE_SIMT=1,
 * GDN_NO_FUSED_NORM=1, GDN_NO_PDL=1).  gdn_set_options replaces the word and
 * returns the previous one (unknown bits are dropped); it takes effect for calls made after
 * it.  Changing it while another host thread issues calls is allowed, but which value such a
 * call sees is unspecified.
 */
#define GDN_OPT_FORCE_FP32_PATH 1u
#define GDN_OPT_SEPARATE_NORM 2u
#define GDN_OPT_NO_PDL 4u
#define GDN_OPT_ALL 7u
uint32_t gdn_set_options(uint32_t flags);
uint32_t gdn_get_options(void);

/*
 * Limit of every bounded device-side wait of the tensor-core kernels (an mbarrier that the
 * bulk copies or the tensor cores complete, a peer CTA's exchange word), in nanoseconds of the
 * GPU's global timer, on the current device.  Default 2e9 (2 s).  A wait that runs out records
 * GDN_ERR_DEVICE_TIMEOUT in the device status word (gdn_read_device_status) and the kernel
 * leaves early: its outputs are then unspecified.  Synchronous (a copy to device memory on the
 * legacy default stream; call it with no library work in flight).  Returns GDN_OK,
 * GDN_ERR_SHAPE for 0, or GDN_ERR_CUDA.
 */
int gdn_set_wait_limit_ns(uint64_t ns);

/*
 * Diagnostic of the bounded waits: one CTA allocates tensor memory, initialises an mbarrier
 * that nothing will ever complete, and waits on it with the limit set by
 * gdn_set_wait_limit_ns, as the prefill kernels wait on theirs.  The wait runs out, the kernel
 * records GDN_ERR_DEVICE_TIMEOUT in the device status word, frees its tensor memory and
 * returns; no copy is in flight at any time.  Asynchronous on `stream`; read the result with
 * gdn_read_device_status(stream).  Returns GDN_OK or GDN_ERR_CUDA (launch failure).
 */
int gdn_selftest_wait_timeout(gdn_stream_t stream);

/* Library version as major * 10000 + minor * 100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN_H_ */
