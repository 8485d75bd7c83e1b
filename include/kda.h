/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) library,
 * libkda.so.
 *
 * The operator.  Per sequence n and head h, with a dk x dv fp32 state S
 * (row = key channel, column = value channel):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t,          alpha_t = exp(log_alpha_t)  (per key channel)
 *
 * Sources (page title and section):
 *   - "Kimi Linear" summary (pt.news.hada.io), "Controle fino de memoria no
 *     Kimi Delta Attention": a per-channel diagonal forget gate replaces the
 *     scalar gate of Gated DeltaNet; the transition is a specialised
 *     Diagonal-Plus-Low-Rank matrix tied to the key.
 *   - same page, "Algoritmo paralelo por chunks": fixed-size chunks, the
 *     final state of one chunk is the initial state of the next; WY / UT
 *     representation; lower-triangular inverse by forward substitution;
 *     output = inter-chunk recurrent term + intra-chunk parallel term.
 *   - same page, "Da atencao linear ao Gated DeltaNet": the delta rule and its
 *     Householder form.
 *   The pages print no equation; the update above is the plainest reading of
 *   their prose (decay first, output from the post-update state, no 1/sqrt(dk)
 *   query scale, natural-log gates).
 *
 * Conventions for every entry point
 * ---------------------------------
 *   - All tensor arguments are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains them.  Calls are asynchronous
 *     on `stream` (a cudaStream_t passed as void*; NULL = legacy default).
 *   - Arguments are validated on the host before anything is launched; a
 *     failing check returns an error status and launches nothing.
 *   - The library never aborts, asserts, traps or prints.
 *   - Alignment (KDA_ERR_ALIGN otherwise): S0, S_T, S and the workspace
 *     16 bytes; q, k, v, o and log_alpha 4 bytes (16 bytes on the tensor-core
 *     path, see kda_chunk_fwd); beta and cu_seqlens their element size.
 *   - Contiguous layouts (token-major, head next, channel innermost):
 *       q, k, log_alpha : [B, T, H, dk]        v, o : [B, T, H, dv]
 *       beta            : [B, T, H]
 *       S0, S_T, S      : [N, H, dk, dv] fp32, dv innermost
 *     With cu_seqlens (int32, N+1 non-decreasing offsets, cu[0] = 0,
 *     cu[N] = T) the batch is packed: B must be 1, T is the packed total and
 *     sequence n owns tokens [cu[n], cu[n+1]).  Without it N = B.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_ABI_VERSION 7

typedef enum {
  KDA_OK = 0,
  KDA_ERR_NULL = -1,        /* a required pointer is NULL                     */
  KDA_ERR_SHAPE = -2,       /* non-positive / inconsistent sizes              */
  KDA_ERR_DTYPE = -3,       /* unknown dtype code                             */
  KDA_ERR_ALIGN = -4,       /* a pointer is not aligned as required           */
  KDA_ERR_UNSUPPORTED = -5, /* valid but not implemented (e.g. dk not 64/128) */
  KDA_ERR_WORKSPACE = -6,   /* workspace missing or smaller than required     */
  KDA_ERR_CUDA = -7,        /* a CUDA runtime call or launch failed           */
  KDA_ERR_TIMEOUT = -8,     /* a device-side bounded wait gave up             */
  KDA_ERR_INTERNAL = -9,    /* a device-side consistency check failed         */
  KDA_ERR_ARGUMENT = -10    /* other invalid argument (bad cu_seqlens, flags) */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Problem description shared by all entry points. */
typedef struct kda_shape {
  int32_t B;          /* batch rows (must be 1 when cu_seqlens is given)     */
  int32_t T;          /* tokens per batch row; packed total with cu_seqlens  */
  int32_t H;          /* heads                                               */
  int32_t dk, dv;     /* key / value head dimensions: 64 or 128 each         */
  int32_t chunk;      /* chunk length C of the chunkwise form: must be 64    */
  int32_t n_seqs;     /* N = number of packed sequences (with cu_seqlens)    */
  int32_t io_dtype;   /* kda_dtype of q, k, v and o                          */
  int32_t gate_dtype; /* kda_dtype of log_alpha and beta                     */
  uint32_t flags;     /* KDA_FLAG_* bits                                     */
} kda_shape;

/* Copy cu_seqlens to the host and check it before launching.  This
 * synchronises `stream`; without the flag cu_seqlens is trusted. */
#define KDA_FLAG_VALIDATE_CU_SEQLENS 0x1u
/* Run the token-by-token CUDA-core recurrence (fp32, no chunking) even where
 * the tensor-core path applies; fp32 io and dk or dv = 64 always take it.  A
 * reference path for validation, not a fast one. */
#define KDA_FLAG_PATH_RECURRENT 0x4u
/* Where kda_chunk_fwd_gated applies its output epilogue on the tensor-core
 * path (neither: the library decides from the CTA split; both: invalid).
 * FUSED: in the prefill kernel's output warps; SEPARATE: in a pass over o
 * after the prefill.  Other flags are ignored by the other entry points. */
#define KDA_FLAG_GATE_FUSED 0x8u
#define KDA_FLAG_GATE_SEPARATE 0x10u
/* Tuning of the tensor-core path (0 = automatic): KDA_FLAG_STATE_CTAS(n)
 * fixes the number of state CTAs (each walks whole (sequence, head) chains),
 * KDA_FLAG_GRID_CTAS(n) caps the number of CTAs of the launch (at most one per
 * SM).  Values are clamped to what the problem and the device allow.
 * kda_chunk_fwd_workspace_size() depends on both. */
#define KDA_FLAG_STATE_CTAS(n) ((((uint32_t)(n)) & 0xFFu) << 8)
#define KDA_FLAG_GRID_CTAS(n) ((((uint32_t)(n)) & 0xFFu) << 16)

/*
 * kda_chunk_fwd_workspace_size -- preferred bytes of device workspace for
 * kda_chunk_fwd with `shape` on the CURRENT device.  0 on the CUDA-core path.
 * On the tensor-core path the workspace holds a few KB of counters and an
 * operand ring of 66,560-byte slots for each of R "state" CTAs (R is chosen
 * per call from the number of (sequence, head) pairs and the SM count, at
 * most one less than the SM count).  The preferred depth keeps the whole ring
 * within about 48 MB, so that it stays in L2 next to the streaming inputs,
 * with 4 to 16 slots per state CTA: at most ~50 MB on a 148-SM B200, and
 * independent of the sequence lengths.  Any workspace from a 2-slot to a
 * 16-slot ring works (deeper rings tolerate more imbalance between chains);
 * below 2 slots kda_chunk_fwd returns KDA_ERR_WORKSPACE.  Returns 0 for shapes
 * the library rejects; kda_chunk_fwd then reports the reason.
 */
size_t kda_chunk_fwd_workspace_size(const kda_shape* shape);

/*
 * kda_prefill_plan -- how the tensor-core prefill would run `shape` on a
 * device with num_sms SMs (num_sms <= 0: the current device's count): the
 * split of its one-CTA-per-SM grid into state CTAs (one serial chain of
 * chunks each, chains i, i + R, ...) and transform CTAs, the preferred
 * operand-ring depth per state CTA, whether kda_chunk_fwd_gated would fuse
 * the output epilogue (honouring KDA_FLAG_GATE_*), and the workspace sizes.
 * Host-only (with num_sms > 0 it touches no device).  KDA_ERR_UNSUPPORTED
 * for shapes the tensor-core path does not take.
 */
typedef struct kda_prefill_plan_info {
  int32_t state_ctas;        /* R                                                 */
  int32_t grid_ctas;         /* all CTAs of the launch                            */
  int32_t ring_depth;        /* operand-ring slots per state CTA (preferred)      */
  int32_t fuse_output_gate;  /* 1: in the prefill kernel; 0: a separate pass      */
  uint64_t workspace_bytes;      /* = kda_chunk_fwd_workspace_size on that device */
  uint64_t min_workspace_bytes;  /* the smallest workspace accepted (2-slot ring)  */
} kda_prefill_plan_info;
kda_status kda_prefill_plan(const kda_shape* shape, int32_t num_sms, kda_prefill_plan_info* out);

/*
 * kda_chunk_fwd -- chunkwise-parallel prefill ("Algoritmo paralelo por
 * chunks" on the Kimi Linear summary page): runs the recurrence above over
 * every token of every sequence and head, starting from S0.
 *
 *   q, k, log_alpha, v, beta  inputs (io_dtype / gate_dtype, layouts above).
 *                             log_alpha <= 0 is expected (alpha in (0,1]).
 *   S0          initial states [N, H, dk, dv] fp32, or NULL for zeros.
 *   cu_seqlens  NULL for a dense batch, else N+1 int32 offsets (B == 1).
 *   o           output [B, T, H, dv] in io_dtype; must not alias an input.
 *   S_T         final states [N, H, dk, dv] fp32, or NULL; may alias S0.
 *   workspace   device scratch (see kda_chunk_fwd_workspace_size; NULL
 *               allowed when that size is 0); contents on entry are ignored
 *               and on exit undefined.
 *
 * Paths: bf16 io with dk = dv = 128 runs on the tcgen05 tensor cores (fp32
 * state, bf16 operands, fp32 accumulation), one cooperative launch with one
 * CTA per SM: "state" CTAs each carry whole (sequence, head) chains through
 * their chunks, "transform" CTAs compute the state-independent per-chunk
 * operands in parallel and hand them over through a ring in the workspace.
 * q, k, v, log_alpha and o must then be 16-byte aligned (TMA reads, 16-byte
 * row stores).  fp32 io, dk or dv = 64, and KDA_FLAG_PATH_RECURRENT run the
 * fp32 token-by-token CUDA-core recurrence instead (it keeps fp32 inputs
 * within the 1e-4 tolerance; it is latency-bound, three barriers per token).
 * The chunk length is 64 on every path.  Sequences of length 0 copy S0 to
 * S_T.  The call must not overlap another use of the same workspace on the
 * GPU.
 */
kda_status kda_chunk_fwd(const kda_shape* shape, const void* q, const void* k, const void* v,
                         const void* log_alpha, const void* beta, const float* S0,
                         const int32_t* cu_seqlens, void* o, float* S_T, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd_gated -- kda_chunk_fwd followed by the per-head output
 * normalisation and gate that the "Kimi Linear" summary
 * (section "Configuracao do modelo Kimi Linear") applies after the operator
 * and before the output projection: an RMSNorm per head and a data-dependent
 * output gate.  The page gives no formula; this call computes, for every
 * token t and head h, over the dv values of o_t:
 *
 *     o'_t = o_t / sqrt(mean_j(o_t[j]^2) + eps) * norm_weight * sigmoid(g_t)
 *
 * and writes o' (io_dtype) to `o` in place of o_t; S_T is unchanged.
 *
 *   out_gate     g, [B, T, H, dv] in io_dtype (the gate's pre-activation, from
 *                the model's low-rank projection); 16-byte aligned.
 *   norm_weight  [dv] fp32, shared by all heads; 16-byte aligned.
 *   eps          >= 0, added to the mean square.
 * Everything else as kda_chunk_fwd, on every path.  The tensor-core prefill
 * applies the epilogue in its output warps where its state CTAs have time
 * to spare (short, many sequences), else a second kernel on `stream` applies
 * it to o in place (reads o and g, writes o); KDA_FLAG_GATE_FUSED /
 * KDA_FLAG_GATE_SEPARATE force either.  The CUDA-core paths apply it to each
 * token's o in their kernel (fp32 io with the accurate expf).  The
 * sigmoid is computed as (1 + tanh(g/2)) / 2 with the hardware tanh
 * approximation: within about 2.5e-4 absolute.
 */
kda_status kda_chunk_fwd_gated(const kda_shape* shape, const void* q, const void* k, const void* v,
                               const void* log_alpha, const void* beta, const float* S0, const int32_t* cu_seqlens,
                               const void* out_gate, const float* norm_weight, float eps, void* o, float* S_T,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * kda_chunk_fwd_layer -- the operator as the Kimi Linear layer uses it, with
 * its producer steps done inside the prefill kernel (the "Kimi Linear"
 * summary, section "Configuração do modelo Kimi Linear": q and k are
 * L2-normalised for the stability of the transition's eigenvalues; the
 * channel-wise decay gate comes from a low-rank projection through a decay
 * function like GDN's and Mamba's) and, optionally, its consumer step (the
 * per-head RMSNorm and output gate of kda_chunk_fwd_gated).  Equivalent to
 *
 *     kda_chunk_fwd(q / |q|, k / |k|, v, log_alpha, beta, ...)   with
 *     |x| = sqrt(sum_c x[c]^2 + KDA_QK_NORM_EPS) per (token, head) row and
 *     log_alpha[t][h][c] = -exp(A_log[h]) * softplus(gate_f[t][h][c] + dt_bias[h][c])
 *
 * followed by the output epilogue when out_gate is not NULL, without the
 * normalised q, k or log_alpha ever reaching HBM.
 *
 *   q, k      raw (not normalised) [B, T, H, dk] bf16.
 *   gate_f    the decay gate's projection output, [B, T, H, dk] bf16.
 *   A_log     [H] fp32 (the per-head rate is exp(A_log)); 4-byte aligned.
 *   dt_bias   [H, dk] fp32; 16-byte aligned.
 *   out_gate, norm_weight, eps   as kda_chunk_fwd_gated, or out_gate and
 *             norm_weight both NULL for no epilogue (one NULL: KDA_ERR_NULL).
 * Everything else as kda_chunk_fwd, on every path.  On the tensor-core path
 * gate_f must be bf16 (gate_dtype KDA_BF16, else KDA_ERR_UNSUPPORTED);
 * softplus and exp are evaluated in fp32 with the hardware 2^x and log2
 * approximations, and log alpha enters the chunk's cumulative sum with 16
 * significant bits (relative error below 2^-16; the bf16 log_alpha of
 * kda_chunk_fwd carries 8).  The CUDA-core paths (fp32 io, dk or dv = 64,
 * KDA_FLAG_PATH_RECURRENT) evaluate them with the accurate expf / log1pf.
 */
#define KDA_QK_NORM_EPS 1e-6f
kda_status kda_chunk_fwd_layer(const kda_shape* shape, const void* q, const void* k, const void* v,
                               const void* gate_f, const float* A_log, const float* dt_bias, const void* beta,
                               const float* S0, const int32_t* cu_seqlens, const void* out_gate,
                               const float* norm_weight, float eps, void* o, float* S_T, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * kda_decode_step_layer -- kda_decode_step (or, with state_slots,
 * kda_decode_step_slots) with the layer's producer steps in the kernel and
 * the optional output epilogue, as kda_chunk_fwd_layer defines them: q, k
 * raw [B, 1, H, dk]; gate_f [B, 1, H, dk] in the gate dtype; A_log [H] and
 * dt_bias [H, dk] fp32 (4-byte aligned); state dense [B, H, dk, dv] fp32
 * (state_slots NULL) or a pool of num_slots slots; out_gate [B, 1, H, dv]
 * (io dtype, 16-byte aligned) and norm_weight [dv] fp32, or both NULL.  The
 * decode kernel applies the epilogue to each o before storing it.  Every
 * shape of kda_decode_step is supported.
 */
kda_status kda_decode_step_layer(const kda_shape* shape, const void* q, const void* k, const void* v,
                                 const void* gate_f, const float* A_log, const float* dt_bias, const void* beta,
                                 float* state, const int32_t* state_slots, int32_t num_slots, const void* out_gate,
                                 const float* norm_weight, float eps, void* o, void* stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate.
 *
 * The pages have no counterpart to this call; it is a convenience of this
 * library.  Some callers have no way to obtain device memory where they run
 * the prefill: a plugin loaded into a framework whose memory pool already
 * owns the GPU and offers no allocator across a C boundary, or a
 * latency-critical serving loop that bans cudaMalloc because it synchronises
 * the device and stalls every other stream.  This call takes the arguments of
 * kda_chunk_fwd without the workspace and runs the same path, with the
 * tensor-core path's workspace (its operand ring and counters) in a fixed
 * scratch array that lives in the library's device image.
 *
 *   - The array holds KDA_NOALLOC_SCRATCH_BYTES (64 MiB).  Every GPU that
 *     loads the library reserves it until the process exits.
 *   - The tensor-core path sizes its operand ring to what fits the array (2
 *     to 16 slots per state CTA).  A shape that cannot fit even the 2-slot
 *     ring is rejected with KDA_ERR_WORKSPACE before anything is launched; on
 *     a 148-SM B200 that ring needs at most ~20 MB, so no valid shape is
 *     rejected there.  The CUDA-core path needs no scratch.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress)
 *     on the current device; the lookup allocates nothing.  The first call on
 *     a device may load the library's device code there, so make that first
 *     call before any stream capture begins.
 *   - Every call shares the one array, which keeps the last call's contents.
 *     The counters that must start at zero are cleared on the stream at the
 *     start of every call; every other byte is written before it is read.
 *     Calls whose executions overlap on the GPU (different streams or host
 *     threads) race on the array: serialise them.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

kda_status kda_chunk_fwd_noalloc(const kda_shape* shape, const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta, const float* S0,
                                 const int32_t* cu_seqlens, void* o, float* S_T, void* stream);

/*
 * kda_decode_step -- one recurrent token for each of B independent
 * (sequence, head) states, updated in place (the constant-size recurrent
 * state of the "Kimi Linear" articles: one read and one write of S).
 *
 *   shape       B = number of sequences, T must be 1, chunk is ignored.
 *   q, k, log_alpha : [B, H, dk];  v, o : [B, H, dv];  beta : [B, H].
 *   S           [B, H, dk, dv] fp32, read and overwritten with the new state.
 *   o           output; must not alias any input.
 */
kda_status kda_decode_step(const kda_shape* shape, const void* q, const void* k, const void* v,
                           const void* log_alpha, const void* beta, float* S, void* o,
                           void* stream);

/*
 * Serving-state variants.  A serving engine keeps the recurrent states of its
 * live requests in one pool, [num_slots, H, dk, dv] fp32, and hands each
 * batch an int32 slot index per sequence (continuous batching: the batch is
 * a permutation of live requests, not a prefix of the pool).  These calls
 * read and write the states in place in the pool through that index; they
 * are otherwise kda_chunk_fwd and kda_decode_step.
 *
 *   state_pool     [num_slots, H, dk, dv] fp32 device array, 16-byte aligned;
 *                  read and overwritten in place.
 *   num_slots      rows of the pool (> 0).
 *   state_slots    int32 device array with one entry per sequence (N for the
 *                  prefill, B for the decode step).  slot >= 0: the state of
 *                  that sequence lives in that pool row.  slot < 0: padding,
 *                  the sequence has no cached state: it runs from a zero state
 *                  and its final state is dropped (its output is still
 *                  written).  slot >= num_slots is refused on the device: that
 *                  sequence is treated as padding and the call records
 *                  KDA_ERR_ARGUMENT for kda_check_device_error.
 *                  Non-negative slots of one call must be distinct (two
 *                  sequences writing one row give an undefined state).
 *   has_initial_state  (prefill only) uint8 device array, one per sequence:
 *                  0 = start from zeros (a new request; the pool row's old
 *                  contents are ignored), else resume from the state in the
 *                  pool (a prompt continued after a cached prefix, or a
 *                  chunked prefill).  NULL = resume for every sequence.
 *
 * The other arguments, the paths and the errors are those of kda_chunk_fwd
 * (workspace: kda_chunk_fwd_workspace_size) and kda_decode_step.
 */
kda_status kda_chunk_fwd_slots(const kda_shape* shape, const void* q, const void* k, const void* v,
                               const void* log_alpha, const void* beta, float* state_pool, int32_t num_slots,
                               const int32_t* state_slots, const uint8_t* has_initial_state,
                               const int32_t* cu_seqlens, void* o, void* workspace, size_t workspace_bytes,
                               void* stream);

kda_status kda_decode_step_slots(const kda_shape* shape, const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta, float* state_pool, int32_t num_slots,
                                 const int32_t* state_slots, void* o, void* stream);

/*
 * kda_check_device_error -- synchronises `stream`, then returns and clears
 * the error code a kernel recorded on the current device (a bounded wait
 * that gave up reports KDA_ERR_TIMEOUT).  KDA_OK when none was recorded.
 */
kda_status kda_check_device_error(void* stream);

/* Static, human-readable text for a status code. */
const char* kda_status_string(kda_status status);

/* KDA_ABI_VERSION of the built library. */
int32_t kda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
