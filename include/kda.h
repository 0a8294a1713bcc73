/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention forward library.
 *
 * Kimi Delta Attention (KDA) keeps, per head, a fixed-size dk x dv fp32
 * state S that every token rewrites in place:
 *
 *     alpha_t = exp(max(g_t, g_floor))                      (per key channel)
 *     S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t     = scale * S_t^T q_t           [* sigmoid(z_t) with an output gate]
 *
 * Sources (web pages on Kimi K3, cited by title and section):
 *   - "Kimi-K3 为什么这么强？", §① ②: per-channel diagonal gate Diag(alpha)
 *     replacing gated DeltaNet's scalar gate; the three-step update (every row
 *     forgets at its own rate, the current key's row keeps (1 - beta), the new
 *     value is written as an interpolation).
 *   - "Kimi K3 深度拆解", 突破一: the transition is diagonal-plus-low-rank.
 *   - fupanwang.com Kimi K3 report digest, section
 *     "KDA：百万上下文先要过「数值 算子」这一关": fixed-size recurrent state; a
 *     lower bound on the per-step log-decay keeps the cumulative decay of a
 *     16-token block inside BF16 range so the diagonal block runs on dense
 *     tensor cores (Fig. 3); the output gate is an input-dependent channel
 *     switch on the recurrence output.  Section "基础设施": chunked prefill
 *     (intra-chunk parallel, overlapped with cross-chunk state passing) and
 *     context parallelism by segment states and a prefix scan.
 *   - "Kimi K3 技术深度解析", §一: the state is a snapshot updated in place
 *     during decode.
 *   The pages do not print the floor formula; here it is max(g, g_floor) with
 *   g_floor a parameter (default -5).
 *
 * Conventions for every entry point
 *   - Pointers marked "device" are CUDA device pointers on the current device;
 *     the caller allocates and owns every buffer (inputs, outputs, workspace).
 *     The library never allocates device memory.
 *   - Calls are asynchronous and ordered on `stream`; nothing is synchronised
 *     except in kda_get_device_status.  A call returns before its kernels run.
 *   - Arguments are validated on the host before anything is launched; a bad
 *     argument returns an error status and launches nothing.  No exception,
 *     abort or exit crosses the ABI.
 *   - Layouts are contiguous row-major:
 *       q, k, g      [T_tot, H, dk]       v, o, gate   [T_tot, H, dv]
 *       beta         [T_tot, H]           S0, S_T      [N, H, dk, dv] (fp32)
 *     A fixed-length batch [B, T, H, d] is the same memory with
 *     cu_seqlens = {0, T, 2T, ..., BT}.
 *   - io_dtype KDA_BF16: q, k, v, g, beta, gate and o are bf16; the state is
 *     always fp32.  KDA_FP32: every tensor is fp32.
 *   - dk and dv must each be 64 or 128.
 *   - g is the per-step log-decay (natural log) and must be <= 0 (a
 *     precondition, not checked); values below g_floor act as g_floor.
 *     g_floor must lie in [-5.45, 0] so that exp(16 * g_floor) and its inverse
 *     stay normal fp32/bf16 numbers.
 */
#ifndef KDA_B200_KDA_H
#define KDA_B200_KDA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, overlap, bad cu_seqlens */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. dk = 96)        */
    KDA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required       */
    KDA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed             */
    KDA_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up               */
    KDA_ERR_DEVICE_BOUNDS = 6  /* a device-side bounds check fired                 */
} kda_status;

typedef enum { KDA_BF16 = 0, KDA_FP32 = 1 } kda_dtype;

/* Description of one chunked prefill call. */
typedef struct {
    int64_t total_tokens;  /* T_tot: packed tokens over all sequences (>= 0)           */
    int32_t num_seqs;      /* N >= 1                                                    */
    int32_t num_heads;     /* H >= 1                                                    */
    int32_t dk, dv;        /* 64 or 128 each                                            */
    kda_dtype io_dtype;
    float scale;           /* read-out scale; pass 1/sqrt(dk) for the usual choice      */
    float g_floor;         /* lower bound on the log-decay; -5 is the usual choice      */
    int32_t chunk;         /* 0 = automatic, 16 or 64: a tiling choice, not semantics  */
    int32_t max_seqlen;    /* longest sequence if known, else 0                         */
} kda_fwd_desc;

/*
 * Bytes of device workspace kda_chunk_fwd needs for `desc` (always a multiple
 * of 256).  `cu_seqlens_host` (N+1 host int32, nullable) lets the library plan
 * the long-sequence segment split; the same pointer (or the same values) must
 * then be passed to kda_chunk_fwd.  Returns 0 when no workspace is needed and
 * SIZE_MAX when the description itself is invalid.
 */
size_t kda_chunk_fwd_workspace_size(const kda_fwd_desc *desc,
                                    const int32_t *cu_seqlens_host);

/*
 * Chunked prefill over variable-length packed sequences (the FlashKDA role:
 * intra-chunk work in parallel, the state carried chunk to chunk).
 *
 *   q, k, g, v, beta  device, io_dtype, layouts above (read only)
 *   S0                device fp32 [N,H,dk,dv] initial states, or NULL = zeros
 *   cu_seqlens        device int32 [N+1], non-decreasing, cu_seqlens[0] = 0,
 *                     cu_seqlens[N] = total_tokens.  A length-0 sequence
 *                     returns S_T = S0 for it and writes no output rows.
 *   cu_seqlens_host   host copy of cu_seqlens or NULL; when given it is
 *                     validated (monotone, ends at total_tokens) and used to
 *                     order work longest-first and to split long sequences.
 *   gate              device io_dtype [T_tot,H,dv] gate logits z, or NULL;
 *                     when given o = o * sigmoid(z) elementwise.
 *   o                 device io_dtype [T_tot,H,dv] output (must not overlap
 *                     any input)
 *   S_T               device fp32 [N,H,dk,dv] final states, or NULL; must not
 *                     overlap S0 or any input.
 *   workspace         device buffer of at least
 *                     kda_chunk_fwd_workspace_size(desc, cu_seqlens_host)
 *                     bytes, 256-byte aligned; may be NULL when that size is 0.
 *
 * bf16 outputs are rounded to nearest even from fp32.
 */
kda_status kda_chunk_fwd(const kda_fwd_desc *desc,
                         const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *S0,
                         const int32_t *cu_seqlens,
                         const int32_t *cu_seqlens_host,
                         const void *gate, void *o, float *S_T,
                         void *workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/* Description of one decode step: `batch` sequences, one token each. */
typedef struct {
    int32_t batch;       /* B >= 1 */
    int32_t num_heads;   /* H >= 1 */
    int32_t dk, dv;      /* 64 or 128 each */
    kda_dtype io_dtype;
    float scale;
    float g_floor;
} kda_decode_desc;

/*
 * One decode step ("snapshot instead of log": the state is rewritten in place).
 *
 *   q, k, g   device io_dtype [B,H,dk];  v device io_dtype [B,H,dv]
 *   beta      device io_dtype [B,H]
 *   S         device fp32 [B,H,dk,dv], read and overwritten with the new state
 *   gate      device io_dtype [B,H,dv] gate logits, or NULL
 *   o         device io_dtype [B,H,dv] output (must not overlap S or inputs)
 */
kda_status kda_decode_step(const kda_decode_desc *desc,
                           const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *S,
                           const void *gate, void *o, cudaStream_t stream);

/*
 * Speculative-decode verify and commit (the replay of the Kimi K3 report
 * digest, section 基础设施: the target model checks D draft tokens at once,
 * then only the accepted prefix is committed to the state, in place).
 * Acceptance is decided outside attention, from the outputs, so these are
 * two calls over the same D tokens per sequence:
 *   kda_spec_verify: outputs of all D tokens, as D consecutive decode steps
 *                    from S would give them; S is only read.
 *   kda_spec_commit: applies the first accepted[b] tokens of sequence b
 *                    (clamped to [0, D]) to S in place; 0 leaves S untouched.
 * Each call streams every head's state once, whatever D is (D decode steps
 * would stream it D times in each direction).
 *
 *   q, k, g  device io_dtype [B, D, H, dk] (token-major per sequence)
 *   v        device io_dtype [B, D, H, dv];  beta  device io_dtype [B, D, H]
 *   S        device fp32 [B, H, dk, dv], 16-byte aligned
 *   gate     device io_dtype [B, D, H, dv] gate logits or NULL (verify only)
 *   o        device io_dtype [B, D, H, dv] (verify) -- must not overlap S or inputs
 *   accepted device int32 [B] (commit)
 * Returns KDA_ERR_INVALID_ARG for a bad descriptor (draft outside
 * 1..KDA_SPEC_MAX_DRAFT), null pointers or overlaps, KDA_ERR_UNSUPPORTED for
 * head sizes other than 64 or 128, KDA_ERR_CUDA if the launch fails.
 */
#define KDA_SPEC_MAX_DRAFT 64

typedef struct {
    int32_t batch, num_heads, dk, dv;
    int32_t draft;              /* D, tokens per sequence */
    kda_dtype io_dtype;
    float scale, g_floor;
} kda_spec_desc;

kda_status kda_spec_verify(const kda_spec_desc *desc, const void *q, const void *k, const void *v,
                           const void *g, const void *beta, const float *S, const void *gate,
                           void *o, cudaStream_t stream);

kda_status kda_spec_commit(const kda_spec_desc *desc, const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *S, const int32_t *accepted,
                           cudaStream_t stream);

/*
 * kda_chunk_fwd without any caller-provided device memory.  The pages have
 * no counterpart to this entry point: it exists for callers that cannot hand
 * the library a workspace, such as a plugin interface that passes only the
 * input and output buffers, or a runtime that plans all device memory up
 * front and allows no allocation once it runs.
 *
 * Arguments are those of kda_chunk_fwd minus cu_seqlens_host and the
 * workspace; the results agree with kda_chunk_fwd's within the parity
 * tolerances.  Without cu_seqlens_host this entry point never splits a long
 * sequence into segments: every (sequence, head) pair runs as one CTA, so
 * with fewer pairs than SMs (one long sequence, few heads) it leaves SMs
 * idle and rounds differently from kda_chunk_fwd, which splits such
 * sequences.  The scratch it needs
 * (one int32 per sequence) is a fixed array inside the library, sized for
 * KDA_NOALLOC_MAX_SEQS sequences; every GPU that loads the library keeps
 * that array (256 KiB) until the process exits.
 *   - num_seqs > KDA_NOALLOC_MAX_SEQS returns KDA_ERR_WORKSPACE and launches
 *     nothing.
 *   - The call allocates no device or host memory.
 *   - The first call in each context looks up the array's device address
 *     (with that device current); make that first call before any stream
 *     capture begins on the device.  The address is cached with the context
 *     it belongs to: after cudaDeviceReset (or any new primary context) the
 *     next call looks it up again.
 *   - All calls on a device share the one array and it keeps the last
 *     call's contents (each call rewrites the part it reads before reading
 *     it).  Calls whose kernels can overlap on the GPU -- on different
 *     streams without ordering between them -- race on the array: order them
 *     on one stream or with events.
 */
#define KDA_NOALLOC_MAX_SEQS 65536
kda_status kda_chunk_fwd_noalloc(const kda_fwd_desc *desc,
                                 const void *q, const void *k, const void *v,
                                 const void *g, const void *beta, const float *S0,
                                 const int32_t *cu_seqlens, const void *gate,
                                 void *o, float *S_T, cudaStream_t stream);

/*
 * Synchronises `stream`, then reads and clears this device's error word,
 * which kernels set when a bounded wait gives up (KDA_ERR_TIMEOUT) or a
 * device-side bounds check fires (KDA_ERR_DEVICE_BOUNDS).  The word is shared
 * by every call on the device.  Returns KDA_ERR_CUDA if the sync fails.
 */
kda_status kda_get_device_status(cudaStream_t stream);

/*
 * State snapshots at token offsets (the prefix-cache hook: a cache of states
 * at positions that are multiples of a hash granularity, Kimi K3 report
 * digest, section 基础设施).  For sequence n and m = 1 .. floor(L_n /
 * interval), slot base[n] + m - 1 of `states` receives the state after the
 * sequence's first m * interval tokens (S0 included): fp32 [dk x dv] per
 * head, laid out [total][num_heads][dk][dv].
 *   interval: tokens between snapshots, a positive multiple of 64.
 *   total:    slots in `states` (0: no snapshots are written).
 *   base:     device array of num_seqs + 1 int64, normally the exclusive
 *             prefix sum of floor(L_n / interval).  The kernels check every
 *             slot against [0, total) and record KDA_ERR_DEVICE_BOUNDS
 *             (kda_get_device_status) instead of writing outside it.
 *   states:   device, caller-owned; must not overlap any other buffer.
 */
typedef struct {
    int32_t interval;
    int64_t total;
    const int64_t *base;
    float *states;
} kda_snapshots;

/*
 * kda_chunk_fwd plus state snapshots (see kda_snapshots): the same
 * arguments, checks and results, and in addition the snapshot states.  With
 * cu_seqlens_host given, the slots the sequences need are also checked
 * against snap->total on the host.  Returns KDA_ERR_INVALID_ARG for a null
 * `snap`, a bad interval or overlapping snapshot buffers.
 */
kda_status kda_chunk_fwd_snapshots(const kda_fwd_desc *desc, const kda_snapshots *snap,
                                   const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const float *S0, const int32_t *cu_seqlens,
                                   const int32_t *cu_seqlens_host, const void *gate, void *o,
                                   float *S_T, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * kda_chunk_fwd from and to HOST memory: q, k, v, g, beta, gate, S0 (inputs)
 * and o, S_T (outputs) are host pointers in the layouts of kda_chunk_fwd;
 * cu_seqlens_host (host) is required.  The batch is cut into up to 8 groups
 * of whole sequences and pipelined over three streams: the host-to-device
 * copy of group i+1 and the device-to-host copy of group i-1 overlap the
 * prefill of group i on `stream`.  Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister) for the copies to overlap; pageable
 * ones work but serialise.  The device workspace (256-byte aligned) holds two
 * input and two output slots and the prefill's own workspace:
 * kda_chunk_fwd_host_workspace_size(desc, cu_seqlens_host, with_gate,
 * with_S0, with_S_T) bytes.  When the call returns the work is enqueued;
 * synchronising `stream` waits for every copy.  Calls on one device are
 * serialised while they enqueue (they share two copy streams).  Errors as
 * kda_chunk_fwd; KDA_ERR_WORKSPACE for a short or misaligned workspace.  An
 * error after the first group was enqueued can leave copies in flight:
 * synchronise the device before reusing the buffers.
 */
size_t kda_chunk_fwd_host_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host,
                                         int32_t with_gate, int32_t with_S0, int32_t with_S_T);
kda_status kda_chunk_fwd_host(const kda_fwd_desc *desc, const void *q, const void *k, const void *v,
                              const void *g, const void *beta, const float *S0,
                              const int32_t *cu_seqlens_host, const void *gate, void *o, float *S_T,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward of the prefill (training; the report digest's FlashKDA serves
 * training and prefill, section 基础设施): the gradients of
 * L = sum(o * dout) + sum(S_T * dS_T) through the recurrence of
 * kda_chunk_fwd, with the same descriptor, inputs and layouts.
 *   dout   [T][H][dv], dtype of the inputs: gradient of o (required).
 *   dS_T   fp32 [num_seqs][H][dk][dv]: gradient of the final state, or NULL (zero).
 *   dq, dk, dg [T][H][dk]; dv [T][H][dv]; dbeta [T][H]: written, input dtype.
 *   dgate  [T][H][dv]: written when gate is given (required then).
 *   dS0    fp32 [num_seqs][H][dk][dv]: gradient of S0, written when not NULL.
 * S0, dS_T and dS0 must be 16-byte aligned.
 * The derivative of max(g, g_floor) is taken as 1 where g >= g_floor.
 * cu_seqlens_host is required.  Internally the forward runs once with state
 * snapshots every 64 tokens into the workspace.  Then, for bf16 I/O with
 * dk = dv = 128 and 16-byte aligned q, k, g, dout and gate, the chunked form:
 * per 64-token chunk the gradient chain's constants, the chain over the
 * chunks (two CTAs per sequence and head, half the value columns each),
 * and every gradient of a chunk from its start state and the gradient
 * reaching its end (tensor-core products);
 * otherwise (fp32 I/O, other head sizes, unaligned tensors) one CTA per
 * (sequence, head) recomputes each chunk's states from its snapshot and runs
 * the recurrence backwards token by token.  The results match the gradients
 * of the token recurrence within the parity tolerances (largest error over the
 * output's RMS: fp32 I/O 1e-4; bf16 I/O 2e-2 beyond half a bf16 ulp).  Workspace
 * (device, 256-byte aligned):
 * kda_chunk_bwd_workspace_size(desc, cu_seqlens_host) bytes (SIZE_MAX for a
 * bad descriptor).  dk, dv in {64, 128}, else KDA_ERR_UNSUPPORTED;
 * KDA_ERR_INVALID_ARG for null, overlapping or inconsistent arguments,
 * KDA_ERR_WORKSPACE for a short or misaligned workspace.  Asynchronous.
 */
size_t kda_chunk_bwd_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host);
kda_status kda_chunk_bwd(const kda_fwd_desc *desc, const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *S0, const int32_t *cu_seqlens,
                         const int32_t *cu_seqlens_host, const void *gate, const void *dout,
                         const float *dS_T, void *dq, void *dk, void *dv, void *dg, void *dbeta,
                         void *dgate, float *dS0, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * Context-parallel prefill across GPUs (KCP, Kimi K3 report digest, section
 * 基础设施): a long sequence is cut into contiguous pieces, one per rank.
 * Over a piece the state map is affine, S_end = M S_start + S_loc, with M the
 * product of the piece's transitions (I - beta k k^T) Diag(alpha), latest on
 * the left, and S_loc the state the piece grows from S_start = 0.  Every rank
 * summarises its piece (kda_segment_summary), the summaries are all-gathered
 * (the caller's collective; a fixed 2 x dk x dv fp32 per sequence and head),
 * each rank folds those of the ranks before it into its start state
 * (kda_state_combine) and reruns its piece from there with outputs
 * (kda_chunk_fwd with S0 = that state).
 *
 * kda_segment_summary: for each sequence n of the batch (desc, q, k, v, g,
 * beta and cu_seqlens as in kda_chunk_fwd; the piece of sequence n on this
 * rank is tokens cu_seqlens[n] .. cu_seqlens[n+1]):
 *   S_loc [num_seqs][num_heads][dk][dv] fp32, device: the state after the
 *         piece starting from S0 (if given, fp32 [num_seqs][num_heads][dk][dv])
 *         or from zero.  Required.
 *   M     [num_seqs][num_heads][dk][dk] fp32, device: the transition product,
 *         or NULL to skip it (the first piece of a sequence needs none).
 * cu_seqlens_host (num_seqs + 1 int32, host) is required: the work list is
 * built on the host.  When the chains are fewer than the SMs, long pieces are
 * cut into sub-segments whose summaries the scan kernel folds (the same
 * decomposition one level down).  The workspace (device, 256-byte aligned)
 * must hold kda_segment_summary_workspace_size(desc, cu_seqlens_host,
 * M != NULL) bytes.  S_loc and M must be 16-byte aligned.  Covers bf16 I/O
 * with dk = dv = 128 (the tensor-core kernel), else KDA_ERR_UNSUPPORTED.
 * KDA_ERR_INVALID_ARG for a bad descriptor, null or overlapping buffers or
 * bad host seqlens; KDA_ERR_WORKSPACE for a short workspace.  Asynchronous on
 * `stream`.
 */
size_t kda_segment_summary_workspace_size(const kda_fwd_desc *desc, const int32_t *cu_seqlens_host,
                                          int32_t with_M);
kda_status kda_segment_summary(const kda_fwd_desc *desc, const void *q, const void *k,
                               const void *v, const void *g, const void *beta, const float *S0,
                               const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                               float *S_loc, float *M, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Folds P = num_summaries piece summaries, in piece order, into the start
 * state of piece P:  S = S_loc(0);  S = M(p) S + S_loc(p) for p = 1 .. P-1
 * (M(0) is not read: the first piece's S_loc already starts from S0).
 *   summaries: device fp32 [P][2][num_seqs][num_heads][dk][dv]: per piece,
 *              S_loc then M (dk = dv), which is what an all-gather of each
 *              rank's contiguous (S_loc, M) buffer produces.
 *   S_in:      device fp32 [num_seqs][num_heads][dk][dv], written.
 * Both 16-byte aligned and disjoint.  dk = dv = 128, else
 * KDA_ERR_UNSUPPORTED; KDA_ERR_INVALID_ARG for P < 1 or bad sizes or
 * pointers.  Asynchronous on `stream`.
 */
typedef struct {
    int32_t num_seqs;
    int32_t num_heads;
    int32_t dk;
    int32_t dv;
    int32_t num_summaries;
} kda_combine_desc;

kda_status kda_state_combine(const kda_combine_desc *desc, const float *summaries, float *S_in,
                             cudaStream_t stream);

/*
 * Diagnostic (the pages have no counterpart): runs one bounded device-side
 * wait on a barrier that nothing completes, with the same wait primitive the
 * prefill kernels use, so that the timeout path can be exercised without a
 * hang or a fault.  The wait gives up after `max_polls` polls (1 .. 65536),
 * sets the timeout bit of the device error word and the kernel returns; read
 * it with kda_get_device_status (which reports KDA_ERR_TIMEOUT and clears
 * it).  Returns KDA_ERR_INVALID_ARG for a poll count outside that range,
 * KDA_ERR_CUDA if the launch fails, else KDA_OK.
 */
kda_status kda_selftest_bounded_wait(int32_t max_polls, cudaStream_t stream);

/* Static, human-readable name of a status code. */
const char *kda_status_string(kda_status status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_KDA_H */
