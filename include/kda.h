/*
 * kda.h — C ABI of the KDA (Kimi Delta Attention) library for NVIDIA B200 (sm_100a).
 *
 * The operation. "Kimi Linear：让长上下文大模型真正实用的线性注意力架构" (juejin.cn),
 * section 三 5️⃣ gives the KDA update rule
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *
 * (beta = learning rate, alpha = forget rate, S = memory state); section 三 1️⃣
 * says the forget rate is per channel (alpha_t[i], one per key channel). The
 * library reads out with the updated state, o_t = scale * S_t^T q_t, and takes
 * the gate in log space, alpha_t = exp(log_alpha_t). S is dk x dv per head, so
 * Diag(alpha_t) scales the dk rows of S.
 *
 * Layouts. Every tensor is a dense, row-major DEVICE buffer, 16-byte aligned:
 *   q, k        [B, T, H, dk]   dtype given by qkv_dtype (fp32 or bf16)
 *   v, o        [B, T, H, dv]   qkv_dtype (o has the same dtype as q, k, v)
 *   log_alpha   [B, T, H, dk]   fp32, expected <= 0 (alpha in (0, 1])
 *   beta        [B, T, H]       fp32
 *   S0, S_final [N, H, dk, dv]  fp32, dv contiguous
 * Sequences: without cu_seqlens, N = B and row b of the batch is one sequence of
 * T tokens. With cu_seqlens (int32 [n_seqs + 1], device memory, cu_seqlens[0] = 0,
 * non-decreasing, cu_seqlens[n_seqs] = T) the batch must have B = 1 and sequence
 * n owns the packed tokens [cu_seqlens[n], cu_seqlens[n+1]); N = n_seqs. Zero-
 * length sequences are allowed (their S_final equals their S0).
 *
 * Supported sizes: dk = dv in {32, 64, 128}. bf16 inputs with dk = dv = 128 run on
 * the tcgen05 tensor-core path; all other supported cases run on the fp32 SIMT
 * path (see kda_chunk_fwd_ex).
 *
 * Ownership and asynchrony. The caller owns every buffer, including the
 * workspace; the library allocates no device memory and never synchronises the
 * stream. Calls are enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 * the legacy default stream) and return once the launches are queued. Buffers
 * must stay valid until the stream reaches that point. Concurrent calls on
 * different streams need separate workspaces.
 *
 * Errors. Arguments are checked on the host before anything is launched; a bad
 * argument returns an error status and launches nothing. A failed launch returns
 * KDA_ERR_CUDA. The library never aborts, exits or traps. Every wait inside the
 * tensor-core kernels is bounded; a wait that runs out makes the kernel return
 * early and records a nonzero code in the prefill workspace's status word, so
 * the results of that call are not valid. The word is read by
 * kda_chunk_fwd_status (after the call) or, with KDA_DEBUG_SYNC=1 in the
 * environment, by every prefill call itself, which then waits for its work and
 * returns KDA_ERR_DEVICE_STATUS.
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad cu_seqlens shape */
    KDA_ERR_UNSUPPORTED = 2,   /* head size or dtype the library does not implement */
    KDA_ERR_ALIGNMENT = 3,     /* a buffer is not 16-byte aligned */
    KDA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    KDA_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    KDA_ERR_DEVICE_STATUS = 6  /* a kernel gave up a bounded wait: results invalid */
} kda_status_t;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype_t;

/* Prefill algorithm selector for kda_chunk_fwd_ex. */
typedef enum {
    KDA_ALGO_AUTO = 0,    /* tcgen05 path when supported, else SIMT */
    KDA_ALGO_SIMT = 1,    /* fp32 CUDA-core path: any supported dtype and size */
    KDA_ALGO_TCGEN05 = 2, /* tensor-core path: bf16, dk = dv = 128 only */
    KDA_ALGO_TCGEN05_SEQUENTIAL = 3  /* tensor-core path without the time split */
} kda_algo_t;

/* Human-readable name of a status code (static storage; never NULL). */
const char *kda_status_string(kda_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
int kda_version(void);

/* Number of kernels this library has launched in this process so far (all
 * entry points, all devices). Differences of two readings count the launches
 * of the calls made in between. */
unsigned long long kda_launch_count(void);

/*
 * Device status of the last prefill that used `workspace` (any kda_*chunk_fwd*
 * entry point, either phase). The library defines no counterpart on the pages;
 * it reports whether the kernels' own failure detection fired. Reads the
 * workspace's status word on `stream` and waits for the stream. The prepare
 * phase clears the word; a later failure in either phase sets it to a nonzero
 * code (the first failing wait's), which stays until the next prepare.
 *   workspace, workspace_bytes  the prefill's workspace (>= 256 bytes)
 *   device_code                 receives the word (0: no wait ran out)
 * Returns KDA_OK, KDA_ERR_DEVICE_STATUS when the word is nonzero, or an
 * argument / CUDA error.
 */
kda_status_t kda_chunk_fwd_status(const void *workspace, size_t workspace_bytes,
                                  int *device_code, void *stream);

/*
 * Debugging aid for the failure path (process-wide; not needed in normal use):
 * `polls` replaces the poll limit of every bounded wait in the tensor-core
 * kernels launched afterwards (0 restores the default of 2^20 polls), and a
 * nonzero `starve_carry` makes the sequential kernel's copy producer issue no
 * copies, so that its first wait on a chunk record runs out while nothing
 * asynchronous is in flight. The kernels then return early and the status word
 * reports the failure. Always returns KDA_OK.
 */
kda_status_t kda_debug_set_wait_limit(unsigned int polls, int starve_carry);

/*
 * Workspace bytes that kda_chunk_fwd needs for this problem, i.e. for the path
 * KDA_ALGO_AUTO selects (0 on invalid sizes). The workspace holds the per-chunk intermediate matrices of the
 * chunked form between the chunk-parallel and the sequential kernel; it is
 * device memory owned by the caller, needs no initialisation and may be reused
 * across calls on the same stream. For varlen calls pass B = 1, T = total
 * packed tokens and n_seqs = number of sequences; otherwise n_seqs is ignored.
 */
size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs,
                                    kda_dtype_t qkv_dtype);

/* Workspace bytes kda_chunk_fwd_ex needs with the given kda_algo_t (the size for
 * the path that algo selects; KDA_ALGO_AUTO gives the same value as
 * kda_chunk_fwd_workspace_size). 0 on invalid sizes or an unsupported algo. */
size_t kda_chunk_fwd_workspace_size_ex(int B, int T, int H, int dk, int dv, int n_seqs,
                                       kda_dtype_t qkv_dtype, int algo);

/*
 * Chunked prefill: runs the recurrence over every sequence from S0 (NULL = zero
 * state), writes o for every token and, if S_final is not NULL, the state after
 * each sequence's last token. Source: the update rule above ("Kimi Linear"
 * juejin.cn page, section 三 5️⃣), evaluated in the exact chunked form (64-token
 * chunks, a triangular solve per chunk, fp32 state carried on chip between
 * chunks); results equal the token-by-token recurrence up to rounding.
 *
 *   q, k, v, o       qkv_dtype device buffers (layouts above)
 *   log_alpha, beta  fp32 device buffers
 *   S0, S_final      fp32 [N, H, dk, dv] or NULL; S0 and S_final may alias
 *   cu_seqlens       int32 device buffer [n_seqs + 1] or NULL (then n_seqs is ignored)
 *   scale            read-out scale (commonly dk^-0.5)
 *   workspace        >= kda_chunk_fwd_workspace_size(...) bytes of device memory
 *   stream           cudaStream_t or NULL
 * T = 0 is allowed and only copies S0 to S_final (zeros without S0).
 */
kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                           const float *log_alpha, const float *beta, const float *S0,
                           const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                           int dk, int dv, float scale, void *o, float *S_final,
                           void *workspace, size_t workspace_bytes, void *stream);

/* kda_chunk_fwd with an explicit algorithm choice (kda_algo_t). Asking for
 * KDA_ALGO_TCGEN05 on a problem it does not support returns KDA_ERR_UNSUPPORTED.
 * On the tensor-core path (AUTO and TCGEN05) the sequential phase is split in
 * time when a problem has so few (sequence, head) chains that most SMs would
 * idle (see kda_chunk_fwd_timesplit); KDA_ALGO_TCGEN05_SEQUENTIAL never splits. */
kda_status_t kda_chunk_fwd_ex(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                              const float *log_alpha, const float *beta, const float *S0,
                              const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                              int dk, int dv, float scale, void *o, float *S_final,
                              void *workspace, size_t workspace_bytes, int algo,
                              void *stream);

/*
 * Chunked prefill on the tensor-core path (bf16, dk = dv = 128) with the
 * sequential phase split into `segments` time segments per sequence, so that
 * a long sequence with few heads keeps more SMs busy. The
 * sequential chunk walk of one (sequence, head) only runs on as many SMs as
 * there are 64-column halves of its state; the split runs it in two parallel
 * passes instead. Pass 1: segment 0 from S0 with outputs, and for every later
 * segment the state from a zero start and the segment's transition (the
 * product of the chunk steps' linear parts, a 128 x 128 matrix carried like a
 * state that starts at the identity). A combine kernel then forms each
 * segment's true entry state in fp32 (end = transition x entry + zero-start
 * state). Pass 2: every later segment again from its entry state, with
 * outputs. Results equal kda_chunk_fwd_ex's up to rounding. The recurrence is
 * the one of the "Kimi Linear" juejin.cn page, section 三 5️⃣; the pages give no
 * time split (the chunk-parallel form is section 三 2️⃣'s remark).
 *   segments   0: choose automatically (as KDA_ALGO_TCGEN05), 1: no split,
 *              2..64: that many segments per sequence (sequences with fewer
 *              chunks get empty segments)
 * Other arguments, layouts and errors as kda_chunk_fwd_ex; the workspace is
 * kda_chunk_fwd_timesplit_workspace_size bytes (it grows by 192 KB per segment,
 * sequence and head). Unsupported problems return KDA_ERR_UNSUPPORTED.
 */
size_t kda_chunk_fwd_timesplit_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs,
                                              kda_dtype_t qkv_dtype, int segments);
kda_status_t kda_chunk_fwd_timesplit(const void *q, const void *k, const void *v,
                                     kda_dtype_t qkv_dtype, const float *log_alpha,
                                     const float *beta, const float *S0,
                                     const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                                     int dk, int dv, float scale, void *o, float *S_final,
                                     void *workspace, size_t workspace_bytes, int segments,
                                     void *stream);

/*
 * The two phases of kda_chunk_fwd_ex, exported separately (same arguments, same
 * workspace). kda_chunk_fwd_ex(...) is exactly kda_chunk_fwd_prepare(...)
 * followed by kda_chunk_fwd_carry(...) on the same stream.
 *   prepare: the chunk-parallel phase. Plans the sequences and, for every
 *            64-token chunk and head, forms the gate cumulative sums, the
 *            intra-chunk matrices and the triangular solve, storing the chunk's
 *            intermediates in the workspace. Reads q, k, v, log_alpha, beta.
 *   carry:   the sequential phase. Walks each sequence's chunks in order with
 *            the fp32 state on chip, writing o and S_final. Reads the workspace,
 *            S0 and cu_seqlens-derived plan; does not read q, k, v or the gates.
 * Useful to time the phases or to run the chunk-parallel phase ahead of time.
 */
kda_status_t kda_chunk_fwd_prepare(const void *q, const void *k, const void *v,
                                   kda_dtype_t qkv_dtype, const float *log_alpha,
                                   const float *beta, const float *S0,
                                   const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                                   int dk, int dv, float scale, void *o, float *S_final,
                                   void *workspace, size_t workspace_bytes, int algo,
                                   void *stream);
kda_status_t kda_chunk_fwd_carry(const void *q, const void *k, const void *v,
                                 kda_dtype_t qkv_dtype, const float *log_alpha,
                                 const float *beta, const float *S0,
                                 const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                                 int dk, int dv, float scale, void *o, float *S_final,
                                 void *workspace, size_t workspace_bytes, int algo,
                                 void *stream);

/*
 * Recurrent decode: one new token for each of N independent sequences. Applies
 * the update rule once per (sequence, head) to the state S in place and writes
 * o = scale * S_new^T q. Source: the same update rule; the kernel evaluates it
 * in one pass over S using o = scale * (S'^T q + (k^T q) u) with
 * S' = Diag(alpha) S and u = beta (v - S'^T k), so S is read once and written
 * once.
 *
 *   q, k        qkv_dtype [N, H, dk]      v, o   qkv_dtype [N, H, dv]
 *   log_alpha   fp32 [N, H, dk]           beta   fp32 [N, H]
 *   S           fp32 [N, H, dk, dv], read and overwritten
 */
kda_status_t kda_decode_step(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                             const float *log_alpha, const float *beta, float *S, int N,
                             int H, int dk, int dv, float scale, void *o, void *stream);

/*
 * Multi-token decode: T new tokens for each of N independent sequences, applied
 * in order with the state held on chip between them; S is read once and
 * written once per call. Source: the same update rule, applied T times (each
 * token as in kda_decode_step). Equals T chained kda_decode_step calls, and
 * kda_chunk_fwd with B = N, S0 = S_final = S (up to rounding); meant for small
 * T (speculative verification, continuing a prefill by a few tokens), where the
 * chunked prefill would spend most of its time on per-chunk intermediates.
 *
 *   q, k        qkv_dtype [N, T, H, dk]   v, o   qkv_dtype [N, T, H, dv]
 *   log_alpha   fp32 [N, T, H, dk]        beta   fp32 [N, T, H]
 *   S           fp32 [N, H, dk, dv], read and overwritten
 * Errors as kda_decode_step; T = 0 returns KDA_OK without touching anything
 * (only S must then be non-null). N * T must fit in a signed 32-bit int.
 */
kda_status_t kda_decode_tokens(const void *q, const void *k, const void *v,
                               kda_dtype_t qkv_dtype, const float *log_alpha,
                               const float *beta, float *S, int N, int T, int H, int dk,
                               int dv, float scale, void *o, void *stream);

/*
 * Gated DeltaNet (GDN) variants: the same update rule with one forget rate per
 * token and head instead of one per channel, i.e. Diag(alpha_t) = alpha_t I.
 * Source: "Kimi Linear：让长上下文大模型真正实用的线性注意力架构" (juejin.cn),
 * section 三 1️⃣ (GDN has a single forget rate per head; KDA refines it per
 * channel) with the rule of section 三 5️⃣. Results equal the KDA entry points
 * given log_alpha broadcast over the dk channels.
 *
 * kda_gdn_chunk_fwd: arguments, layouts, workspace (kda_chunk_fwd_workspace_size_ex
 * with the same algo), errors and paths as kda_chunk_fwd_ex, except
 *   log_alpha   fp32 [B, T, H]  (one log forget rate per token and head, <= 0)
 * On the tensor-core path (bf16, dk = dv = 128) the scalar decay comes out of
 * the channel contraction, so its chunk-parallel phase is a lighter kernel than
 * the per-channel one; the sequential phase is shared.
 *
 * kda_gdn_chunk_fwd_prepare: its chunk-parallel phase alone; the sequential
 * phase, which reads only the workspace, S0 and the plan, is kda_chunk_fwd_carry
 * with the same arguments.
 *
 * kda_gdn_decode_tokens: as kda_decode_tokens, except
 *   log_alpha   fp32 [N, T, H]
 */
kda_status_t kda_gdn_chunk_fwd(const void *q, const void *k, const void *v,
                               kda_dtype_t qkv_dtype, const float *log_alpha,
                               const float *beta, const float *S0, const int32_t *cu_seqlens,
                               int n_seqs, int B, int T, int H, int dk, int dv, float scale,
                               void *o, float *S_final, void *workspace,
                               size_t workspace_bytes, int algo, void *stream);
kda_status_t kda_gdn_chunk_fwd_prepare(const void *q, const void *k, const void *v,
                                       kda_dtype_t qkv_dtype, const float *log_alpha,
                                       const float *beta, const float *S0,
                                       const int32_t *cu_seqlens, int n_seqs, int B, int T,
                                       int H, int dk, int dv, float scale, void *o,
                                       float *S_final, void *workspace, size_t workspace_bytes,
                                       int algo, void *stream);
kda_status_t kda_gdn_decode_tokens(const void *q, const void *k, const void *v,
                                   kda_dtype_t qkv_dtype, const float *log_alpha,
                                   const float *beta, float *S, int N, int T, int H, int dk,
                                   int dv, float scale, void *o, void *stream);

/*
 * Backward of the prefill (for training; the pages state only the forward rule,
 * so this is the rule's derivative): the gradients of
 *     L = <dO, o> + <dS_final, S_final>
 * with respect to q, k, v, log_alpha, beta and S0, for the arguments of
 * kda_chunk_fwd (same layouts, sequences and scale). Computed in fp32 on CUDA
 * cores for every supported head size, by the chunk-parallel form below
 * (KDA_BWD_AUTO; results are deterministic). The token walk (KDA_BWD_TOKEN,
 * through kda_chunk_bwd_ex) replays the states from checkpoints kept every 32
 * tokens and adds per-slice partial gradients (dk / 32 slices of 32 value
 * columns) in a fixed order; at d = 128 its workspace is about 8.2 KB per
 * token and head plus 2.2 MB per (sequence, head), e.g. 2.2 GB for B = 1,
 * H = 32, T = 8192.
 *   dO              qkv_dtype [B, T, H, dv]
 *   dS_final        fp32 [N, H, dk, dv] or NULL (zero)
 *   grad_q, grad_k  fp32 [B, T, H, dk]       grad_v     fp32 [B, T, H, dv]
 *   grad_log_alpha  fp32 [B, T, H, dk]       grad_beta  fp32 [B, T, H]
 *   grad_S0         fp32 [N, H, dk, dv] or NULL (not returned)
 * Workspace: kda_chunk_bwd_workspace_size bytes (that of KDA_BWD_AUTO). Errors as
 * kda_chunk_fwd_ex.
 * Tokens outside every sequence (cu_seqlens ending before B*T) are not written.
 * kda_gdn_chunk_bwd: the same for one gate per token and head (log_alpha and
 * grad_log_alpha fp32 [B, T, H]).
 */
size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int n_seqs,
                                    kda_dtype_t qkv_dtype);
/*
 * Backward algorithms. KDA_BWD_TOKEN walks every sequence token by token (the
 * states replayed from checkpoints). KDA_BWD_CHUNKED goes through the chunked
 * form of the rule (what kda_chunk_bwd and kda_gdn_chunk_bwd run, and
 * KDA_BWD_AUTO): per-chunk records (W, U~, e^g q, e^{g_C - g} k, P, e^{g_C}), a forward
 * and a reverse walk over the chunks (one CTA per sequence, head and 32 value
 * columns), then the token gradients of all chunks in parallel; fp32 CUDA-core
 * arithmetic where every exponential is of a non-positive number, so any gate
 * is safe. Its workspace holds, per (chunk, head) at d = 128, the record
 * (148 KB), the entry state and chunk-end gradient (64 KB each), U and dU
 * (32 KB each) and the token-gradient products (115 KB): about 7.1 KB per
 * token and head.
 */
enum { KDA_BWD_AUTO = 0, KDA_BWD_TOKEN = 1, KDA_BWD_CHUNKED = 2 };
/* Workspace bytes for a backward algorithm (0 on invalid sizes or algo). */
size_t kda_chunk_bwd_workspace_size_ex(int B, int T, int H, int dk, int dv, int n_seqs,
                                       kda_dtype_t qkv_dtype, int algo);
/* kda_chunk_bwd (gate_per_channel 1) or kda_gdn_chunk_bwd (0) with an explicit
 * algorithm; the workspace is kda_chunk_bwd_workspace_size_ex(..., algo) bytes.
 * An unknown algo returns KDA_ERR_INVALID_ARG before any device work. */
kda_status_t kda_chunk_bwd_ex(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                              const float *log_alpha, const float *beta, const float *S0,
                              const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                              int dk, int dv, float scale, const void *dO,
                              const float *dS_final, float *grad_q, float *grad_k,
                              float *grad_v, float *grad_log_alpha, float *grad_beta,
                              float *grad_S0, void *workspace, size_t workspace_bytes,
                              int gate_per_channel, int algo, void *stream);
kda_status_t kda_chunk_bwd(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                           const float *log_alpha, const float *beta, const float *S0,
                           const int32_t *cu_seqlens, int n_seqs, int B, int T, int H, int dk,
                           int dv, float scale, const void *dO, const float *dS_final,
                           float *grad_q, float *grad_k, float *grad_v, float *grad_log_alpha,
                           float *grad_beta, float *grad_S0, void *workspace,
                           size_t workspace_bytes, void *stream);
kda_status_t kda_gdn_chunk_bwd(const void *q, const void *k, const void *v,
                               kda_dtype_t qkv_dtype, const float *log_alpha,
                               const float *beta, const float *S0, const int32_t *cu_seqlens,
                               int n_seqs, int B, int T, int H, int dk, int dv, float scale,
                               const void *dO, const float *dS_final, float *grad_q,
                               float *grad_k, float *grad_v, float *grad_log_alpha,
                               float *grad_beta, float *grad_S0, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * kda_chunk_fwd_noalloc — the chunked prefill for callers that cannot allocate
 * device memory (no counterpart in the paper; it exists for callers such as a
 * plugin whose host application owns all device memory, or code that must not
 * trigger the device synchronisation an allocation can cause).
 *
 * Same arguments and results as kda_chunk_fwd_ex, minus the workspace: the
 * library uses a fixed scratch array of KDA_NOALLOC_SCRATCH_BYTES in its own
 * device memory, held by every GPU that loads the library until the process
 * exits. The caller still provides every input and output buffer. The call
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library call).
 *   - Problems whose workspace for the same algo
 *     (kda_chunk_fwd_workspace_size_ex with this call's algo) exceeds
 *     KDA_NOALLOC_SCRATCH_BYTES are rejected on the host with
 *     KDA_ERR_WORKSPACE before anything is launched; invalid arguments are
 *     rejected on the host as kda_chunk_fwd_ex rejects them.
 *   - The first call on each device (and the first after the device's
 *     context was reset) looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture on the device.
 *   - With KDA_DEBUG_SYNC=1 in the environment the call waits for its work
 *     and reports a bounded wait that ran out as KDA_ERR_DEVICE_STATUS, as
 *     kda_chunk_fwd_ex does.
 *   - Every call shares the one array and leaves its contents behind. The
 *     kernels initialise every part of it they read, so nothing carries over
 *     from one call to the next; but calls whose execution overlaps on the GPU
 *     (different streams, or different host threads) race on the array and
 *     must be serialised by the caller.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                   kda_dtype_t qkv_dtype, const float *log_alpha,
                                   const float *beta, const float *S0,
                                   const int32_t *cu_seqlens, int n_seqs, int B, int T, int H,
                                   int dk, int dv, float scale, void *o, float *S_final,
                                   int algo, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H */
