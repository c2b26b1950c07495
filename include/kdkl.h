/*
 * kdkl — fused, chunked KL distillation loss of a student output head against
 * an offline teacher top-K cache, for one NVIDIA B200 (sm_100a).
 *
 * Method: "Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and
 * a Fused Chunked KL Loss".  The teacher is run once and only its top-K
 * (vocabulary index, logit) pairs per token are kept (mind-verse.de article,
 * section "Zwei systemische Optimierungen", item 1; llm-wiki note, section
 * "사전 계산 파이프라인", step 3).  The loss folds the student's output
 * projection into the KL computation and never holds the full
 * [tokens x vocabulary] logit matrix; the backward recomputes each chunk's
 * projection (mind-verse.de article, three-variant list, "Fused chunked KL").
 * kdkl_forward_backward computes the same outputs in one call, keeping each
 * chunk's logits for that chunk's gradient instead of recomputing them.
 *
 * Definitions (N tokens, hidden size d, vocabulary V, K cached entries, tau):
 *   z[n, v]   = sum_j hidden[n, j] * W[v, j]              (student logits)
 *   lse[n]    = log sum_v exp(z[n, v])
 *   P_T[n, .] = softmax(topk_logit[n, .] / tau) over the row's in-range entries,
 *               zero on every other vocabulary entry
 *   KL_n      = sum_v P_T(v) (log P_T(v) - (z[n, v] - lse[n]))
 *               (llm-wiki note, section "표준 KD의 손실 함수")
 *   loss      = sum_n m_n KL_n / N_valid,  m_n = mask[n] and the row is usable,
 *               N_valid = sum_n m_n  (loss = 0 when N_valid = 0)
 *   G[n, v]   = m_n (g / N_valid) (exp(z[n, v] - lse[n]) - P_T[n](v))
 *   dHidden   = G W   [N, d],   dW = G^T hidden   [V, d]
 * tau divides the teacher logits only (there is no tau^2 factor).
 *
 * Conventions for every entry point below:
 *   - All tensors are dense, row-major, on the current CUDA device, and owned
 *     by the caller.  The library never allocates device memory: scratch comes
 *     from the caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream).  Nothing synchronises except
 *     kdkl_read_device_flags.  No state is kept between calls.  After one
 *     eager call on a device, kdkl_forward(_ex), kdkl_backward(_ex) and
 *     kdkl_forward_backward can be captured in a CUDA graph (every launch and
 *     memset goes to `stream`); a replay reads the buffers' current contents.
 *   - Argument checks run on the host before any launch; a failed check
 *     returns its status and launches nothing.  kdkl_last_error() then holds a
 *     one-line reason.
 *   - Data errors found on the device (cache index outside [0, V), repeated
 *     index, non-finite teacher logit, an internal wait that timed out) never
 *     trap: they set bits of a device flag word kept in the workspace, which
 *     the caller reads with kdkl_read_device_flags.  Entries with an index
 *     outside [0, V) are dropped; repeated indices add up; a row with a NaN or
 *     +inf logit, or with no usable entry, is treated as masked.
 *   - Schedule tuning (not needed for normal use): the environment variables
 *     KDKL_SYNC_WINDOW, KDKL_SYNC_KWINDOW, KDKL_SPLIT_GROUP_MB,
 *     KDKL_TILE_COL_GROUP, KDKL_DIE_ORDER and KDKL_L2_HINTS, read once per
 *     process, change only the order in which the GEMMs' CTA groups take their
 *     tiles, how closely they are kept together and the L2 priority of their
 *     loads; every output is bit-identical under any of them.
 *     KDKL_ROWS_BUDGET_MB changes the forward's vocabulary split count, and so
 *     the order of each row's log-sum-exp merge (rounding only).
 */
#ifndef KDKL_H
#define KDKL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDKL_OK = 0,
  KDKL_ERR_NULL = 1,        /* a required pointer is NULL */
  KDKL_ERR_SHAPE = 2,       /* N < 0, d % 8 != 0, K outside [1, 256], K > V, tau not finite > 0, ... */
  KDKL_ERR_ALIGN = 3,       /* a pointer breaks its alignment rule (listed per argument) */
  KDKL_ERR_UNSUPPORTED = 4, /* no sm_100 device current, or a size beyond the library's limits */
  KDKL_ERR_WORKSPACE = 5,   /* workspace smaller than kdkl_workspace_bytes() */
  KDKL_ERR_CUDA = 6         /* a CUDA runtime call or launch failed */
} kdkl_status;

/* Bits of the device flag word (kdkl_read_device_flags). */
enum {
  KDKL_DEV_IDX_RANGE = 1u, /* some cached index was outside [0, V); the entry was dropped */
  KDKL_DEV_IDX_DUP = 2u,   /* some row repeated a cached index; the probabilities were added */
  KDKL_DEV_NONFINITE = 4u, /* some row had a NaN/+inf (or only -inf) logit; the row was masked */
  KDKL_DEV_TIMEOUT = 8u,   /* an internal pipeline wait gave up (after 2 s): the kernel stopped early,
                              so this call's outputs, and those of every later call on the stream
                              that read them, are invalid */
  KDKL_DEV_BOUNDS = 16u    /* bounds-checking build (libkdkl_debug.so) only: an index check in a
                              kernel failed and the access was skipped; outputs are invalid */
};

/*
 * Bytes of scratch that kdkl_forward / kdkl_backward need for these sizes.
 * The amount is linear in N plus one N-independent chunk buffer of
 * chunk_tokens x V bf16 values (the backward's per-chunk logit gradient); it
 * never holds an N x V buffer.  chunk_tokens = 0 sizes that buffer for the
 * library's default capacity, min(N rounded up to 128, 8192) tokens, within
 * which the backward's planner picks its chunk (kdkl_backward_plan); other
 * values are rounded up to a multiple of 128 and used as given.  Returns 0 for
 * sizes that the entry points would reject.
 */
size_t kdkl_workspace_bytes(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens);

/*
 * Forward: loss and per-token log-sum-exp.
 *   hidden      [N, d] bf16, 16-byte aligned (student last hidden states)
 *   W           [V, d] bf16, 16-byte aligned (output-head weight, nn.Linear layout, no bias)
 *   topk_idx    [N, K] int32, 4-byte aligned (teacher cache: vocabulary indices)
 *   topk_logit  [N, K] fp32, 4-byte aligned (teacher cache: logits)
 *   mask        [N] uint8 (0 = token excluded, e.g. a packed-sequence boundary)
 *   N >= 0, d % 8 == 0 (d >= 8), 1 <= K <= 256, K <= V, tau finite and > 0
 *   loss        [1] fp32 out (device), 4-byte aligned
 *   lse         [N] fp32 out (device), 4-byte aligned; written for every row, masked ones too
 *   workspace   >= kdkl_workspace_bytes(N, d, V, K, c) bytes for any chunk size c (the
 *               forward does not touch the backward's chunk buffer), 256-byte aligned
 * N = 0 writes loss = 0 and nothing else.
 */
kdkl_status kdkl_forward(const void* hidden, const void* W, const int32_t* topk_idx,
                         const float* topk_logit, const uint8_t* mask, int64_t N, int32_t d,
                         int32_t V, int32_t K, float tau, float* loss, float* lse,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward: dHidden and dW of g * loss, recomputing each chunk's projection.
 *   inputs as kdkl_forward, plus
 *   lse          [N] fp32 in: the lse written by kdkl_forward on the same inputs
 *   grad_loss    [1] fp32 in (device) = g, or NULL for g = 1
 *   dHidden      [N, d] bf16 out, 16-byte aligned (fp32 accumulation, rounded once);
 *                rows that do not count (masked or unusable) are written as 0
 *   dW           [V, d] fp32 out, 16-byte aligned, overwritten (not accumulated into)
 *   chunk_tokens tokens per backward chunk (0 = default); bounds the chunk buffer
 *   workspace    >= kdkl_workspace_bytes(N, d, V, K, chunk_tokens) bytes, 256-byte aligned
 * N = 0 writes dW = 0 and nothing else.
 */
kdkl_status kdkl_backward(const void* hidden, const void* W, const int32_t* topk_idx,
                          const float* topk_logit, const uint8_t* mask, int64_t N, int32_t d,
                          int32_t V, int32_t K, float tau, const float* lse,
                          const float* grad_loss, void* dHidden, float* dW,
                          int64_t chunk_tokens, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Forward for callers that cannot allocate device memory.  (The paper has no
 * counterpart of this entry point; it is an interface addition.)
 *
 * Some callers cannot hand kdkl a workspace: a loss hook whose host framework
 * passes only inputs and outputs, a runtime that plans every device byte up
 * front and forbids later allocations, or a hot loop that must not call
 * cudaMalloc because an allocation may synchronise the device.  This entry
 * point takes the same inputs and outputs as kdkl_forward, and the same
 * results, but no workspace: its scratch is a 32 MiB array built into the
 * library, which every GPU that loads the library keeps until the process
 * exits.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Sizes whose forward scratch exceeds 32 MiB are rejected with
 *     KDKL_ERR_UNSUPPORTED before any launch: the scratch takes a fixed 6.3 MB
 *     plus about 8 * K + 130 bytes per token, so up to about 29,000 tokens
 *     fit at K = 100.
 *   - The first call on each device looks up that device's copy of the array
 *     (cudaGetSymbolAddress) with the device current; make that first call
 *     before any stream capture.  The lookup is kept per device and CUDA
 *     context: after cudaDeviceReset the next call looks the array up again.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind.  Each call clears what must start at zero, so leftovers do not
 *     matter, but two calls that overlap on the GPU (other streams, other host
 *     threads) race on the array and corrupt each other's results.
 *   - The device flag word lives in that array too, so kdkl_read_device_flags
 *     cannot read it; use kdkl_forward to see data-error flags.
 */
kdkl_status kdkl_forward_noalloc(const void* hidden, const void* W, const int32_t* topk_idx,
                                 const float* topk_logit, const uint8_t* mask, int64_t N, int32_t d,
                                 int32_t V, int32_t K, float tau, float* loss, float* lse, void* stream);

/*
 * Options of the extended entry points (kdkl_forward_ex / kdkl_backward_ex).
 * kdkl_options_init fills the defaults, under which the extended entry points
 * compute exactly what kdkl_forward / kdkl_backward compute.
 *
 * Cache format (the llm-wiki note, section "사전 계산 파이프라인", recommends
 * 16-bit indices and bf16 values, 4 bytes per cached entry):
 *   KDKL_CACHE_I32_F32  topk_idx int32, topk_logit fp32 (4-byte aligned)
 *   KDKL_CACHE_U16_BF16 topk_idx uint16, topk_logit bf16 (2-byte aligned); needs V <= 65536
 *
 * Loss-design variants (the paper reports ablations on loss design; these are
 * the standard knowledge-distillation forms, one shared student softmax):
 *   P_S = softmax(z / student_tau)
 *   per valid row: gamma * KL(P_T || P_S) + ce_weight * (-log P_S(label))
 *   gamma = kd_weight * (student_tau^2 if kd_scale_tau_sq else 1)
 *   labels[n] outside [0, V) (e.g. -100) add no hard-label term for row n.
 * The loss is still normalised by N_valid; lse is then the log-sum-exp of
 * z / student_tau, and kdkl_backward_ex must get the same options as the
 * forward that produced it.
 */
typedef enum { KDKL_CACHE_I32_F32 = 0, KDKL_CACHE_U16_BF16 = 1 } kdkl_cache_format;

typedef struct {
  int32_t cache_format;     /* kdkl_cache_format */
  float student_tau;        /* finite, > 0 (default 1) */
  float kd_weight;          /* finite, >= 0 (default 1) */
  int32_t kd_scale_tau_sq;  /* nonzero: multiply the KL term by student_tau^2 (default 0) */
  float ce_weight;          /* finite, >= 0 (default 0: no hard-label term) */
  const int32_t* labels;    /* [N] int32 device, 4-byte aligned; required when ce_weight > 0 */
  /* Data-parallel normaliser: a device count to divide the loss and the
   * gradients by instead of this call's own N_valid (the sum over ranks of each
   * rank's kdkl_count_valid count, after an all-reduce).  NULL = this call's own
   * count (default).  Forward and backward must get the same count. */
  const uint32_t* n_valid_global;
  /* N tile width of the backward's dHidden and dW GEMMs (their N axis is d):
   * 0 = the planner's choice (default; see kdkl_backward_plan), else one of
   * 128, 160, 192, 224, 240, 256.  It changes how the output is partitioned
   * into tiles, not the arithmetic: each output element is accumulated over
   * the same 64-wide reduction blocks in the same order. */
  int32_t bwd_tile_n;
} kdkl_options;

void kdkl_options_init(kdkl_options* options);

/* Device address of the N_valid count that the last kdkl_count_valid, forward or
 * backward call on this workspace computed: this call's own rows, even when
 * options->n_valid_global was given (uint32, stream-ordered after that call; no CUDA
 * call is made; NULL when workspace is NULL). */
const uint32_t* kdkl_n_valid_device(const void* workspace);

/*
 * Count of the rows that enter the loss, without the projection: runs the
 * forward's per-row preparation of the teacher cache (the mask, dropped and
 * non-finite entries; see the data-error rules above) and leaves the count at
 * kdkl_n_valid_device(workspace) and the data-error flags in the flag word.
 * It exists for data parallelism (the paper's training runs shard tokens across
 * GPUs): each rank counts its own shard, the counts are summed across ranks on
 * the device (an all-reduce), and the sum is passed as options->n_valid_global
 * to kdkl_forward_ex and kdkl_backward_ex.  Each rank's loss is then its rows'
 * share of the global loss (the sum over ranks is the global loss), its dHidden
 * is final, and its dW is its term of the global dW.
 *   topk_idx, topk_logit, mask, N, V, K, tau, options: as kdkl_forward_ex
 *   workspace >= kdkl_workspace_bytes(N, d, V, K, c) for any d and c, 256-byte
 *     aligned; the same workspace may then be passed to the forward and backward
 * N = 0 leaves a count of 0.
 */
kdkl_status kdkl_count_valid(const void* topk_idx, const void* topk_logit, const uint8_t* mask, int64_t N,
                             int32_t V, int32_t K, float tau, const kdkl_options* options, void* workspace,
                             size_t workspace_bytes, void* stream);

/* kdkl_forward with options (NULL = defaults); topk_idx / topk_logit typed by options->cache_format. */
kdkl_status kdkl_forward_ex(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                            const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                            const kdkl_options* options, float* loss, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * The backward's work plan, computed on the host without any CUDA work: the N
 * tile width of the dHidden and dW GEMMs and the tokens per chunk that
 * kdkl_backward / kdkl_backward_ex use for these arguments on a device with
 * `sm_count` SMs (0 = ask the current device).  An explicit chunk_tokens is
 * used as given (rounded up to a multiple of 128, at most N rounded up); with
 * chunk_tokens = 0 the chunk is chosen at or below the workspace's default
 * chunk capacity (8192 tokens).  The planner minimises a wave-count cost model
 * of the two GEMMs: the dHidden GEMM has only (chunk / 256) x ceil(d / tile_n)
 * output tiles, each reducing over the whole vocabulary, so a partly filled
 * last wave of tiles idles most of the GPU for a long time.
 * Errors: KDKL_ERR_NULL (an output pointer is NULL), KDKL_ERR_SHAPE,
 * KDKL_ERR_UNSUPPORTED (bad options or no device when sm_count = 0).
 */
kdkl_status kdkl_backward_plan(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens,
                               const kdkl_options* options, int32_t sm_count, int32_t* tile_n_out,
                               int64_t* chunk_tokens_out);

/* kdkl_backward with options (NULL = defaults); must match the forward's options. */
kdkl_status kdkl_backward_ex(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                             const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                             const kdkl_options* options, const float* lse, const float* grad_loss,
                             void* dHidden, float* dW, int64_t chunk_tokens, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Fused forward + backward, without the backward's logit recompute.  The pages'
 * fused chunked loss recomputes each chunk's logits in the backward, so the
 * projection runs twice and nothing N x V is ever stored (mind-verse.de
 * article, section "Zwei systemische Optimierungen", the "Fused chunked KL"
 * item).  This entry point computes each token chunk's logits once: one GEMM
 * folds them into the online log-sum-exp and gather and also stores them (fp32)
 * in a chunk buffer; once the chunk's rows have their lse, G is formed from the
 * stored logits, and the chunk's dHidden and dW GEMMs run.  The chunk buffer is
 * N-independent, so peak memory still grows only linearly with N, and the step
 * does 6 N d V flops instead of 8 N d V.
 * It computes what kdkl_forward_ex followed by kdkl_backward_ex compute with the
 * same options: loss, lse, dHidden and dW (grad_loss, a device scalar or NULL = 1,
 * must be known at call time).  Results agree with the separate calls up to
 * rounding order: each row's log-sum-exp is merged from a different number of
 * vocabulary splits.
 *   workspace >= kdkl_forward_backward_workspace_bytes(N, d, V, K, chunk_tokens):
 *     the loss workspace plus chunk x V fp32 logits (4.2 GB at 8192 x 128,256)
 *   chunk_tokens is rounded up to a multiple of 256; 0 = the backward planner's
 *     choice within the default capacity (kdkl_backward_plan reports it)
 *   argument checks and errors as kdkl_forward_ex and kdkl_backward_ex; loss must
 *     be non-NULL and 4-byte aligned
 */
size_t kdkl_forward_backward_workspace_bytes(int64_t N, int32_t d, int32_t V, int32_t K, int64_t chunk_tokens);
kdkl_status kdkl_forward_backward(const void* hidden, const void* W, const void* topk_idx, const void* topk_logit,
                                  const uint8_t* mask, int64_t N, int32_t d, int32_t V, int32_t K, float tau,
                                  const kdkl_options* options, const float* grad_loss, float* loss, float* lse,
                                  void* dHidden, float* dW, int64_t chunk_tokens, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * Teacher top-K cache producer: the step that builds the cache the loss reads.
 * The teacher runs once and, for each token position, only its K most likely
 * vocabulary entries are kept as (index, logit) pairs (mind-verse.de article,
 * section "Zwei systemische Optimierungen", item 1; llm-wiki note, section
 * "사전 계산 파이프라인", steps 2-3).  Given the teacher's last hidden states and
 * output head, this computes z = hidden W^T tile by tile on the tensor cores
 * (never storing z) and keeps each row's K largest logits:
 *   hidden      [N, d] bf16, 16-byte aligned; W [V, d] bf16, 16-byte aligned
 *   1 <= K <= 128, K <= V <= 65,280 * floor(1024 / K) (522,240 at K = 128), d % 8 == 0
 *   topk_idx    [N, K] int32 out; topk_logit [N, K] fp32 out (the fp32 logits z)
 *   each row ordered by logit descending, ties to the smaller index
 *   workspace   >= kdkl_teacher_topk_workspace_bytes(N, d, V, K), 256-byte aligned
 * The output is directly a KDKL_CACHE_I32_F32 cache for kdkl_forward.
 */
size_t kdkl_teacher_topk_workspace_bytes(int64_t N, int32_t d, int32_t V, int32_t K);
kdkl_status kdkl_teacher_topk(const void* hidden, const void* W, int64_t N, int32_t d, int32_t V, int32_t K,
                              int32_t* topk_idx, float* topk_logit, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Reads the device flag word of the most recent forward/backward call that
 * used `workspace` (each call clears it first).  Synchronises `stream`.
 */
kdkl_status kdkl_read_device_flags(const void* workspace, void* stream, uint32_t* flags_out);

/*
 * Optional per-kernel timing (tracing aid; off by default).  While enabled,
 * every kernel the library launches is bracketed by a pair of CUDA events
 * recorded on the caller's stream, tagged with the kernel's name.
 * kdkl_timing_read waits for the pending events, adds their durations into
 * per-kernel totals, copies up to max_entries totals into `out` (names are
 * static strings) and returns how many kernel kinds exist; reset != 0 clears
 * the totals afterwards.  Enabling costs two event records per launch.
 */
typedef struct {
  const char* name;   /* "prepass", "fwd_lse_gemm", "merge", "bwd_grad_gemm", "bwd_dhidden_gemm", "bwd_dw_gemm",
                         "teacher_topk_gemm", "teacher_topk_merge" */
  uint64_t launches;  /* launches timed since the last reset */
  double total_ms;    /* summed device time of those launches */
} kdkl_kernel_time;

kdkl_status kdkl_timing_enable(int enable);
int kdkl_timing_read(kdkl_kernel_time* out, int max_entries, int reset);

/*
 * Self-test of the kernels' bounded waits (failure detection without a GPU
 * fault).  Every wait inside the kernels gives up after a time limit, sets
 * KDKL_DEV_TIMEOUT in the workspace's flag word and lets the kernel return, so
 * the context stays usable.  This launches one thread that waits, through the
 * same wait routine, on a barrier that nothing completes, with a limit of
 * limit_ns (1 us .. 1 s); afterwards kdkl_read_device_flags reports
 * KDKL_DEV_TIMEOUT and workspace bytes [8, 16) hold the waited time (uint64 ns).
 * workspace: >= 256 bytes, 256-byte aligned.
 */
kdkl_status kdkl_selftest_wait_timeout(void* workspace, uint64_t limit_ns, void* stream);

/* Static name of a status code. */
const char* kdkl_status_string(kdkl_status status);

/* One-line reason for the last non-OK status returned on this host thread ("" if none). */
const char* kdkl_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KDKL_H */
