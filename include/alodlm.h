/*
 * alodlm.h — C ABI of the ALoDLM denoising-step library (libalodlm.so), sm_100a only.
 *
 * One denoising step of an adaptively looped masked diffusion LM ("ALoDLM: Adaptively
 * Looped Diffusion Language Models", paper digest page, sections "Core method",
 * "Method steps" (Algorithm 1) and Eq. 3).  The model is a Qwen3-style decoder cut into
 * a Prelude, a weight-shared Recurrent Core that is looped per token, and a Coda; after
 * each loop the Coda's readout r^(s) feeds an LM head (vocab distribution, entropy,
 * argmax) and an ExitGate (halting probability).  Confident positions commit their
 * argmax token, whose embedding re-enters the loop as discrete context (Eq. 3); the
 * others carry their latent state into the next loop, up to K.  A depth-aware KV cache
 * serves the prefix at the matching loop depth, falling back to the deepest depth the
 * position reached (section "Technical novelty").
 *
 * Conventions for every entry point:
 *   - Returns ALODLM_OK (0) or a negative ALODLM_E* code; nothing aborts or exits and no
 *     exception crosses the ABI.  alodlm_last_error() gives a one-line reason.
 *   - "device" pointers are CUDA device memory of the handle's device, "host" pointers
 *     are ordinary host memory.  The caller owns every buffer it passes in; the handle
 *     owns the packed weights, the KV arena and all scratch.
 *   - Work is enqueued on the handle's stream; calls return before the GPU finishes
 *     unless stated otherwise.  alodlm_sync() waits and reports device-side errors.
 *   - A handle is not thread-safe: one host thread at a time.
 */
#ifndef ALODLM_H
#define ALODLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define ALODLM_OK 0
#define ALODLM_EINVAL (-1)   /* bad argument: null pointer, size out of range, unsupported shape */
#define ALODLM_ENOMEM (-2)   /* device allocation failed or would pass cfg.mem_limit_bytes */
#define ALODLM_ECUDA (-3)    /* a CUDA runtime/driver call failed (text in last_error) */
#define ALODLM_EDEVICE (-4)  /* a kernel flagged an inconsistency (bounds, bad id) */
#define ALODLM_ETIMEOUT (-5) /* a bounded device-side wait gave up; the step's outputs are invalid */
#define ALODLM_ESTATE (-6)   /* call out of order (step before prefill, batch differs from prefill) */

/* commit rules: two readings of the halting threshold (a mean over the unresolved positions,
   as the paper states it, or each position's own cumulative halt) */
#define ALODLM_RULE_PAPER 0     /* commit H <= tau; stop when mean a over U >= lambda (the pages' q),
                                   or U empty, or s = K; if nothing committed in the step, commit
                                   the lowest-entropy position of the last loop */
#define ALODLM_RULE_PER_TOKEN 1 /* commit H <= tau or a_i >= lambda, and all of U at s = K */

/* storage type of weight matrices handed to alodlm_create */
#define ALODLM_DTYPE_BF16 0
#define ALODLM_DTYPE_F32 1

#if defined(__GNUC__)
#define ALODLM_API __attribute__((visibility("default")))
#else
#define ALODLM_API
#endif

typedef struct alodlm alodlm_t; /* opaque handle */

/* Model and capacity.  Supported: head_dim 64 or 128; hidden, n_q_heads*head_dim and inter
 * multiples of 16; n_q_heads a multiple of n_kv_heads; n_core >= 1 (n_prelude, n_coda >= 0);
 * 1 <= k_max <= 64; max_block <= 1024; max_batch <= 1024. */
typedef struct {
    int hidden, n_q_heads, n_kv_heads, head_dim, inter, vocab;
    int n_prelude, n_core, n_coda;
    int k_max;                          /* deepest loop the KV arena holds (prefill builds 1..k_max) */
    int max_batch, max_prefix, max_block;
    float rope_base;                    /* 1e6 for Qwen3 */
    float rms_eps;                      /* 1e-6 */
    int mask_id;                        /* [MASK] token id (vocab-1 in the synthetic configs) */
    int qk_norm;                        /* 1: per-head RMSNorm of q and k (Qwen3) */
    size_t mem_limit_bytes;             /* 0 = no limit; otherwise create fails with ENOMEM beyond it */
    int debug_dump;                     /* 1: keep per-loop copies of h^(s-1), h~^(s), r^(s) (parity checks) */
} alodlm_cfg;

/* One decoder layer: device pointers, row-major [out, in].  Matrices in weights.matrix_dtype,
 * gains always float32.  q [nq*hd, H], k/v [nkv*hd, H], o [H, nq*hd], gate/up [I, H],
 * down [H, I]; attn_norm/mlp_norm [H], q_norm/k_norm [hd]. */
typedef struct {
    const void *attn_norm, *q, *k, *v, *o, *q_norm, *k_norm, *mlp_norm, *gate, *up, *down;
} alodlm_layer_w;

typedef struct {
    int matrix_dtype;             /* ALODLM_DTYPE_BF16 or ALODLM_DTYPE_F32 (rounded to bf16, nearest-even) */
    const void *embed;            /* device [vocab, hidden], the input embedding Emb */
    const void *lm_head;          /* device [vocab, hidden] */
    const float *final_norm;      /* device [hidden] */
    const float *exit_w;          /* device [hidden], ExitGate weight */
    float exit_b;                 /* ExitGate bias */
    const alodlm_layer_w *layers; /* host array, n_prelude + n_core + n_coda entries in model order */
} alodlm_weights;

/* Outputs of one step, all caller-owned DEVICE buffers. K below is the step's k_max. */
typedef struct {
    int32_t *tokens;      /* [B,N] committed token, the given id at non-mask positions, mask_id if uncommitted */
    int32_t *exit_depth;  /* [B,N] loop s (1..K) at which the position committed, 0 if not */
    float *entropy;       /* [B,K,N] H_i^(s) in nats for i in U at loop s, NaN elsewhere */
    float *halt;          /* [B,K,N] lambda_i^(s), NaN elsewhere */
    float *cum_halt;      /* [B,K,N] a_i^(s) after the loop-s update, NaN elsewhere */
    int32_t *loops_run;   /* [B] loops the sequence ran in this step */
    int32_t *active_rows; /* [K] block rows run through Core/Coda at loop s (sequences still looping x N) */
    int32_t *readout_rows;/* [K] rows read out (|U| summed over looping sequences) at loop s */
} alodlm_step_out;

/* Create a handle on the current CUDA device.
 * [digest "Core method"]: Prelude = layers [0, n_prelude), Core = next n_core (weight-shared,
 * looped), Coda = last n_coda.  The weights are read during the call only (packed to bf16
 * into handle-owned memory: fused QKV, gate/up interleaved); the caller may free them after.
 * Allocates the depth-aware KV arena: (n_prelude + k_max*n_core + n_coda) slots of
 * max_batch x n_kv_heads x (max_prefix + max_block) x head_dim, K and V, bf16.
 * stream: a cudaStream_t (NULL = legacy default stream).
 * Errors: EINVAL (shape/null, or a KV arena of 2^31 head vectors or more, which the
 * attention's 32-bit tensor-map coordinates cannot address), ENOMEM, ECUDA.  On error *out is
 * NULL and the text is in alodlm_last_error(NULL). */
ALODLM_API int alodlm_create(const alodlm_cfg *cfg, const alodlm_weights *weights, void *stream, alodlm_t **out);

/* Build the depth-aware KV cache of the prefix.
 * [digest "Technical novelty", "Prerequisites"]: prefix position j with exit depth e_j runs
 * the Core e_j times; its Core KV at depth d > e_j is its depth-e_j KV (written at prefill
 * time, so a step reads one dense slot per depth); the Coda runs once on the depth-e_j state.
 * Prefix attention is causal; positions are 0..P-1.
 * Depth on demand (digest "Limitations": build the cache only as deep as needed and fill deeper
 * depths incrementally): at depth d only the positions with e_j >= d run the Core (rows
 * compacted), and no Core depth beyond max_j e_j is built -- a step at a deeper loop reads the
 * deepest built one, which holds every position's KV at that depth under the fallback rule.
 * prefix_ids: device int32 [B,P], ids in [0, vocab).  exit_depth: device int32 [B,P] in
 * 1..k_max, or NULL for k_max everywhere (read back to the host once).  1 <= B <= max_batch,
 * 1 <= P <= max_prefix.  Replaces any previous prefill.  Errors: EINVAL, ECUDA, EDEVICE (exit
 * depth out of range at once; id out of range on the next sync). */
ALODLM_API int alodlm_prefill(alodlm_t *h, const int32_t *prefix_ids, int B, int P, const int32_t *exit_depth);

/* Append N positions to every sequence's cached prefix: positions P..P+N-1 holding ids (a
 * decoded block), so that the next step's block sits at P+N.
 * [digest "Method steps", Algorithm 1 (5); "Technical novelty"]: committed tokens are written
 * into the sequence and later blocks attend to them; every position is served at its own loop
 * depth, the deepest it reached standing in for deeper ones.  The new positions go through
 * what alodlm_prefill does for prefix positions -- Prelude, the Core e_j times (Core KV at depth
 * d > e_j = the depth-e_j KV), the Coda once on the depth-e_j state -- attending to every
 * cached position (at its own slot) and causally to each other.  The result equals one
 * prefill of the longer prefix (prefix attention is causal).
 * ids: device int32 [B,N] in [0, vocab); B must equal the prefill's; 1 <= N <= max_block and
 * P + N <= max_prefix.  exit_depth: device int32 [B,N] in 1..k_max (e.g. a decoded block's
 * commit depths, with positions that held a given id or never committed set to k_max), or
 * NULL for k_max everywhere.  If a new position loops deeper than any cached one, the cached
 * positions' Core KV is first extended to that depth (copies of their deepest built depth).
 * Errors: EINVAL, ESTATE (before prefill, batch differs), ECUDA, EDEVICE (exit depth out of
 * range at once, id out of range on the next sync).  After an error the cached prefix is
 * invalid until the next prefill. */
ALODLM_API int alodlm_append(alodlm_t *h, const int32_t *ids, int B, int N, const int32_t *exit_depth);

/* One denoising step over a block of N positions per sequence (positions P..P+N-1).
 * [digest "Method steps", Algorithm 1 (1)-(5); Eq. 3]:
 *   U = mask positions; h^(0) = Prelude(Emb(block)); for s = 1..k_max:
 *   h~ = Core(h^(s-1)) against prefix Core KV at depth s; r = RMSNorm_f(Coda(h~));
 *   for i in U: H_i (entropy, nats), y_i (argmax, lowest id on ties), lambda_i =
 *   sigmoid(w.r_i + b), a_i += (1 - a_i) lambda_i; commit per `rule`; h^(s) = Emb(y) on
 *   committed rows, h~ elsewhere; stop per `rule`.  The block attends to the whole prefix
 *   and to itself (bidirectional).  Sequences that stop leave the batch (rows compacted);
 *   the readout runs on U rows only; logits never reach global memory.
 * block_ids: device int32 [B,N]; B must equal the prefill's B; 1 <= N <= max_block;
 * 1 <= k_max <= cfg.k_max; rule = ALODLM_RULE_*.  lambda is the halting threshold.
 * Asynchronous except for one 16-byte device-to-host read per loop (loop control).
 * Errors: EINVAL, ESTATE, ECUDA, ETIMEOUT, EDEVICE. */
ALODLM_API int alodlm_denoise_step(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda,
                        int k_max, int rule, const alodlm_step_out *out);

/* alodlm_denoise_step with sampled commits: a position that commits takes a token drawn from
 * its distribution p_i^(s) instead of the argmax.
 * [digest "Method steps", Algorithm 1 (3)]: each committed position samples y_i ~ p_i^(s).
 * The draw is Gumbel-max with counter-based random numbers, so any other implementation can
 * draw the same tokens: for vocabulary id v of position i of sequence b at loop s, the 64-bit
 * word v mod 4 of Philox4x64-10 (Salmon et al., SC 2011) at counter (v div 4, b*N + i, s, 0)
 * under key (seed, step) gives u = (its 53 high bits + 1/2) * 2^-53 and g_v = -log(-log u);
 * the token is the id of the largest z_v + g_v (in double precision, the lowest id on ties).
 * It is fused into the LM-head readout: the logits still never reach global memory.  The
 * entropy, the halting and the forced commit are as in alodlm_denoise_step (a forced commit
 * takes its position's sampled token).  Arguments and errors as for alodlm_denoise_step;
 * `step` is the caller's denoising-step index (part of the key). */
ALODLM_API int alodlm_denoise_step_sampled(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H,
                                           float lambda, int k_max, int rule, uint64_t seed, uint64_t step,
                                           const alodlm_step_out *out);

/* Outputs of a block decode, all caller-owned DEVICE buffers (S = the call's max_steps,
 * K = its k_max). */
typedef struct {
    int32_t *tokens;       /* [B,N] the block after the last step (mask_id where still masked) */
    int32_t *commit_step;  /* [B,N] 1-based step that committed the position; 0 for given ids and
                              positions never committed */
    int32_t *commit_depth; /* [B,N] loop s (1..K) of that step, 0 if never committed */
    int32_t *steps_run;    /* [B] steps that had masks of the sequence at their start */
    int32_t *loops;        /* [S,B] loops run by each sequence in each step (0 for steps not taken) */
    int32_t *rows;         /* [S,2,K] per step: active_rows[K] then readout_rows[K] (as in a step) */
} alodlm_decode_out;

/* Denoise one block until no [MASK] is left, or for max_steps steps.
 * [digest "Method steps", Algorithm 1 (5)]: after each denoising step the committed tokens are
 * written into the sequence and the next step starts, until no [MASK] remains.  Step t + 1
 * takes the tokens of step t as its block ids (every step sees the same prefix KV; the block
 * is re-embedded from its ids).  The whole batch steps together: a sequence without masks
 * still takes part in a step (nothing of it changes) but stops counting steps.
 * Arguments as for alodlm_denoise_step; max_steps >= 1 (N suffices under the paper's rule,
 * which commits at least one position per step; 1 under ALODLM_RULE_PER_TOKEN).
 * steps_taken (host, may be NULL) receives the number of steps run.  Synchronises with the
 * host once per step (a 4-byte "masks left" flag) besides the steps' own reads.  Uses
 * handle-owned scratch for the steps' traces, so calls on one handle must not overlap.
 * Errors: EINVAL, ESTATE, ECUDA, ETIMEOUT, EDEVICE; after an error the outputs are undefined
 * (a failing step returns its own code). */
ALODLM_API int alodlm_decode_block(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda,
                                   int k_max, int rule, int max_steps, const alodlm_decode_out *out, int *steps_taken);

/* alodlm_decode_block with sampled commits (alodlm_denoise_step_sampled): step t (1-based) of
 * the decode draws under key (seed, t). */
ALODLM_API int alodlm_decode_block_sampled(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H,
                                           float lambda, int k_max, int rule, int max_steps, uint64_t seed,
                                           const alodlm_decode_out *out, int *steps_taken);

/* Wait for the handle's stream; returns ETIMEOUT/EDEVICE if a kernel raised the device error
 * word since the last call (the word is then cleared), ECUDA on a CUDA error. */
ALODLM_API int alodlm_sync(alodlm_t *h);

/* Test hook for the error path (no counterpart in the paper): enqueue on the handle's stream a
 * kernel whose one bounded wait (on an mbarrier nothing arrives on) expires after the library's
 * wait limit (about 2 s), raising the device error word exactly as a timed-out wait inside a
 * step would.  The next alodlm_sync then returns ETIMEOUT and clears the word; the handle
 * stays usable (no step kernel keeps state across launches that an expired wait could leave
 * part-way).  No GPU fault is involved.  Errors: EINVAL (null handle), ECUDA. */
ALODLM_API int alodlm_inject_wait_timeout(alodlm_t *h);

/* Work partitions of the kernels' launches, for host-side tests (no counterpart in the paper:
 * they state how the library cuts a GEMM or an attention launch into CTAs).  Pure functions:
 * no handle, no device work, callable without a GPU.  `out` is a caller-owned int32 array.
 * Errors: EINVAL on a null `out` or a size below 1 (text in alodlm_last_error(NULL)).
 *
 * alodlm_plan_gemm: the per-tile linear-layer kernel for out[M, N] = act[M, K] W[N, K]^T:
 * out[0] activation rows per tile (32/64/128/256), out[1] split-K ranks per tile (one cluster,
 * a power of two), out[2] 64-wide k-tiles per rank, out[3] k-tiles in all (4 ints). */
ALODLM_API int alodlm_plan_gemm(int M, int N, int K, int32_t *out);

/* alodlm_plan_gemm_noalloc: the stream-K partition of alodlm_gemm_bf16_noalloc (M <= 64) on
 * num_sms SMs: out[0] activation rows per tile, out[1] CTAs, out[2] (weight tile, k-tile) units
 * per CTA, out[3] the most CTAs that share one weight tile (split partials kept per tile),
 * out[4] 128-row weight tiles, out[5] k-tiles per weight tile (6 ints). */
ALODLM_API int alodlm_plan_gemm_noalloc(int M, int N, int K, int num_sms, int32_t *out);

/* alodlm_plan_attention: one attention launch over packed_rows (= query heads per KV head x
 * rows per sequence) query rows per (sequence, KV head), keys [0, kv_len); causal rows, the
 * SM count, whether the two-query-tile kernel may serve it (head_dim 128, rows without row
 * tables) and whether 16-CTA clusters fit: out[0] 128-row query tiles, out[1] 1 if two query
 * tiles share a CTA, out[2] key splits per query tile (one cluster, a power of two), out[3]
 * keys per split (a multiple of 128), out[4] 1 if the last split also takes the keys past
 * out[2] x out[3] (5 ints). */
ALODLM_API int alodlm_plan_attention(int packed_rows, int n_kv_heads, int n_seq, int kv_len, int causal, int num_sms,
                                     int two_tile_ok, int cluster16_ok, int32_t *out);

/* Free everything the handle owns (synchronises first).  NULL is a no-op. */
ALODLM_API void alodlm_destroy(alodlm_t *h);

/* Last error text of the handle (or of the last failed create when h is NULL).  Valid until the
 * next call on the same handle. */
ALODLM_API const char *alodlm_last_error(const alodlm_t *h);

/* Debug copies (cfg.debug_dump = 1): copy the last step's float32 [B, N, hidden] state of loop
 * `loop` (1-based) into the caller's device buffer dst (enqueued on the handle's stream):
 * which = 0 loop input h^(s-1), 1 Core output h~^(s), 2 readout state r^(s) (after the final
 * RMSNorm), 3 output of the first Core layer at loop s.  Rows of sequences that had stopped before `loop` hold stale data.
 * EINVAL without debug_dump, before a step, or out of range. */
ALODLM_API int alodlm_debug_state(alodlm_t *h, int which, int loop, float *dst);

/* Copy K (which = 0) or V (1) of KV slot `slot` for sequence b, positions [0, n_pos), into the
 * caller's device buffer dst laid out bf16 [n_kv_heads, n_pos, head_dim] (handle's stream).
 * Slots: Prelude layer l -> l; Core layer c at depth d (1-based) -> n_prelude + (d-1)*n_core + c;
 * Coda layer j -> n_prelude + k_max*n_core + j.  Positions P..P+N-1 hold the last step's block
 * K/V of the last loop that wrote the slot.  A Core depth beyond the deepest one built reads that
 * one (the same values under the fallback rule).  For parity checks.  EINVAL out of range. */
ALODLM_API int alodlm_kv_slot(alodlm_t *h, int which, int slot, int b, int n_pos, void *dst);

/* Counters of the last denoise step: kernels launched, loops run (max over the batch) and,
 * if timing was enabled, per kernel class the summed device time (ms) and launch count and the
 * algorithmic bytes and flops (see alodlm_kernel_class_name).  times/launches/bytes/flops may be
 * NULL; each is an array of ALODLM_N_KCLASS entries. */
#define ALODLM_N_KCLASS 9
ALODLM_API int alodlm_step_stats(const alodlm_t *h, int *kernel_launches, double *times_ms, int *launches,
                      double *bytes, double *flops);
/* 1: time every kernel class with CUDA events on the handle's stream during the next steps
 * (adds event records between launches); 0: off (default). */
ALODLM_API int alodlm_set_timing(alodlm_t *h, int on);
/* 1 (default): record each loop of a step as a CUDA graph on first use and replay it (needs a
 * stream other than the legacy/per-thread default stream; timing mode launches directly);
 * 0: launch every kernel directly and drop the recorded graphs. */
ALODLM_API int alodlm_set_graphs(alodlm_t *h, int on);

/* Name of kernel class k (0 <= k < ALODLM_N_KCLASS): "gemm" (linear layers on the CTA-pair and
 * persistent kernels: many activation rows), "attention", "readout_gemm", "readout_combine",
 * "norm", "qkv_rope", "commit", "other", "gemm_tile" (linear layers on the per-tile split-K
 * kernel: few activation rows). */
ALODLM_API const char *alodlm_kernel_class_name(int k);

/* Plain bf16 GEMM through the library's tcgen05 kernels (the ones the step's linear layers use,
 * with W in plain row-major layout): C[m, n] = sum_k A[m, k] * W[n, k],
 * A device bf16 [M, K], W device bf16 [N, K] (both row-major, K-major), C device float32
 * [M, N].  K a multiple of 8 (16-byte rows for TMA), M, N >= 1, all pointers 16-byte aligned.
 * workspace: caller-owned device scratch of workspace_bytes >= 256 bytes, zeroed by the caller
 * before its first use.  Its first 4 bytes are the device status word (non-zero after a call
 * means a bounded wait inside the kernel timed out and C is invalid; the caller clears it);
 * the rest is reserved.  Split-K partial sums meet inside a thread-block cluster and are
 * added in a fixed order, so results are deterministic.  Runs on `stream` of the current
 * device and allocates nothing.  For kernel-level tests and benchmarks.
 * Errors: EINVAL, ECUDA. */
ALODLM_API int alodlm_gemm_bf16(const void *A, const void *W, float *C, int M, int N, int K, float *workspace,
                     size_t workspace_bytes, void *stream);

/* Allocation-free variant of alodlm_gemm_bf16 for a few activation rows (the library's
 * stream-K kernel): C[m, n] = sum_k A[m, k] * W[n, k], A device bf16 [M, K], W device bf16
 * [N, K], C device float32 [M, N], all row-major and 16-byte aligned.  The paper has no
 * counterpart; this entry point exists for callers that cannot allocate device memory
 * themselves: code whose device memory is owned and budgeted by a host framework's own
 * pool, and latency-critical paths that must not pay for cudaMalloc/cudaFree, which can
 * synchronise the device.  It takes no workspace and calls no allocator: its scratch (the
 * status word, per-tile counters and split partials, 16 MB + 4 KB) is a fixed array compiled
 * into the library, which every GPU that loads the library's kernels holds until the
 * process exits.
 * Limits: 1 <= M <= 64, 1 <= N <= 32768, 8 <= K <= 32768, K % 8 == 0; outside them (or if
 * the split of a shape would not fit the array) it returns EINVAL, reason in
 * alodlm_last_error(NULL).
 * status: NULL, or a caller-owned device int32 that receives this call's status word after
 * the kernel (on `stream`): 0, or non-zero if a bounded wait inside the kernel timed out, in
 * which case C is invalid.
 * The first call on a device (and the first call after the device's context changed, e.g.
 * after cudaDeviceReset) looks up the array's device address with that device current; make
 * that first call before any stream capture.  Every call shares the one array: each call
 * clears its status word and counters on `stream` before the kernel, and calls that overlap
 * on the GPU (other streams, other host threads) race and corrupt each other's results --
 * serialise them.  Errors: EINVAL, ECUDA. */
ALODLM_API int alodlm_gemm_bf16_noalloc(const void *A, const void *W, float *C, int M, int N, int K, int32_t *status,
                                        void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ALODLM_H */
