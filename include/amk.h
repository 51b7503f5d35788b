/*
 * amk.h -- C ABI of libamk: batch-1 decode of a Llama-family decoder as ONE
 * persistent cooperative kernel launch per token on B200 (sm_100a).
 *
 * The operation.  "RightNow-AI/AutoMegaKernel" README (bittide mirror), opening
 * summary: one launch = one forward pass = one token; the whole forward is
 * fused into a single persistent launch because batch-1 decode is bandwidth
 * bound.  Same page, "What is built and verified": one thread block per SM,
 * counter synchronisation, a full Llama-style decode that matches eager
 * PyTorch, and a KV cache threaded across steps so greedy tokens match eager
 * greedy decoding.  paperfeed "RightNow-AI/AutoMegaKernel", "How it works":
 * the per-SM scheduler loop, the instruction set (GEMV tiles, attention
 * tile, RMSNorm, RoPE, SwiGLU, dequant) and a scheduler that lowers the model
 * to a tiled task DAG.  x-techcon "AutoMegaKernel ... persistent cooperative
 * kernel" article, section 1 "statically verified schedule IR": the checks a
 * schedule must pass before it may be launched.
 *
 * Conventions for every function below.
 *  - Return value: AMK_OK (0) or a negative amk_status.  No function aborts
 *    the process or throws; a failed call leaves its outputs untouched unless
 *    stated otherwise.
 *  - "device pointer": memory of the CUDA device current when amk_create was
 *    called.  "host pointer": ordinary CPU memory (pinned or pageable).
 *  - Ownership: weights are BORROWED (the caller keeps them alive and
 *    unchanged until amk_destroy).  Everything else a handle uses (KV cache,
 *    counters, task table, activations, logits) is OWNED by the handle and
 *    freed by amk_destroy.
 *  - Streams: work is enqueued on the stream given to amk_create.  Calls are
 *    asynchronous unless a host output pointer is passed, in which case the
 *    call synchronises that stream before returning.
 *  - A handle is not thread safe; use one handle per host thread.
 */
#ifndef AMK_H
#define AMK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AMK_API __attribute__((visibility("default")))
#else
#define AMK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
typedef enum {
    AMK_OK = 0,
    AMK_ERR_INVALID_ARG = -1,  /* NULL/misaligned pointer, bad size or id */
    AMK_ERR_UNSUPPORTED = -2,  /* shape the lowering cannot tile (reason in amk_last_error) */
    AMK_ERR_VALIDATION = -3,   /* the static validator rejected the schedule */
    AMK_ERR_POS_RANGE = -4,    /* pos < 0, pos >= max_ctx, or token out of range */
    AMK_ERR_LAUNCH = -5,       /* cooperative launch refused (CTAs not co-resident) */
    AMK_ERR_TIMEOUT = -6,      /* a device wait ran past its limit; handle poisoned */
    AMK_ERR_CUDA = -7,         /* another CUDA runtime error */
    AMK_ERR_OOM = -8,          /* device allocation failed */
    AMK_ERR_POISONED = -9,     /* an earlier step timed out; call amk_reset_kv */
    AMK_ERR_NO_DEVICE = -10    /* no CUDA device (host-only functions still work) */
} amk_status;

/* ---- model description ---------------------------------------------------- */
typedef enum { AMK_QUANT_BF16 = 0, AMK_QUANT_W8A16 = 1, AMK_QUANT_W4A16 = 2 } amk_quant;

/* Shapes of a Llama-family decoder (no biases).  head_dim must be even,
 * n_heads a multiple of n_kv_heads.  max_ctx = number of KV-cache rows the
 * handle allocates; decode positions are 0 .. max_ctx-1. */
typedef struct {
    int32_t hidden, n_layers, n_heads, n_kv_heads, head_dim, ffn, vocab, max_ctx;
    float rms_eps;       /* RMSNorm epsilon (e.g. 1e-5) */
    float rope_theta;    /* RoPE base (e.g. 1e4) */
    int32_t tied_embeddings; /* 1: the LM head is the embedding table */
    int32_t quant;       /* amk_quant of the linear weights */
} amk_config;

/* Weights: every leaf is a DEVICE pointer, 16-byte aligned, row-major
 * [out_features][in_features].  Per-layer fields are HOST arrays of n_layers
 * device pointers.  The embedding, norm gains and a tied head are always
 * bf16.  With AMK_QUANT_W8A16 the linear weights (and an untied LM head) are
 * int8 with one fp16 scale per output row: w_jk = scale_j * q_jk (README,
 * results section: W8A16 per-output-channel int8).  With AMK_QUANT_W4A16
 * (gist.science summary, "Belangrijkste Bijdragen": int4 weight-only) they
 * are packed int4, [out][in / 2] bytes, input 2i in the low nibble of byte i
 * (4-bit two's complement), with one fp16 scale per 128 inputs of a row:
 * scales [out][ceil(in / 128)], w_jk = scale_j,k/128 * q_jk; every in must be
 * a multiple of 32.  amk_create packs each int4 matrix once into a copy the
 * handle owns (codes and scales of a row together); the caller's arrays are
 * not read by decode steps.  Scale arrays are ignored for bf16. */
typedef struct {
    const void *embed;         /* bf16 [vocab][hidden] */
    const void *final_norm;    /* bf16 [hidden] */
    const void *lm_head;       /* bf16|int8|int4 [vocab][hidden]; NULL when tied */
    const void *lm_head_scale; /* fp16 [vocab] (W8A16) or [vocab][hidden/128] (W4A16), untied */
    const void *const *attn_norm, *const *ffn_norm;  /* bf16 [hidden] */
    const void *const *wq;     /* [n_heads*head_dim][hidden] */
    const void *const *wk, *const *wv; /* [n_kv_heads*head_dim][hidden] */
    const void *const *wo;     /* [hidden][n_heads*head_dim] */
    const void *const *wgate, *const *wup; /* [ffn][hidden] */
    const void *const *wdown;  /* [hidden][ffn] */
    const void *const *sq, *const *sk, *const *sv, *const *so; /* fp16 [rows] or [rows][groups] */
    const void *const *sgate, *const *sup, *const *sdown;
} amk_weights;

/* Schedule knobs (the pages' ScheduleConfig: tiling, SM assignment,
 * pipelining depth; README "two autoresearch loops").  Zero fields take the
 * defaults from amk_default_options. */
typedef struct {
    int32_t ring_stages;      /* shared-memory weight ring depth (>= 2); 0 = auto:
                                 192 KiB / stage_bytes */
    int32_t stage_bytes;      /* bytes per ring stage (multiple of 1024); 0 = auto:
                                 48 KiB for W8A16 weights, 64 KiB for bf16 */
    int32_t attn_splits;      /* split-K chunks per KV head; 0 = auto */
    int32_t tasks_per_sm;     /* GEMV row tiles per SM per level; 0 = auto */
    int32_t n_sms;            /* persistent CTAs; 0 = all SMs of the device */
    uint32_t wait_timeout_us; /* limit of every device-side wait */
    int32_t debug_skip_signal_task; /* test hook: this task id never signals (level
                                 counters: no add; flagged waits: its flagged words carry
                                 a wrong tag), so a later wait runs out; -1 = off */
    int32_t profile;          /* 1: record per-CTA phase timers (amk_get_profile) */
    int32_t l2_prefetch_kb;   /* while its ring is full, each SM prefetches this many KiB
                                 of its coming weight stream into L2; 0 = off */
    int32_t ffn_fused;        /* one FFN level per layer: gate/up, SwiGLU and the matching
                                 Wdown columns in one task, the slices' down projections
                                 summed into the residual in 64-bit fixed point (amk_create
                                 keeps a packed copy of every Wdown for it; the level
                                 counters then order the steps, see flagged_waits).
                                 1 (default): separate levels with flagged waits; with
                                 flagged_waits = -1, fused when the shape allows and
                                 hidden * element size <= 1.5 KB.  2: whenever the shape
                                 allows; -1: separate gate/up and down levels */
    int32_t pos0_plan;        /* 1 (default): steps at position 0 run a second, validated
                                 schedule without the attention level (softmax over one
                                 key: each head's output is its KV head's V row); -1: off */
    int32_t inflight_kb;      /* cap on the weight bytes each SM's bulk copies keep in flight
                                 (KiB; 0 = default 64, < 0 = no cap).  Queued copies delay
                                 every other memory access of the SM: with 192 KiB in flight
                                 an L2 hit takes ~1.2 us and a grid-wide counter round ~12
                                 us on B200, with 64 KiB ~0.6 us and ~3 us, while the stream
                                 still reaches ~96% of its bandwidth */
    int32_t copy_piece_kb;    /* largest piece a ring stage's copy is issued in, each piece
                                 on its own mbarrier (KiB; 0 = default 64: one piece per
                                 stage; smaller pieces let the cap bind more finely but cost
                                 the producer more issue work) */
    int32_t sm_rotate;        /* SM assignment: each level's tiles go to the least-loaded
                                 SMs scanning from SM (level index * sm_rotate) mod n_sms,
                                 so the knob moves tiles between SMs without changing the
                                 balance; 0 (default) = always from SM 0 */
    int32_t debug_checks;     /* 1: debug checks (race-detection substitutes): amk_create
                                 bounds-checks every resolved task record (rows within their
                                 matrix, KV blocks within the handle's cache, chunk geometry
                                 covering the rows) and puts a 256-byte guard of 0xA5 after
                                 every device buffer the handle owns, which amk_check_guards
                                 verifies after steps; 0 (default): off */
    int32_t flagged_waits;    /* how a task waits for its inputs.  1 (default): every
                                 activation a level hands to the next is a flagged word
                                 (the fp32 value and the step's tag in one 64-bit word),
                                 and a task's poll of the words it reads is its wait: no
                                 level counter, no release fence behind a task's stores
                                 (B200: 4% faster on Llama-7B at context 2048, 7% on
                                 TinyLlama at 0, 8% on SmolLM2 at 128).  -1, or a fused
                                 FFN level: the level counters (release-add by each task,
                                 acquire-poll by the next level's).  With the FFN level
                                 split (either protocol), the SwiGLU vector goes to the
                                 down projection as 32-bit words: the fp32 value rounded to 15 mantissa bits (a
                                 relative error of at most 2^-16), an 8-bit tag in its
                                 low byte */
} amk_options;

typedef struct amk_handle amk_handle;
typedef struct amk_plan amk_plan;

/* ---- schedule IR (the validator's input) -------------------------------- */
/* x-techcon article, section 1: the schedule is a typed SM-level task DAG
 * synchronised by monotonic counters.  A task waits on counters, runs, then
 * adds 1 to each counter it signals.  Access kinds describe what a task does
 * to a range of a buffer within one epoch (one decode step): */
typedef enum {
    AMK_ACC_READ = 0,      /* reads a value produced in this epoch */
    AMK_ACC_WRITE = 1,     /* plain store */
    AMK_ACC_ACCUM = 2,     /* commutative atomic accumulate (add / max) */
    AMK_ACC_READ_PREV = 3, /* reads the value the previous epoch left */
    AMK_ACC_RESET = 4,     /* stores the accumulation identity for the next epoch */
    AMK_ACC_READ_FLAGGED = 5 /* reads flagged words of this epoch: the task polls each word
                                until it carries the epoch's tag, which its single WRITE (or
                                the completion of its ACCUMs) puts there -- a wait on the
                                data itself instead of on a counter */
} amk_access_kind;

enum { AMK_BUF_OUTPUT = 1 }; /* amk_graph_buffer.flags: a result of the step */

typedef struct { int32_t counter, threshold; } amk_graph_wait;
typedef struct { int32_t buffer, kind; int64_t begin, end; } amk_graph_access;
typedef struct {
    int64_t size;   /* elements */
    int32_t flags;  /* AMK_BUF_OUTPUT */
    int32_t pair;   /* -1, or the buffer holding this one's next-epoch copy */
} amk_graph_buffer;
typedef struct {
    int32_t sm;
    int32_t wait_begin, wait_count;     /* into waits[] */
    int32_t signal_begin, signal_count; /* into signals[] (counter ids) */
    int32_t access_begin, access_count; /* into accesses[] */
} amk_graph_task;
typedef struct {
    int32_t n_tasks, n_counters, n_buffers, n_sms;
    int32_t n_waits, n_signals, n_accesses;
    const amk_graph_task *tasks;
    const amk_graph_wait *waits;
    const int32_t *signals;
    const amk_graph_access *accesses;
    const amk_graph_buffer *buffers;
    const int32_t *queue_offsets;  /* [n_sms + 1] */
    const int32_t *queue_tasks;    /* [n_tasks]: SM s runs queue_tasks[off[s]..off[s+1]) in order */
} amk_graph;

/* Validator rules (x-techcon article section 1 and gist.science summary,
 * "De Safety Gate"), checked in this order; the first failure is reported:
 *  V7 referential integrity (ids, ranges, one queue per task, queue = task.sm)
 *  V2 every wait threshold t satisfies 1 <= t <= producers(counter)
 *  V3 a counter with more than one producer is only waited at full count
 *  V10 every element of a READ_FLAGGED range is written in the epoch by
 *     exactly one WRITE, or accumulated by ACCUMs and not written (otherwise
 *     the reader would wait for ever, or could take a value that another
 *     write then replaces)
 *  V1 the producer -> consumer graph is acyclic
 *  V4 every per-SM queue is a linear extension of that graph
 *  V5 every READ happens after every overlapping WRITE/ACCUM of another task
 *  V6 overlapping WRITE/WRITE, WRITE/ACCUM and RESET/RESET of different tasks
 *     are ordered; READ_PREV happens before every overlapping WRITE, ACCUM,
 *     RESET; RESET happens after every other overlapping access
 *  V8 every AMK_BUF_OUTPUT buffer is written or accumulated
 *  V9 for a buffer with a pair, the RESET ranges on the pair cover every
 *     ACCUM range on the buffer (the next epoch's accumulators start at zero)
 * "happens after" = reachable in the union of counter edges (each producer of
 * a counter -> each task waiting on it), flagged edges (each task with a WRITE
 * or ACCUM overlapping a READ_FLAGGED range -> the reader) and queue edges. */
typedef enum {
    AMK_RULE_OK = 0, AMK_RULE_V1 = 1, AMK_RULE_V2 = 2, AMK_RULE_V3 = 3,
    AMK_RULE_V4 = 4, AMK_RULE_V5 = 5, AMK_RULE_V6 = 6, AMK_RULE_V7 = 7,
    AMK_RULE_V8 = 8, AMK_RULE_V9 = 9, AMK_RULE_V10 = 10
} amk_rule;

typedef struct {
    int32_t rule;      /* amk_rule; AMK_RULE_OK when accepted */
    int32_t task_a, task_b, counter, buffer; /* offending items, -1 if n/a */
    char message[256];
} amk_validation_report;

/* ---- library ------------------------------------------------------------- */
AMK_API const char *amk_version(void);
AMK_API const char *amk_strerror(int status);
/* Text of the last error raised on the calling thread (static storage). */
AMK_API const char *amk_last_error(void);

/* Fills *out with the default schedule knobs.  Host only. */
AMK_API int amk_default_options(amk_options *out);

/* Validates an arbitrary task graph (host only, no GPU needed).  Returns
 * AMK_OK if accepted, AMK_ERR_VALIDATION if rejected (details in *report,
 * which may be NULL), AMK_ERR_INVALID_ARG if g is NULL or its counts are
 * negative.  Does not keep any pointer. */
AMK_API int amk_validate_graph(const amk_graph *g, amk_validation_report *report);

/* Lowers a model shape to the per-SM task DAG for n_sms persistent CTAs and
 * validates it, without touching a GPU (host only).  *out is owned by the
 * caller and freed with amk_plan_destroy.  Returns AMK_ERR_UNSUPPORTED for
 * shapes the lowering cannot tile, AMK_ERR_VALIDATION if the validator
 * rejects the result (report filled when non-NULL). */
AMK_API int amk_plan_create(const amk_config *cfg, const amk_options *opt, int32_t n_sms,
                    amk_plan **out, amk_validation_report *report);
/* A read-only view of the plan's graph; valid until amk_plan_destroy. */
AMK_API int amk_plan_graph(const amk_plan *p, amk_graph *out);
/* Per-task kind and layer of a plan ([n_tasks] each; host memory, may be NULL). */
AMK_API int amk_plan_task_info(const amk_plan *p, int32_t *kind, int32_t *layer);
AMK_API void amk_plan_destroy(amk_plan *p);
/* The schedule the plan's steps at position 0 run (amk_options.pos0_plan):
 * validated with the plan, owned by it (not to be destroyed), or NULL. */
AMK_API const amk_plan *amk_plan_pos0(const amk_plan *p);

/* Creates a decoder: lowers, validates (rejection -> AMK_ERR_VALIDATION),
 * allocates the KV cache (bf16 [n_layers][2][n_kv_heads][max_ctx][head_dim],
 * zeroed) and the workspace on the current device, and captures the stream
 * (a cudaStream_t; NULL = legacy default stream).  opt may be NULL. */
AMK_API int amk_create(const amk_config *cfg, const amk_weights *w, const amk_options *opt,
               void *cuda_stream, amk_handle **out);
AMK_API void amk_destroy(amk_handle *h);

/* Zeroes the KV cache, counters and accumulators, and clears a poisoned
 * state.  Asynchronous on the handle's stream. */
AMK_API int amk_reset_kv(amk_handle *h);

/* One decode step = one cooperative launch (README, opening summary).
 *  token_id: the input token at position pos, or -1 to use the greedy token
 *            of the previous step on the device (no host round trip).
 *  pos:      0 <= pos < max_ctx; the step appends K and V at row pos and
 *            attends over rows 0..pos.  Rows < pos must hold earlier steps'
 *            (or amk_get_kv-filled) values.
 *  logits_dev: device float [vocab] that receives the logits, or NULL (the
 *            handle's own buffer is used).
 *  argmax_host: host int32 that receives the greedy token (smallest index of
 *            the largest logit), or NULL.  Non-NULL synchronises the stream.
 * A device wait that runs past wait_timeout_us makes the kernel stop and
 * this call (or the next synchronising one) return AMK_ERR_TIMEOUT. */
AMK_API int amk_decode_step(amk_handle *h, int32_t token_id, int32_t pos,
                    float *logits_dev, int32_t *argmax_host);

/* As amk_decode_step, then copies the logits into HOST memory logits_host
 * [vocab] (may be NULL) and the greedy token into *argmax_host (may be NULL).
 * Always synchronises the stream. */
AMK_API int amk_decode_step_host(amk_handle *h, int32_t token_id, int32_t pos,
                         float *logits_host, int32_t *argmax_host);

/* Device pointers to layer's K and V cache blocks, each
 * bf16 [n_kv_heads][max_ctx][head_dim] (for synthetic long-context fills and
 * tests).  The handle keeps ownership. */
AMK_API int amk_get_kv(amk_handle *h, int32_t layer, void **k_dev, void **v_dev);

/* Device pointer to the handle's logits buffer, fp32 [vocab]. */
AMK_API int amk_get_logits(amk_handle *h, float **logits_dev);

typedef struct {
    int32_t n_tasks, n_counters, n_sms, ring_stages, stage_bytes, attn_splits;
    int32_t smem_bytes, threads_per_cta;
    int64_t weight_bytes;   /* weight + scale + norm bytes streamed per step */
    int64_t kv_row_bytes;   /* K+V bytes of one position over all layers */
    int64_t epoch;          /* decode steps since the last reset */
    int32_t flagged_waits;  /* 1: tasks wait on flagged words, 0: on level counters */
    int32_t ffn_fused;      /* 1: one FFN level per layer */
} amk_plan_stats;
AMK_API int amk_get_stats(amk_handle *h, amk_plan_stats *out);
/* The same figures for a host plan (amk_plan_create), with the resolved
 * schedule knobs (ring shape, attention splits); epoch is 0.  Host only: no
 * device is touched.  AMK_ERR_INVALID_ARG on a NULL argument. */
AMK_API int amk_plan_get_stats(const amk_plan *p, amk_plan_stats *out);

/* Introspection for tests: device pointers (owned by the handle) to the
 * activations the last step left, per layer l, as flagged words (64 bits:
 * the fp32 value in the low half, the step's tag in the high half; act: 32
 * bits, the fp32 value with its 8 low mantissa bits replaced by an 8-bit tag):
 *   qkv  [n_layers][qkv_rows]  q | k | v before RoPE, qkv_rows = (n_heads + 2*n_kv_heads)*head_dim
 *   xmid [n_layers][hidden]    residual stream after attention
 *   xout [n_layers][hidden]    residual stream after the FFN (with a fused FFN level
 *                              the residual after it lives in a fixed-point buffer instead)
 *   act  [n_layers][ffn]       SwiGLU activations (unused with a fused FFN level) */
typedef struct { uint64_t *qkv, *xmid, *xout; uint32_t *act; int32_t qkv_rows; } amk_workspace;
AMK_API int amk_get_workspace(amk_handle *h, amk_workspace *out);

/* Phase timers of the last step, recorded when amk_options.profile was 1
 * (tracing; README, "Honesty rules": always report the distance to the
 * roofline and where the time goes).  Fills `out` (host, n_u64 entries) with
 * n_sms * AMK_PROF_KINDS * AMK_PROF_FIELDS uint64 values, index
 * ((cta * AMK_PROF_KINDS) + kind) * AMK_PROF_FIELDS + field, where kind is
 * the task kind (1 QKV, 2 ATTN, 3 OPROJ, 4 GATEUP, 5 DOWN, 6 LMHEAD) and the
 * fields are: 0 tasks, 1 ns waiting on counters, 2 ns in prologues (less the
 * polls of field 3 made there), 3 ns consumer thread 0 polled flagged words
 * past its first load of them (amk_options.flagged_waits: the wait for the
 * task's inputs), 4 ns from the end of the counter wait to the signal, 5 ns
 * in epilogues, 6 ns all consumer warps together waited for
 * ring stages, 7 ns all consumer warps together spent in their GEMV or
 * attention loops outside those waits.  Kind 0 holds per-CTA totals: field 0
 * the kernel start (globaltimer ns), 1 the consumers' end, 2 ns the producer
 * waited for free stages, 3 the producer's end, 4 bytes the producer copied,
 * 5 ns the producer spent between tasks (reading descriptors and pointers).
 * Synchronises the stream.  AMK_ERR_INVALID_ARG if profiling was off or
 * n_u64 is too small. */
#define AMK_PROF_KINDS 8
#define AMK_PROF_FIELDS 8
AMK_API int amk_get_profile(amk_handle *h, uint64_t *out, int64_t n_u64);

/* Debug checks (amk_options.debug_checks = 1): synchronises the handle's
 * stream and reads back the guard after every device buffer the handle owns;
 * *n_bad = the number of guards a kernel or copy wrote into (0 when every
 * buffer stayed within its bounds): canary words in place of a race
 * detector, so that a task writing past its buffer shows up.
 * AMK_ERR_INVALID_ARG if the handle was created without debug checks. */
AMK_API int amk_check_guards(amk_handle *h, int32_t *n_bad);

/* After AMK_ERR_TIMEOUT: the task that gave up, the counter it waited on,
 * the value it saw and the value it needed (a flagged read that gave up:
 * counter -1, the tag it last saw and the step's tag). */
typedef struct { int32_t code, task, counter, sm; uint32_t seen, target; } amk_error_info;
AMK_API int amk_get_error_info(amk_handle *h, amk_error_info *out);

/* ---- measurement ------------------------------------------------------- */
/* The read ceiling of the decode step's weight stream (README, "Why a
 * megakernel": the floor of a decode step is the bytes it reads over the
 * memory bandwidth): the kernel's own bulk copies -- cp.async.bulk into a
 * shared-memory ring of `stages` stages of stage_bytes on mbarriers, one CTA
 * per SM on n_sms CTAs, evict-first L2 policy -- with nothing consuming them,
 * over `bytes` of the device buffer buf (caller-owned, at least 1 GiB so that
 * L2 cannot hold it, 16-byte aligned; only read).  One warm-up launch, then
 * `reps` timed ones (CUDA events on cuda_stream); *gbs = the best read rate
 * in GB/s.  Synchronises the stream; allocates n_sms words of device memory
 * for the copies' status.  AMK_ERR_INVALID_ARG on a bad argument,
 * AMK_ERR_TIMEOUT if a copy did not land within 1 s, AMK_ERR_CUDA otherwise. */
AMK_API int amk_read_ceiling(const void *buf, int64_t bytes, int32_t n_sms, int32_t stage_bytes,
                             int32_t stages, int32_t reps, void *cuda_stream, double *gbs);

/* ---- decoding without allocating -------------------------------------- */
/* (No counterpart in the AutoMegaKernel pages: an addition for callers that
 * may not allocate device memory.)  Some callers cannot call cudaMalloc: a
 * plugin inside an inference server or framework whose allocator owns every
 * device byte, or a latency-critical loop where cudaMalloc/cudaFree would
 * stall on an implicit device synchronisation.  amk_create allocates, so
 * such a caller uses this entry point instead.  It runs the same decode step
 * as amk_decode_step but allocates nothing: the caller passes the weights,
 * the KV cache and the logits buffer, and the step's scratch (task table,
 * counters, error word, argmax key, activations) lives in one fixed static
 * device array of AMK_NOALLOC_SCRATCH_BYTES bytes, which every GPU that
 * loads this library holds until the process exits.
 *  plan:       from amk_plan_create, for at most the current device's SM count
 *              (a host object; create it once, outside the loop).
 *  w:          as for amk_create (device pointers, borrowed for the call).
 *  kv_cache:   caller-owned device bf16 [n_layers][2][n_kv_heads][max_ctx][head_dim],
 *              16-byte aligned; rows < pos must hold earlier steps' K/V (zeros
 *              at first); the call writes row pos.
 *  token_id:   0 <= token_id < vocab (no device-side token chaining here).
 *  logits_dev: caller-owned device float [vocab] that receives the logits.
 *  argmax_host: host int32 for the greedy token, or NULL.  Non-NULL makes the
 *              call synchronise the stream and report a device error
 *              (AMK_ERR_TIMEOUT); with NULL the call only enqueues work and
 *              device errors are not reported.
 * Returns AMK_ERR_UNSUPPORTED, without touching the GPU, when the model's
 * scratch would exceed AMK_NOALLOC_SCRATCH_BYTES (amk_last_error says how
 * much it needs), and when cuda_stream is capturing (the schedule uploads
 * read host stack memory).  AMK_ERR_INVALID_ARG for the position-0 schedule
 * (amk_plan_pos0) at any pos other than 0.  Every call looks up the static
 * array's device address (cudaGetSymbolAddress; the first lookup on a device
 * may load the library's device code), so the address stays right after a
 * cudaDeviceReset.  A call uploads the
 * schedule (the task table resolved against w and kv_cache) into the shared
 * array unless the previous call on the device left the same plan's table
 * there, resolved against the same pointers in the same CUDA context; every
 * call clears the counters.  The array keeps the last call's contents: calls
 * that can overlap on the GPU (other streams, other host threads) race on it
 * and must be serialised by the caller. */
#define AMK_NOALLOC_SCRATCH_BYTES (16u << 20)
AMK_API int amk_decode_step_noalloc(const amk_plan *plan, const amk_weights *w, void *kv_cache,
                                    int32_t token_id, int32_t pos, float *logits_dev,
                                    int32_t *argmax_host, void *cuda_stream);

#ifdef __cplusplus
}
#endif
#endif /* AMK_H */
