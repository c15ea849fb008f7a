/*
 * mk.h - C ABI of the B200 (sm_100a) decode-step megakernel.
 *
 * One call of mk_decode_step runs one auto-regressive decode step of a
 * Llama-style transformer for a ragged batch as ONE persistent kernel launch:
 * embedding-row gather, per layer RMSNorm -> QKV projection -> RoPE -> paged KV
 * append -> GQA attention over each sequence's prior positions -> O projection
 * -> RMSNorm -> SwiGLU MLP, then the final RMSNorm and the LM head.
 *
 * What is computed: "ForgeMegakernel: A General Framework for Efficient
 * Auto-Regressive Model Decode Megakernels" (paperlayer.ai digest of arXiv
 * 2609.12379v1), §2.1 "The decode step" and §2.3 "Megakernels" (the whole step
 * inside one host launch).  How it is organised: the same page's §4.1 (per-SM
 * instruction streams, dependency counters instead of grid-wide barriers, a
 * shared-memory buffer pool), and "Inside the megakernel serving engine for
 * North Mini Code" (one thread block per SM, task descriptors, counters in
 * global memory, weights streamed into shared memory before their activation
 * dependencies are met, paged attention).
 *
 * Conventions for every entry point:
 *   - Return value: MK_OK (0) or a negative mk_status code.  No exceptions cross
 *     the ABI.  mk_last_error() gives a one-line message for the last failure
 *     of a handle (or of the library when there is no handle).
 *   - "device" pointers are CUDA global-memory addresses on the handle's device;
 *     "host" pointers are ordinary CPU memory.  The caller owns every buffer it
 *     passes; it must stay valid until the call's stream work has finished.
 *   - All tensors are dense and row-major.  Weights are bf16 [out][in], the
 *     layout of a Hugging Face nn.Linear.
 */
#ifndef MK_H_
#define MK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MK_API __attribute__((visibility("default")))

/* A CUDA stream (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st *mk_stream_t;

typedef enum mk_status {
  MK_OK = 0,
  MK_ERR_INVALID_ARG = -1,     /* a null/misaligned pointer, size out of range, bad value */
  MK_ERR_UNSUPPORTED_CFG = -2, /* model shape outside what the kernel implements */
  MK_ERR_SCHEDULE_INVALID = -3,/* the static validator rejected the task schedule */
  MK_ERR_CUDA = -4,            /* a CUDA runtime call failed (message has the CUDA error) */
  MK_ERR_DEVICE_TIMEOUT = -5,  /* a device-side wait ran past the handle's time limit */
  MK_ERR_BOUNDS = -6,          /* the device found a token id, position, length or page id out of range */
  MK_ERR_NO_DEVICE = -7        /* no usable sm_100 device */
} mk_status;

/* Model shape.  Supported: head_dim 64 or 128; n_heads % n_kv_heads == 0 with
 * 1 <= n_heads/n_kv_heads <= 8 (<= 4 at head_dim 128); hidden, ffn, vocab and
 * n_heads*head_dim multiples of 8; page_size 16; 1 <= max_batch <= 16. */
typedef struct mk_model_cfg {
  int32_t n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
  int32_t tied;        /* 1: the LM head is the embedding table (lm_head may equal embed) */
  float rope_theta;    /* RoPE base: inv_freq_j = theta^(-2j/head_dim), rotate-half pairing */
  float rms_eps;       /* RMSNorm epsilon, inside the square root */
  int32_t max_batch;   /* largest batch a step may use */
  int32_t max_ctx;     /* largest position + 1 a sequence may reach */
  int32_t page_size;   /* KV tokens per page; must be 16 */
  /* Llama-3.x RoPE frequency scaling ("rope_type llama3"); rope_scale_factor <= 1 turns it
   * off.  With wavelength w_j = 2 pi / inv_freq_j and the original context length N:
   * w_j < N / high_freq_factor keeps inv_freq_j; w_j > N / low_freq_factor divides it by
   * the factor; in between s = (N / w_j - low) / (high - low) blends the two,
   * (1 - s) inv_freq_j / factor + s inv_freq_j.  The table is built once, in double. */
  float rope_scale_factor, rope_low_freq_factor, rope_high_freq_factor;
  int32_t rope_original_max_pos;
  /* 1: Qwen3-style QK-norm - every query and key head vector is RMS-normalised over
   * head_dim (epsilon rms_eps) and multiplied by the layer's gain q_norm / k_norm before
   * RoPE; the stored key is the normalised, rotated one.  0: none. */
  int32_t qk_norm;
} mk_model_cfg;

/* Device pointers to bf16 weights.  The per-layer members are HOST arrays of
 * n_layers device pointers each.  Shapes ([out][in]): embed, lm_head [vocab][hidden];
 * final_norm, attn_norm[l], mlp_norm[l] [hidden]; wq [n_heads*head_dim][hidden];
 * wk, wv [n_kv_heads*head_dim][hidden]; wo [hidden][n_heads*head_dim];
 * w_gate, w_up [ffn][hidden]; w_down [hidden][ffn]; q_norm[l], k_norm[l] [head_dim]
 * (only with cfg.qk_norm; NULL arrays otherwise).  Every pointer 16-byte aligned.
 * The handle keeps the device pointers (not the host arrays); the weights must
 * outlive the handle. */
typedef struct mk_weight_ptrs {
  const void *embed, *final_norm, *lm_head;
  const void *const *attn_norm, *const *wq, *const *wk, *const *wv, *const *wo;
  const void *const *mlp_norm, *const *w_gate, *const *w_up, *const *w_down;
  const void *const *q_norm, *const *k_norm;
} mk_weight_ptrs;

/* Paged KV cache (device, caller-owned).  k_pool and v_pool are bf16
 * [n_layers][num_pages][n_kv_heads][page_size][head_dim]; entry t of sequence i
 * lives in physical page page_table[i*max_pages_per_seq + t/page_size], slot
 * t % page_size.  Keys are stored after RoPE.  page_table is device int32
 * [>= batch][max_pages_per_seq].
 * Layout choice: inside a page the kv head is the outer index (head-major), not the
 * token.  One head's 16 tokens x head_dim values are then contiguous, and the kernel
 * moves one page of one head as a single tiled TMA box with 128-byte swizzle; a
 * token-major page ([page_size][n_kv_heads][head_dim]) would put that head's rows
 * n_kv_heads*head_dim*2 bytes apart and take a strided box per page and head.  Callers
 * holding token-major pages must transpose them once when filling the cache. */
typedef struct mk_kv_cache {
  void *k_pool, *v_pool;
  const int32_t *page_table;
  int32_t num_pages, max_pages_per_seq;
} mk_kv_cache;

typedef struct mk_handle_s *mk_handle_t;
typedef struct mk_plan_s *mk_plan_t;

/* Options of the per-SM task schedule (zero fields take the defaults). */
typedef struct mk_plan_opts {
  int32_t num_sms;           /* CTAs = SMs of the device (default: queried; host-only plans: 148) */
  int32_t attn_slots_per_sm; /* attention ranges (split-K work items) per SM and layer (default 1) */
  int32_t max_blocks;        /* 8-row blocks per GEMV task, 1..8 (default 8) */
} mk_plan_opts;

typedef struct mk_plan_info {
  int64_t n_tasks, n_stages;          /* over all SMs */
  int64_t max_tasks_per_sm;
  int64_t weight_bytes_min_sm, weight_bytes_max_sm; /* bulk-copied weight bytes per SM */
  int64_t attn_slots;                 /* split-K attention slots per layer */
  int64_t n_counters;
} mk_plan_info;

/* ---- the decode step --------------------------------------------------------------- */

/* Build a handle: derive the per-SM task streams for cfg (mk_plan_create with
 * default options), run the static validator, allocate the handle's device state
 * (dependency counters, activation scratch, RoPE table) on the current device and
 * upload the streams.  Host-synchronous.  Errors: INVALID_ARG, UNSUPPORTED_CFG,
 * SCHEDULE_INVALID, CUDA, NO_DEVICE.  *out is set only on success. */
MK_API int mk_create(const mk_model_cfg *cfg, const mk_weight_ptrs *weights, mk_handle_t *out);

/* As mk_create, from a plan built (and possibly altered) by the caller.  flags:
 * MK_CREATE_SKIP_VALIDATE runs the plan without the static validator (test use:
 * a plan with an unreachable wait must then come back as MK_ERR_DEVICE_TIMEOUT).
 * The plan is copied; the caller still destroys it. */
#define MK_CREATE_SKIP_VALIDATE 1
MK_API int mk_create_from_plan(mk_plan_t plan, const mk_weight_ptrs *weights, int32_t flags,
                               mk_handle_t *out);

/* One decode step, stream-ordered and asynchronous (one kernel launch).
 * Besides the logits it returns the greedy next token (argmax_out), reduced inside the
 * same launch from per-task candidates of the LM head, so a greedy caller needs no
 * second kernel and no read of the [batch][vocab] logits.
 *   token_ids  device int32 [batch]: the new token of each sequence
 *   positions  device int32 [batch]: p_i = prior entries of sequence i = the new
 *              token's position; sequences may all differ (ragged batch)
 *   seq_lens   device int32 [batch]: keys attended, must equal positions + 1
 *   batch      1 .. cfg.max_batch
 *   kv         the cache; the step writes exactly one K and one V entry per
 *              (layer, sequence, kv head) at position p_i and nothing else
 *   logits_out device fp32 [batch][vocab]
 *   argmax_out device int32 [batch] or NULL: greedy next token (lowest index of the max)
 * Host-side argument errors return before anything is launched.  Device-side
 * errors (bounds, timeout) are sticky: they are read with mk_get_status after the
 * stream has been synchronised, and every later step returns that error until
 * mk_reset.  One handle runs one step at a time: steps on one handle must be
 * ordered on the GPU (same stream, or synchronised). */
MK_API int mk_decode_step(mk_handle_t h, const int32_t *token_ids, const int32_t *positions,
                          const int32_t *seq_lens, int32_t batch, const mk_kv_cache *kv,
                          float *logits_out, int32_t *argmax_out, mk_stream_t stream);

/* A multi-token step in one launch: several new tokens of one sequence at once, as when a
 * draft's tokens are verified (speculative decoding) or a prompt is fed in chunks.  Each
 * new token is a batch row; the rows of one sequence are consecutive and sit at
 * consecutive positions.  Row r attends causally: to its sequence's prior entries and to
 * the new tokens of the rows before it in its sequence, and appends its own K/V at its
 * position.  The projections read every weight once for all rows, as for a batch.
 *   group_first device int32 [batch]: the first row of row r's sequence (r itself for a
 *               sequence with one new token); rows first..r must satisfy
 *               positions[r] = positions[first] + (r - first)
 *   page_table  rows r of one sequence must map the same pages (the caller repeats the
 *               sequence's row); entries up to each row's position must be present
 *   the rest as for mk_decode_step (seq_lens[r] = positions[r] + 1; logits and argmax per
 *   row, i.e. per new token).
 * A group_first that breaks these rules is reported as MK_ERR_BOUNDS on the device. */
MK_API int mk_verify_step(mk_handle_t h, const int32_t *token_ids, const int32_t *positions,
                          const int32_t *seq_lens, const int32_t *group_first, int32_t batch,
                          const mk_kv_cache *kv, float *logits_out, int32_t *argmax_out,
                          mk_stream_t stream);

/* Top-k sampling of the next token (the engine's sampler, ForgeMegakernel §4.3), done
 * inside the step's launch by the CTA that releases the LM head's last task, one warp per
 * sequence.  For sequence i of step s, with u = uniforms[s][i]:
 *   the k = top_k largest logits (equal logits: the lower vocabulary index first), ranked
 *   from the largest, v_0 >= v_1 >= ... >= v_{k-1};
 *   weights w_r = exp((v_r - v_0) / temperature), in fp32;
 *   the token is the one of the first rank r whose running sum w_0 + ... + w_r, added in
 *   rank order in fp32, exceeds u * (w_0 + ... + w_{k-1}) (rank k-1 if rounding leaves none).
 * The caller draws the uniforms (any generator), so a run is reproducible from its inputs. */
#define MK_MAX_TOP_K 256
typedef struct mk_sampling {
  int32_t top_k;          /* <= 1: greedy (argmax, lowest index of the max); 2 .. MK_MAX_TOP_K */
  float temperature;      /* finite, > 0 */
  const float *uniforms;  /* device fp32 [n_steps][batch], each in [0, 1) */
} mk_sampling;

/* n_steps decode steps in one call, with no host round trip between them (the engine's
 * generation loop behind the launch: ForgeMegakernel §4.3).  Step k (0-based) takes as its
 * token the one step k-1 chose (step 0: token_ids), sits at position positions[i] + k,
 * appends its K/V entry there and attends to the positions[i] + k + 1 keys up to and
 * including it.
 *   n_steps    >= 1
 *   token_ids  device int32 [batch]: the first step's tokens
 *   positions  device int32 [batch]: the first step's positions
 *   batch, kv  as for mk_decode_step; the page table must already map every position
 *              the run reaches, positions[i] + n_steps - 1
 *   sampling   NULL or top_k <= 1: greedy; else top-k sampling as above (host struct; the
 *              uniforms it points to are device memory)
 *   tokens_out device int32 [n_steps][batch]: row k = the token step k chose, which is
 *              also step k+1's input (the rows are read back by the following steps)
 *   logits_out device fp32 [batch][vocab] or NULL: the last step's logits (every step
 *              writes there; with NULL they go to the handle's own buffer)
 * n_steps stream-ordered launches of the step kernel on `stream`; the call does not wait.
 * Host-side argument errors return before anything is launched.  A step that fails on
 * the device (for example a position past max_ctx, or one without a page: MK_ERR_BOUNDS)
 * sets the sticky status, and every later step of the run then returns at once without
 * touching the cache or tokens_out; read the status with mk_get_status after
 * synchronising. */
MK_API int mk_decode_steps(mk_handle_t h, int32_t n_steps, const int32_t *token_ids,
                           const int32_t *positions, int32_t batch, const mk_kv_cache *kv,
                           const mk_sampling *sampling, int32_t *tokens_out, float *logits_out,
                           mk_stream_t stream);

/* The same step from HOST buffers: copies token_ids/positions/seq_lens (host
 * int32 [batch]) to the handle's device staging area, runs the step, copies the
 * logits (host fp32 [batch][vocab], may be NULL) and argmax (host int32 [batch],
 * may be NULL) back, and synchronises the stream before returning.  Pinned host
 * memory makes the copies asynchronous DMA.  The KV cache stays on the device. */
MK_API int mk_decode_step_host(mk_handle_t h, const int32_t *token_ids, const int32_t *positions,
                               const int32_t *seq_lens, int32_t batch, const mk_kv_cache *kv,
                               float *logits_host, int32_t *argmax_host, mk_stream_t stream);

/* The same step without a handle and without allocating: for callers that may not
 * allocate device memory (a process whose HBM belongs to another allocator, such as a
 * caching allocator that has reserved the free memory, or a latency-critical loop in
 * which cudaMalloc/cudaFree would synchronise the device).  The pages describe no such
 * entry point; it is an interface variant of mk_decode_step, with the same kernel.
 *   cfg, weights  as for mk_create; arguments from token_ids on as for mk_decode_step.
 * Scratch: one file-scope __device__ array of 16 MiB per device (task streams, tensor
 * maps, activations, counters, RoPE table).  A model whose scratch exceeds it (it
 * grows with n_layers, max_batch and max_ctx) is rejected with MK_ERR_INVALID_ARG
 * before anything is launched.  No call allocates device or pinned host memory.
 * Set-up: every call looks the array's address up on the current device; the first
 * call on a device (and any call after the array moved, as after a device reset, or
 * with another cfg or other weight pointers) builds and validates the schedule, encodes
 * the tensor maps, clears the array and uploads the tables, synchronising `stream`.
 * Make the first call before any stream capture.
 * Each call synchronises `stream` and returns the step's device status (MK_OK,
 * MK_ERR_DEVICE_TIMEOUT, MK_ERR_BOUNDS); after a device error the next call first
 * clears the counters and the status.  All calls on a device share the one array, so
 * two of its steps that overlapped on the GPU would race on it: the entry point holds
 * a per-device lock until its step has finished, which makes calls from several host
 * threads run one after another.  Messages: mk_last_error(NULL). */
MK_API int mk_decode_step_static(const mk_model_cfg *cfg, const mk_weight_ptrs *weights,
                                 const int32_t *token_ids, const int32_t *positions,
                                 const int32_t *seq_lens, int32_t batch, const mk_kv_cache *kv,
                                 float *logits_out, int32_t *argmax_out, mk_stream_t stream);

/* Sticky device status of the handle's last steps: MK_OK, MK_ERR_DEVICE_TIMEOUT
 * or MK_ERR_BOUNDS.  Read it after synchronising the stream of the step. */
MK_API int mk_get_status(mk_handle_t h);

/* Clear the sticky device status and the dependency counters (the step after a
 * device error starts from a clean state).  Host-synchronous. */
MK_API int mk_reset(mk_handle_t h);

/* Mid-state capture for checking (the per-task timeline is the separate call
 * mk_set_trace: the two are set and cleared independently, and a checking run need not
 * pay for the trace's stores): when layer_hidden is a device fp32 buffer of
 * [n_layers+1][max_batch][hidden], each later step writes the residual stream
 * after the embedding gather (index 0) and after each layer (index l+1) for its
 * batch rows.  NULL turns capture off. */
MK_API int mk_set_debug(mk_handle_t h, float *layer_hidden);

/* Per-task timeline for profiling: when records is a device uint64 buffer of
 * [capacity][8] with capacity >= mk_num_tasks(h), each later step writes, for task
 * k of the flattened per-SM streams, {globaltimer ns before its dependency wait,
 * after the wait, at its end, meta, compute, reduce, epilogue, signal} where
 * meta = op | layer << 8 | sm << 24 | (SM cycles warp 0 waited for pool slots,
 * capped at 2^24-1) << 40 and the four durations are SM clock cycles measured by
 * warp 0 (compute: stage processing after the slot waits; reduce: cross-warp
 * reduction or attention merge; epilogue: the task's writes, attention combine;
 * signal: the counter release).  NULL turns it off. */
MK_API int mk_set_trace(mk_handle_t h, uint64_t *records, int64_t capacity);

/* Number of task descriptors in the handle's per-SM streams (all SMs). */
MK_API int64_t mk_num_tasks(mk_handle_t h);

/* Device-side wait limit in nanoseconds (default 1e9).  A wait that runs out
 * sets MK_ERR_DEVICE_TIMEOUT, every CTA leaves after its copies in flight have
 * landed, and the launch completes. */
MK_API int mk_set_timeout_ns(mk_handle_t h, uint64_t ns);

/* Number of kernel launches each mk_decode_step makes (1). */
MK_API int mk_launches_per_step(mk_handle_t h);

MK_API int mk_destroy(mk_handle_t h);

/* ---- the kernel-per-op step ------------------------------------------------------------ */

/* The same decode step run the way a conventional engine runs it: one kernel per operation
 * (per layer RMSNorm, QKV GEMV, RoPE + KV append, split-K attention, its combine, O GEMV +
 * residual, RMSNorm, gate/up GEMV, SwiGLU, down GEMV + residual; then the final norm, the
 * LM head and the argmax: 10 * n_layers + 4 launches), each launch allowed to overlap its
 * predecessor's tail (programmatic dependent launch).  A comparison for the single-launch
 * step (ForgeMegakernel §1: engines launch 280-448 kernels per token; §2.3): the launches
 * per token, and the device time the kernel boundaries add.  Plain CUDA-core kernels
 * (fp32 arithmetic on bf16 weights and cache); batches up to 8, no QK-norm.
 *   mk_kpo_create: cfg and weights as for mk_create; allocates its buffers.
 *   mk_kpo_step: arguments as for mk_decode_step (the same cache layout and page table),
 *     plus mode: MK_KPO_GRAPH replays a CUDA graph of the launches (captured on the first
 *     call and again when the batch or the cache changes); MK_KPO_STREAM launches them on
 *     the stream; MK_KPO_TIMED launches them without overlap with an event after each and
 *     synchronises, writing the sum of the kernels' own times to *busy_ms (the events add
 *     their own cost); MK_KPO_EMPTY replays a graph of the same launches, same grids, with
 *     a kernel that does nothing but wait for its predecessor: its time is that of the
 *     launches and kernel boundaries alone (no results are written).  In the other modes the
 *     logits and argmax are copied to the caller's buffers at the end of the step. */
typedef struct mk_kpo_s *mk_kpo_t;
#define MK_KPO_GRAPH 0
#define MK_KPO_STREAM 1
#define MK_KPO_TIMED 2
#define MK_KPO_EMPTY 3
MK_API int mk_kpo_create(const mk_model_cfg *cfg, const mk_weight_ptrs *weights, mk_kpo_t *out);
MK_API int mk_kpo_step(mk_kpo_t k, const int32_t *token_ids, const int32_t *positions,
                       const int32_t *seq_lens, int32_t batch, const mk_kv_cache *kv, float *logits_out,
                       int32_t *argmax_out, int32_t mode, float *busy_ms, mk_stream_t stream);
MK_API int mk_kpo_launches_per_step(mk_kpo_t k);
MK_API int mk_kpo_destroy(mk_kpo_t k);
MK_API const char *mk_kpo_last_error(mk_kpo_t k);

/* ---- routing among handles specialised by bounds ------------------------------------ */

/* A handle is built for bounds (cfg.max_batch, cfg.max_ctx); its schedule is specialised to
 * them - a handle for batch <= 4 stages fp32 operand rows and so more weight columns per
 * pool stage than one for batch 8 - the counterpart of the pages' per-kernel compile-time
 * batch size and context bound with requests routed among kernels (ForgeMegakernel §5.3,
 * Figure 5).  A router holds several handles of one model (same weights) and sends each
 * step to the handle with the smallest max_batch >= batch, ties broken by the smallest
 * max_ctx > max_position, then by the lower index.
 *   mk_route_pick: the rule alone, on host arrays of the n handles' bounds; returns the
 *   index, or MK_ERR_INVALID_ARG when no handle fits.  No GPU needed.
 *   mk_router_create: copies the n handle pointers (the router does not own the handles;
 *   they must outlive it).  mk_router_step: max_position is the largest positions[i]
 *   (host int: the positions themselves are device memory); the other arguments as for
 *   mk_decode_step, run on the picked handle, whose index goes to *picked (may be NULL). */
typedef struct mk_router_s *mk_router_t;
MK_API int mk_route_pick(const int32_t *max_batch, const int32_t *max_ctx, int32_t n, int32_t batch,
                         int32_t max_position);
MK_API int mk_router_create(const mk_handle_t *handles, int32_t n, mk_router_t *out);
MK_API int mk_router_step(mk_router_t r, const int32_t *token_ids, const int32_t *positions,
                          const int32_t *seq_lens, int32_t batch, int32_t max_position,
                          const mk_kv_cache *kv, float *logits_out, int32_t *argmax_out,
                          int32_t *picked, mk_stream_t stream);
MK_API int mk_router_destroy(mk_router_t r);

/* Message of the last failure on h (NULL: of the last handle-less call). */
MK_API const char *mk_last_error(mk_handle_t h);

/* ---- the task schedule (host only; no GPU needed) ----------------------------------- */

/* Derive the per-SM instruction streams for cfg.  Units of work per phase are
 * spread so that every SM's cumulative weight bytes stay within one unit of the
 * others; tasks wait only on dependency counters of earlier phases. */
MK_API int mk_plan_create(const mk_model_cfg *cfg, const mk_plan_opts *opts, mk_plan_t *out);

/* Static validator (runs inside mk_create): every wait target is exactly the
 * number of signals its counter receives; the graph of per-SM program order plus
 * counter edges is acyclic (no deadlock with all CTAs co-resident); every work
 * unit of every phase is covered exactly once; every stage fits a pool slot; and
 * every pair of phases that touch the same scratch buffer, one of them writing,
 * is ordered by counters (no race).  Returns MK_OK or MK_ERR_SCHEDULE_INVALID
 * with the first violation written to msg (msg_len bytes, may be 0). */
MK_API int mk_plan_validate(mk_plan_t plan, char *msg, size_t msg_len);

MK_API int mk_plan_stats(mk_plan_t plan, mk_plan_info *out);

/* Host-side fault injection for tests of the validator and of device timeouts.
 * arg selects the layer (or the task for MK_FAULT_DUP_UNIT). */
typedef enum mk_fault {
  MK_FAULT_DROP_WAIT = 1,      /* the down projection of layer arg stops waiting for gate/up */
  MK_FAULT_RAISE_TARGET = 2,   /* the LM head waits for one signal more than it can receive */
  MK_FAULT_REORDER = 3,        /* on one SM, a down task of layer arg moves before its gate/up task */
  MK_FAULT_DUP_UNIT = 4,       /* a task of layer arg's O projection also covers its neighbour's unit */
  MK_FAULT_OVERSIZE_STAGE = 5  /* a task's stage no longer fits a pool slot */
} mk_fault;
MK_API int mk_plan_inject_fault(mk_plan_t plan, int32_t kind, int32_t arg);

MK_API void mk_plan_destroy(mk_plan_t plan);

#ifdef __cplusplus
}
#endif
#endif /* MK_H_ */
