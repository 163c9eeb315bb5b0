/*
 * mk.h — C ABI of the B200 decode megakernel (libmk.so).
 *
 * One persistent kernel runs a whole transformer decode step as a task graph
 * synchronised by Event Tensors ("Event Tensor: A Unified Abstraction for
 * Compiling Dynamic Megakernel", section "Core method": an event tensor is a
 * multi-dimensional array of events, each the completion of a set of
 * SM-granular tasks with a wait count; notify() is an atomic decrement and
 * wait() spins until zero; event dimensions may be symbolic in the batch
 * size; tasks are scheduled statically to per-SM queues or dynamically
 * through a shared queue).  The on-device interpreter is a loop over a switch
 * that takes tasks from a queue in device memory ("Lecture 112: Production
 * Megakernels for Real-World Inference", section "Execution Model").
 *
 * Conventions for every call below:
 *  - No C++ exception crosses this boundary.  Every call returns an
 *    mk_status; on failure mk_last_error() returns a message for the calling
 *    thread (valid until that thread's next mk_* call).
 *  - "device" pointers are CUDA device addresses on the plan's device;
 *    "host" pointers are ordinary host memory.  All weights, caches, inputs,
 *    outputs and the workspace are owned by the caller and must outlive the
 *    plan.  A plan owns host memory only.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Shapes are symbolic: one plan and one compiled kernel serve every batch
 *    size B <= max_batch and every context length < max_ctx, with no
 *    recompilation and no graph re-capture.
 */
#ifndef MK_H_
#define MK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int mk_status;
#define MK_OK 0
#define MK_ERR_INVALID_ARG -1   /* a pointer, size or option is out of range */
#define MK_ERR_UNSUPPORTED -2   /* valid request that this build does not implement */
#define MK_ERR_WORKSPACE -3     /* workspace missing, too small or misaligned */
#define MK_ERR_CUDA -4          /* a CUDA runtime call failed (message has the CUDA error) */
#define MK_ERR_DEVICE_TIMEOUT -5 /* a device spin-wait ran past its limit (see mk_get_status) */
#define MK_ERR_DEVICE_BOUNDS -6 /* the device rejected an index (bad token, slot or context) */
#define MK_ERR_PLAN -7          /* plan validation or simulation found an error */

#define MK_SCHED_STATIC 0   /* per-SM task queues fixed at plan build, counter waits */
#define MK_SCHED_DYNAMIC 1  /* shared device queue; a task is pushed when its event fires */

#define MK_MODEL_DENSE 0     /* dense decoder: attention + SwiGLU FFN per layer */
#define MK_MODEL_MOE_LAYER 1 /* one mixture-of-experts FFN layer (mk_moe_layer); dynamic schedule only */
#define MK_MODEL_MOE_DECODER 2 /* decoder whose FFNs are MoE layers (mk_decode_step); dynamic schedule only */

#define MK_DEBUG_TASK_COUNTS 1u  /* each executed task increments its slot in mk_step_args.task_counts */
#define MK_DEBUG_TRACE 2u        /* the controller records per-task timestamps in mk_step_args.trace */
#define MK_DEBUG_EMPTY_TASKS 4u  /* interpreter measurement (dense plans only): every task keeps its events,
                                    queue pushes and pops but streams no data and runs no body, so a
                                    step times the scheduling alone (its outputs are not computed) */

/* Weights of one mixture-of-experts FFN layer; bf16 row-major, device. */
typedef struct mk_moe_weights {
  const void* w_router;      /* [n_experts][hidden] */
  const float* router_bias;  /* fp32 [n_experts] added to the router logits, or NULL */
  const void* w_gate;        /* [n_experts][expert_ffn][hidden] */
  const void* w_up;          /* [n_experts][expert_ffn][hidden] */
  const void* w_down;        /* [n_experts][hidden][expert_ffn] */
} mk_moe_weights;

/* Per-layer weights of a dense decoder; bf16, row-major [out][in], device. */
typedef struct mk_layer_weights {
  const void* attn_norm;  /* [hidden] RMSNorm gain before attention */
  const void* wq;         /* [n_q_heads*head_dim][hidden] */
  const void* wk;         /* [n_kv_heads*head_dim][hidden] */
  const void* wv;         /* [n_kv_heads*head_dim][hidden] */
  const void* wo;         /* [hidden][n_q_heads*head_dim] */
  const void* ffn_norm;   /* [hidden] RMSNorm gain before the FFN */
  const void* w_gate;     /* [ffn][hidden] */
  const void* w_up;       /* [ffn][hidden] */
  const void* w_down;     /* [hidden][ffn] */
  mk_moe_weights moe;     /* MK_MODEL_MOE_DECODER: this layer's MoE FFN (router, experts) */
} mk_layer_weights;



/* Model description.
 * MK_MODEL_DENSE: head_dim == 64, n_q_heads % n_kv_heads == 0, hidden and
 *   ffn multiples of 256 with hidden <= 2048, n_q_heads*head_dim == hidden.
 * MK_MODEL_MOE_LAYER: only hidden (multiple of 256, <= 2048), n_experts
 *   (<= 64), top_k (<= 8 and <= n_experts), expert_ffn (multiple of 32,
 *   <= 2048), max_tokens (<= 4096) and moe are read.
 * MK_MODEL_MOE_DECODER: the dense fields (ffn, and the dense FFN weights,
 *   are not used) plus n_experts, top_k, expert_ffn and each layer's moe;
 *   the FFN of layer l is the MoE layer on the B tokens' RMSNorm'd residual
 *   rows (ffn_norm gain), added to the residual. */
typedef struct mk_model_desc {
  int kind;               /* MK_MODEL_DENSE or MK_MODEL_MOE_LAYER */
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  float eps;              /* RMSNorm epsilon */
  float rope_theta;       /* rotary base; pair i of a head turns by pos*theta^(-2i/head_dim) */
  int max_batch;          /* largest B a step may use: dense decoder at most 64 (above 8 the plan runs
                             the wide-batch path: materialised bf16 activations and tcgen05 GEMM
                             tasks of 128 weight rows), MoE decoder at most 8 */
  int max_ctx;            /* cache capacity in positions (ctx_lens[b] < max_ctx) */
  int n_slots;            /* sequences the KV cache holds */
  const void* embed;      /* [vocab][hidden] bf16, device */
  const void* lm_head;    /* [vocab][hidden] bf16, device; NULL = tied to embed */
  const void* final_norm; /* [hidden] bf16, device */
  const mk_layer_weights* layers; /* host array [n_layers] of device pointers */
  void* k_cache;          /* bf16 [n_layers][n_slots][n_kv_heads][max_ctx][head_dim], device, post-RoPE keys */
  void* v_cache;          /* bf16, same layout as k_cache */
  int n_experts, top_k, expert_ffn, max_tokens;  /* MK_MODEL_MOE_LAYER and MK_MODEL_MOE_DECODER */
  mk_moe_weights moe;     /* MK_MODEL_MOE_LAYER (the decoder's per-layer experts are in layers[l].moe) */
} mk_model_desc;

/* Plan options; zero-initialise and set what you need (0 = default). */
typedef struct mk_plan_opts {
  int sched;              /* MK_SCHED_STATIC or MK_SCHED_DYNAMIC */
  int n_sm;               /* CTAs of the persistent kernel; 0 = SMs of the current device */
  int host_only;          /* 1: build without touching a GPU (validation/simulation only) */
  int smem_bytes;         /* dynamic shared memory per CTA; 0 = device opt-in maximum */
  /* GEMV task tiles in rows (0 = default): tile_qkv 32 (16 rotate-half
   * pairs); tile_o 16 or 32 (default 32); tile_gu 16 or 32 gate rows plus as
   * many up rows (default 32); tile_down 16, 32 or 64 (default 64); tile_lm 32
   * or 64 (default 64).  kseg: down-projection K segment, a multiple of 256 in
   * [1024, 2048] dividing ffn.  attn_chunk: 64 keys.  Other values are
   * refused with MK_ERR_UNSUPPORTED or MK_ERR_INVALID_ARG. */
  int tile_qkv, tile_o, tile_gu, tile_down, kseg, tile_lm, attn_chunk;
  long long spin_timeout_ns; /* device spin-wait limit; 0 = 2 s */
  unsigned debug_flags;   /* MK_DEBUG_* bits */
  /* Fault injection for failure-detection tests (0 = none).  With
   * MK_SIM_FAULT_COUNT_PLUS_ONE the device plan arms the event that task 0 of
   * family `fault_family` notifies with one wait more than it will ever
   * receive, so the tasks waiting on it run into the spin-wait limit: the
   * kernel records MK_ERR_DEVICE_TIMEOUT (mk_get_status names the waiting
   * task and the counter), every CTA drains its copies and exits, and the
   * CUDA context stays usable.  Only families whose notified event does not
   * depend on the step's symbols (qkv, oproj, gateup, down, lm) are accepted;
   * other values are refused with MK_ERR_INVALID_ARG. */
  int fault;
  int fault_family;
  /* Key chunks (attn_chunk keys each) per attention task, at most 64.  A
   * value > 0 is used as given.  0 = default: a step of up to 8 rows takes a
   * split that follows the step: with C = n_kv_heads * sum_b
   * ceil((ctx_b + 1) / attn_chunk) chunk units and T = ceil(2 n_sm / 3),
   * split = ceil(C / T) clamped to [3, S] (about two thirds of the SMs'
   * worth of tasks), S = 32 for max_batch <= 8 and 24 above; a step of more
   * than 8 rows (a wide-batch plan) takes 24.  Compute warp w of a task takes chunks w, w + 8, ...
   * (warp-MMA scores and P.V with an online softmax).  A task that holds all
   * of its (sequence, kv head)'s chunks writes the finished output; otherwise
   * it leaves one partial, and the last of the pair's tasks to finish merges
   * the pair's partials. */
  int attn_split;
  /* MoE GroupGEMM tiles, chosen per expert from the run-time histogram
   * (0 = default: routing-aware; 1 = routing-aware; 2 = fixed): an expert
   * with more than 64 routed rows gets tiles of 128 rows (its weights stream
   * once per 128 rows), the others tiles of 64 (16 when a tile has at most
   * 16 rows, as the MMA's N). */
  int moe_tiles;
  /* Wide batch (max_batch > 8): how the GEMM tasks' activation operand is
   * stored (0 = default: split when max_batch <= 64; 1 = split; 2 = plain).
   * Split: each row as its bf16 value plus a second row with the bf16
   * remainder (v - value), both multiplied in one MMA and added in the
   * epilogue, so the products see about 16 significant bits of the
   * activation; plain: the bf16 value only.  1 with max_batch > 64 is
   * refused with MK_ERR_UNSUPPORTED. */
  int act_split;
} mk_plan_opts;

typedef struct mk_plan mk_plan;

/* Arguments of one decode step.  All arrays are device memory. */
typedef struct mk_step_args {
  int batch;              /* B, 1 <= B <= max_batch */
  const int* token_ids;   /* int32 [B]: input token of each sequence */
  const int* slot_ids;    /* int32 [B]: KV-cache slot of each sequence (distinct) */
  const int* ctx_lens;    /* int32 [B]: cached tokens; the new token sits at this position */
  float* logits;          /* fp32 [B][vocab] or NULL */
  int* next_tokens;       /* int32 [B]: greedy argmax (ties -> lowest id) */
  unsigned* task_counts;  /* uint32 [mk_plan_task_slots()] or NULL; zeroed by the caller */
  unsigned* trace;        /* uint32 [n_sm][trace_cap][16] or NULL (MK_DEBUG_TRACE): per CTA, record 0
                             is a header {records, notifier batches, notified tasks, fence ns} and
                             records 1.. are tasks {family, index, t_pop, t_ready, t_go, t_done,
                             t_notified, t_compute_start, t_compute_end, t_issue, t_data, and for
                             GEMV tasks t_staged, t_math, t_red, t_epi, t_loads};
                             times are the low 32 bits of %globaltimer in ns */
  int trace_cap;          /* records per CTA in `trace` */
  /* Debug captures (device memory; each NULL to skip, written only when set;
   * B is this step's batch): */
  float* capture_resid;   /* fp32 [n_layers][B][hidden]: the residual stream after each layer */
  void* capture_moe_in;   /* MoE decoder: bf16 [n_layers][B][hidden], each layer's MoE input
                             (RMSNorm of the residual times the ffn_norm gain, as the router reads it) */
  int* capture_topk;      /* MoE decoder: int32 [n_layers][B][top_k], each layer's selected experts */
  int* capture_hist;      /* MoE decoder: int32 [n_layers][n_experts], each layer's expert histogram */
  int* capture_indptr;    /* MoE decoder: int32 [n_layers][n_experts + 1], each layer's exp_indptr */
} mk_step_args;

/* Arguments of one MoE layer call (MK_MODEL_MOE_LAYER).  All arrays are
 * device memory; the debug outputs may be NULL. */
typedef struct mk_moe_args {
  int n_tokens;           /* T, 1 <= T <= max_tokens */
  const void* x;          /* bf16 [T][hidden]: the layer input */
  void* out;              /* bf16 [T][hidden]: sum over the token's top_k experts of weight * expert FFN */
  int* topk_idx;          /* int32 [T][top_k]: selected experts, largest logit first, ties -> lower id */
  float* topk_w;          /* fp32 [T][top_k]: softmax of the selected logits */
  int* hist;              /* int32 [n_experts]: (token, slot) pairs per expert */
  int* indptr;            /* int32 [n_experts + 1]: exclusive prefix sum of hist */
  float* logits;          /* fp32 [T][n_experts]: router logits (bias included) */
  unsigned* task_counts;  /* uint32 [mk_plan_task_slots()] or NULL (MK_DEBUG_TASK_COUNTS); zeroed by the caller */
} mk_moe_args;

typedef struct mk_device_status {
  int code;               /* MK_OK or MK_ERR_DEVICE_* */
  int family;             /* family index of the task that failed, or -1 */
  int index;              /* task index within its family, or -1 */
  int event;              /* event counter index involved, or -1 */
  int sm;                 /* CTA that recorded the error */
} mk_device_status;

typedef struct mk_family_info {
  int op;                 /* MK_OP_* */
  int layer;              /* layer, or -1 for the LM-head families */
  int debug_base;         /* first slot of this family in task_counts */
  int max_extent;         /* slots reserved (largest extent over all bindings) */
  int followup;           /* 1: run by the task whose notify took an event to zero */
  char name[16];
} mk_family_info;

#define MK_OP_QKV 1
#define MK_OP_ATTN 2
#define MK_OP_MERGE 3     /* reserved: not scheduled (a pair's last attention task merges the pair) */
#define MK_OP_OPROJ 4
#define MK_OP_GATEUP 5
#define MK_OP_DOWN 6
#define MK_OP_LM 8
#define MK_OP_LMFIN 10
#define MK_OP_ROUTE 11    /* router logits, top-k, softmax weights, per-expert ranks (8 tokens per task) */
#define MK_OP_MINDPTR 12  /* follow-up: exp_indptr, GroupGEMM tile table, row map, data-dependent event counts */
#define MK_OP_EGU 13      /* GroupGEMM tile: gate/up rows of one expert x its routed rows -> SwiGLU */
#define MK_OP_EDOWN 14    /* GroupGEMM tile: down rows of one expert x its routed rows */
#define MK_OP_COMBINE 15  /* weighted sum of each token's top_k expert outputs (8 tokens per task) */
#define MK_OP_MFIN 16     /* follow-up: end of the layer */
#define MK_OP_NORM 7      /* wide batch, one row: residual materialised, RMSNorm * attention gain -> bf16 */
#define MK_OP_NORM2 9     /* wide batch, one row: RMSNorm * FFN gain -> bf16 */
#define MK_OP_NORMF 17    /* wide batch, one row: final residual, RMSNorm * final gain -> bf16 */

typedef struct mk_sim_report {
  int orders_run;         /* random interleavings executed */
  int tasks_per_order;    /* tasks executed in the last order */
  int races;              /* conflicting accesses not ordered by events */
  int deadlocks;          /* orders that stopped with work left */
  int exactly_once_violations;
  int nonzero_counters;   /* event counters not at zero after an order */
  int static_dynamic_mismatch; /* 1 if the two schedules executed different task sets */
  char first_error[160];
} mk_sim_report;

/* Fault injected into the plan simulator (host only). */
#define MK_SIM_FAULT_NONE 0
#define MK_SIM_FAULT_DROP_NOTIFY 1   /* one task of `fault_family` skips its notify */
#define MK_SIM_FAULT_COUNT_PLUS_ONE 2 /* the wait count of one event of `fault_family` is one too high */
#define MK_SIM_FAULT_NO_WAIT 3       /* tasks of `fault_family` do not wait on their event */
#define MK_SIM_FAULT_COUNT_MINUS_ONE 4 /* the wait count of that event is one too low (also when the
                                        count is armed at run time, as the MoE routing arms its tiles) */

/* Last error message of the calling thread ("" if none). */
const char* mk_last_error(void);

/* Build a plan: validates `m`, tiles every op into task families with
 * symbolic extents, derives the Event Tensors (shapes and wait-count
 * expressions), builds the static per-SM queues and the dynamic successor
 * rules, lowers them to flat integer arrays and validates the result.
 * Host-only and synchronous; touches no GPU when opts->host_only is 1.
 * On success *out owns the plan (free with mk_plan_destroy). */
mk_status mk_plan_build(const mk_model_desc* m, const mk_plan_opts* opts, mk_plan** out);

/* Device workspace the plan needs (bytes, 256-byte aligned start required). */
size_t mk_plan_workspace_bytes(const mk_plan* p);

/* Bind caller-allocated device workspace and upload the lowered plan into it
 * (synchronises `stream`).  Must be called before mk_decode_step.  The dense
 * weight matrices are read through TMA tensor maps encoded here: every weight
 * matrix and norm gain must be 16-byte aligned (MK_ERR_INVALID_ARG
 * otherwise, also when the driver rejects a map); MK_ERR_WORKSPACE for a
 * missing, short or misaligned workspace. */
mk_status mk_plan_bind_workspace(mk_plan* p, void* dev_ptr, size_t bytes, void* stream);

/* One decode step: a single launch of the persistent megakernel on `stream`.
 * Asynchronous; returns launch and argument errors only.  Device-side errors
 * are read with mk_get_status after the stream has synchronised. */
mk_status mk_decode_step(mk_plan* p, const mk_step_args* a, void* stream);

/* Largest plan scratch (mk_plan_workspace_bytes) that mk_decode_step_static
 * serves: 8 MiB, enough for the 16-layer, 2048-wide model at max_batch 4 and
 * max_ctx 8192 (6.7 MiB).  The array is part of libmk.so's device image, so
 * every process that loads the library holds it on each device it uses. */
#define MK_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)

/* mk_decode_step with no workspace and no device allocation.  The Event
 * Tensor pages have no counterpart of this call: it exists for callers that
 * cannot allocate device memory or hand out a workspace, for instance a
 * serving engine that gives all free HBM to its KV-cache pool at start-up and
 * forbids allocation afterwards, or a plain C host program with no device
 * allocator.  The scratch is a module-scope `__device__` array of
 * MK_STATIC_SCRATCH_BYTES (256-byte aligned), one per device.
 *  - The plan must have been built on the current device (not host_only); a
 *    plan needing more scratch than MK_STATIC_SCRATCH_BYTES is rejected with
 *    MK_ERR_WORKSPACE.  mk_plan_bind_workspace is not needed.
 *  - Every call resolves the array's address with cudaGetSymbolAddress
 *    (the first call on a device may load the module), and the first call
 *    with a plan uploads that plan's arrays with cudaMemcpyAsync from host
 *    memory, again after a context reset moved the array: make the first
 *    call before any stream capture.  No graph capture of this call is
 *    supported.
 *  - The array is shared by every plan and every call on the device and keeps
 *    the last call's contents; each call clears the control block and task
 *    queue (cudaMemsetAsync) and starts at launch epoch 1.  Calls that overlap
 *    on the device (other streams, other host threads' streams) race on it.
 *  - Device-side errors are not reported: the control block holding them is
 *    cleared by the next call.  A step stopped by one before its last task
 *    leaves next_tokens unwritten; run the step through mk_decode_step with a
 *    workspace to read the code with mk_get_status.
 * Arguments and launch errors as for mk_decode_step. */
mk_status mk_decode_step_static(mk_plan* p, const mk_step_args* a, void* stream);

/* One mixture-of-experts FFN layer on T tokens: a single launch of the
 * persistent megakernel on `stream` ("Event Tensor: A Unified Abstraction for
 * Compiling Dynamic Megakernel", section "Core method", data-dependent
 * dynamism).  ROUTE tasks compute the router logits, the top_k experts and
 * their softmax weights and count (token, slot) pairs per expert; the task
 * that completes the routing event computes exp_indptr and the GroupGEMM tile
 * table and arms the data-dependent event counts, and the number of gate/up
 * tiles pushed is the one exp_indptr implies; each tile's down tasks wait on
 * that tile's event.  Requires a plan of kind MK_MODEL_MOE_LAYER with
 * MK_SCHED_DYNAMIC and a bound workspace.  Asynchronous; device errors are
 * read with mk_get_status. */
mk_status mk_moe_layer(mk_plan* p, const mk_moe_args* a, void* stream);

/* Read the device status word (synchronous copy).  Returns the recorded
 * device code (MK_OK if none).  After a device error, call mk_plan_reset. */
mk_status mk_get_status(mk_plan* p, mk_device_status* st);

/* Plan and runtime counters.  The last_* fields describe the last launch
 * through mk_decode_step / mk_moe_layer and are read from the device control
 * block with a synchronous copy (call after the stream has synchronised);
 * they are -1 when no workspace is bound, nothing has launched yet, or the
 * plan runs the static schedule. */
typedef struct mk_stats {
  long long launches;          /* kernel launches through this plan, every entry point */
  double build_ms;             /* host time mk_plan_build took */
  int n_families;              /* task families of the plan */
  int n_counters;              /* Event Tensor counters (sum of all event tensors' sizes) */
  int ring_slots;              /* shared-memory ring slots per CTA */
  int n_sm;                    /* CTAs of the persistent kernel */
  long long workspace_bytes;   /* mk_plan_workspace_bytes */
  int queue_ranges_cap;        /* dynamic queue capacity in task ranges (0: static schedule) */
  int last_queue_ranges;       /* ranges pushed during the last launch */
  long long last_queue_tasks;  /* tasks pushed during the last launch (one END per CTA included) */
  long long last_queue_pops;   /* queue pops during the last launch */
} mk_stats;

/* Fill *st.  MK_ERR_INVALID_ARG for null arguments, MK_ERR_CUDA if the
 * control-block copy fails. */
mk_status mk_get_stats(mk_plan* p, mk_stats* st);

/* Clear the device control block (status, barrier and queue counters) and the
 * dynamic queue's entries. */
mk_status mk_plan_reset(mk_plan* p, void* stream);

/* Task-count slots of the debug counter array (mk_step_args.task_counts). */
int mk_plan_task_slots(const mk_plan* p);
int mk_plan_num_families(const mk_plan* p);
mk_status mk_plan_family_info(const mk_plan* p, int family, mk_family_info* out);

/* Where the Event Tensor counters live in the bound workspace: their byte
 * offset from the workspace start and their number (int32 each).  After a
 * step that completed, every counter reads zero: each wait count was met by
 * exactly its number of notifies.  MK_ERR_INVALID_ARG for null arguments. */
mk_status mk_plan_counter_region(const mk_plan* p, long long* byte_offset, int* n_counters);

/* Tile sizes the plan chose, written to out[16] in this order: tile_qkv,
 * tile_o, tile_gu, tile_down, kseg, tile_lm, attn_chunk, n_sm, ring_slots,
 * attn_split (key chunks per attention task; with attn_auto, at most),
 * wide (1: the wide-batch path), act_split (1: wide-batch activations as
 * value + remainder rows), the K segments per tile of the QKV, O-projection
 * and gate/up GEMM tasks (wide batch: a tile's segments run as separate
 * tasks; 1 otherwise), and attn_auto (1: the split follows each step, see
 * mk_plan_opts.attn_split). */
mk_status mk_plan_tiles(const mk_plan* p, int* out);

/* Host validation for one binding of the symbols (B, ctx_lens host array):
 * every event's wait count equals its number of notifiers, every wait
 * targets an event notified only by tasks earlier in the topological order,
 * and the static queues are deadlock-free.  MoE plans are checked on a
 * routing drawn from a fixed seed (the data-dependent counts taken as the
 * routing follow-up arms them).  MK_OK or MK_ERR_PLAN. */
mk_status mk_plan_validate(const mk_plan* p, int batch, const int* ctx_lens_host);

/* Plan simulator (race detector): executes the lowered plan on the host in
 * `n_orders` seeded random interleavings of n_sm simulated SMs, with task
 * bodies that only record the memory regions they read and write.  Checks
 * that every conflicting access pair is ordered by events (vector clocks),
 * that every task runs exactly once, that every counter ends at zero, and
 * that the static and dynamic schedules run the same task set.  For MoE
 * plans (batch = tokens of the layer call; ctx_lens may be NULL for
 * MK_MODEL_MOE_LAYER) every MoE layer gets a routing drawn from `seed` (top_k
 * distinct experts per token, uniform for even seeds, Zipf(1.2)-weighted for
 * odd ones); the routing follow-up then arms the data-dependent event counts
 * and pushes as many GroupGEMM tasks as the routing's exp_indptr implies,
 * and every order runs the dynamic schedule. */
mk_status mk_plan_simulate(const mk_plan* p, int batch, const int* ctx_lens_host,
                           int n_orders, unsigned seed, int fault, int fault_family,
                           mk_sim_report* report);

/* Total bytes of weights, KV reads/writes and outputs one step moves for a
 * binding (the algorithmic HBM traffic of the step). */
double mk_plan_step_bytes(const mk_plan* p, int batch, const int* ctx_lens_host, int with_logits);

void mk_plan_destroy(mk_plan* p);

#ifdef __cplusplus
}
#endif
#endif /* MK_H_ */
