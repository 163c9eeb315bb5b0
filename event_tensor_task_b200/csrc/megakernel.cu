// megakernel.cu — one persistent sm_100a kernel that runs a whole decode step.
//
// Execution model ("Lecture 112: Production Megakernels for Real-World
// Inference", sections "Execution Model" and "Memory Pipelining"; "Event
// Tensor: A Unified Abstraction for Compiling Dynamic Megakernel", section
// "Core method"): one CTA per SM, each running an interpreter — a loop over a
// switch — over tasks taken from a queue in device memory (static: this SM's
// instruction list; dynamic: a shared queue that tasks are pushed onto when
// their event fires).  Tasks synchronise only through Event Tensor counters:
// notify() is an atomic decrement with release semantics, wait() spins with
// acquire loads until the counter is zero.
//
// Warp roles inside a CTA (352 threads):
//   warp 0     producer   walks the task stream ahead of execution and streams
//                         each task's weights into a ring of 16 KB shared-
//                         memory slots: GEMV rows by 2-D/3-D TMA boxes (one
//                         tensor map per weight matrix, 128-byte swizzle, a
//                         task's rows in column slices), cached KV rows and
//                         expert rows by bulk async copies; it never waits on
//                         events, so weight traffic runs ahead of
//                         synchronisation.
//   warp 1     controller takes tasks in order, waits on their events and
//                         releases them to the compute warps through a
//                         two-deep buffer (the next task is staged while the
//                         current one runs).
//   warp 2     notifier   publishes finished tasks with gpu-scope release
//                         decrements, one per distinct counter of a batch; the
//                         decrement that takes a counter to zero queues the
//                         event's follow-up task and, in dynamic mode, pushes
//                         the consumer tasks.
//   warps 3-10 compute    GEMV tasks on tensor cores (warp MMA m16n8k16 bf16,
//                         the batch rows as the n = 8 columns; warp j reads
//                         only slot j of each half of a task), attention
//                         chunks, merges and the MoE task bodies.
// Every spin is bounded by the plan's timeout; on expiry the kernel records an
// error in the control block, raises an abort flag that every spin polls,
// drains its in-flight copies and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstring>
#include <mutex>

#include "../../include/mk.h"
#include "device.cuh"
#include "plan_format.h"

namespace mk {

constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kComputeBase = 96;  // producer, controller and notifier warps come first
constexpr int kThreads = kComputeThreads + kComputeBase;
constexpr int kFifo = 16;
constexpr int kMaxSlots = 16;
constexpr int kDoneQ = 32;    // controller -> notifier
constexpr int kFollowQ = 16;  // notifier -> controller
constexpr int kMaxB = kMaxBatchRows;  // batch rows per step on this path
constexpr int kMaxBlk = 8;    // 256-column blocks of a row (K <= 2048)
constexpr int kMaxKc = 8;     // down-projection K segments (ffn / kseg <= 8192 / 1024)
constexpr int kDynLookahead = 2;
constexpr long long kKvL2Bytes = 64ll << 20;  // half of the 126 MB L2 (see Smem::kv_ef)

// Kernel instances: the plan kinds (MK_MODEL_*) and the wide-batch layouts
// (max_batch > 8) of the dense and the MoE decoder, each with only the code
// paths its plans take (the interpreter roles included), each without and
// with the per-task trace (kTraced: the recording code costs instruction
// fetches even when it records nothing).
constexpr int kKindDenseWide = 3;
constexpr int kKindMoeDecWide = 4;  // the MoE decoder above 8 rows: wide attention half, MoE FFN
constexpr int kTraced = 8;          // instance flag: MK_DEBUG_TRACE plans
template <int K>
struct Kind {
  static constexpr int base = K & 7;
  static constexpr bool trace = (K & kTraced) != 0;
  static constexpr bool wide = base == kKindDenseWide || base == kKindMoeDecWide;
  static constexpr bool moe_layer = base == MK_MODEL_MOE_LAYER;
  static constexpr bool moe_dec = base == MK_MODEL_MOE_DECODER || base == kKindMoeDecWide;
  static constexpr bool moe = moe_layer || moe_dec;
};

struct StepParams {
  int B;                 // batch size; the token count T for an MoE layer
  // MoE layer
  const __nv_bfloat16* moe_x;
  __nv_bfloat16* moe_out;
  int* dbg_idx;
  float* dbg_w;
  int* dbg_hist;
  int* dbg_indptr;
  float* dbg_logits;
  const int* tokens;
  const int* slots;
  const int* ctx;
  float* logits;
  int* next_tokens;
  unsigned* task_counts;
  uint32_t* trace;
  int trace_cap;
  unsigned epoch;
  float* cap_resid;      // [L][B][H] residual after each layer (or null)
  __nv_bfloat16* cap_moe_in;  // MoE decoder: [L][B][H] router input (or null)
};

struct TaskDesc {
  int32_t fam, op, layer, idx;
  int32_t slot_ph;   // ring slot of the task's first copy | parity of its phase << 16
  int32_t nslots;
  int32_t rec;       // trace record of the task (0: none)
  uint32_t t_issue;  // trace: when the producer queued the task (low 32 bits of ns)
};

// Ring geometry of a GEMV op's tasks, fixed for the plan: the task's rows
// (part 0's, then for the rotate-half and gate/up pair ops part 1's) arrive
// in kGemvSlots consecutive ring slots by column: slot j holds columns
// [j cw, (j + 1) cw) of every row, row after row (cw * 2 bytes each).
struct OpGeo {
  int rows_part;  // rows of a part (16 or 32)
  int cw;         // columns per slot (K / kGemvSlots)
  int pairs;      // 1: two parts (rotate-half or gate/up pairs)
};


struct Smem {
  uint64_t full[kMaxSlots], empty[kMaxSlots];
  uint64_t go_bar[2];    // controller -> compute: task k is in cur[k & 1] (count 1)
  uint64_t done_bar[2];  // compute -> controller: task k finished (one arrive per warp)
  uint64_t acc_bar;      // tcgen05: the current GroupGEMM task's accumulator is complete (count 1)
  uint64_t bfull[kBStages], bempty[kBStages];  // wide batch: activation chunks (B operand) in the staging buffer
  uint32_t tmem_base;    // tcgen05: this CTA's tensor-memory allocation (MoE plans)
  uint32_t pad_tm;
  uint64_t fifo_full[kFifo], fifo_empty[kFifo];
  TaskDesc fifo[kFifo];
  TaskDesc cur[2];
  TaskDesc doneq[kDoneQ];
  TaskDesc followq[kFollowQ];
  // per-sequence tables of the step (max_batch entries each, pre one more),
  // in the dynamic region after the staging buffer and the partial tiles
  int *ctx, *slot, *tok, *nch, *pre;
  int fam_ext[kMaxFamilies];
  signed char fam_op[kMaxFamilies], fam_layer[kMaxFamilies];
  // the staging buffer, kSmemFixed bytes past this struct's start: the GEMV
  // activation rows (bf16, row b at b * kActPitch), or fp32 scratch (xs) for
  // the other task bodies; then the GEMV partial tiles (two buffers of
  // [8 warps][32 rows][gbatch]).  Addresses derived from `this`, so the
  // compiler keeps them in the shared window (shared-memory instructions).
  __device__ __forceinline__ unsigned char* stage() { return reinterpret_cast<unsigned char*>(this) + kSmemFixed; }
  __device__ __forceinline__ float* xs() { return reinterpret_cast<float*>(stage()); }
  __device__ __forceinline__ __nv_bfloat16* xa() { return reinterpret_cast<__nv_bfloat16*>(stage()); }
  __device__ __forceinline__ float* gred(int act_bytes) { return reinterpret_cast<float*>(stage() + act_bytes); }
  float red8[kMaxB][kComputeWarps];
  OpGeo geo[OP_COUNT];  // GEMV geometry per op, set in the prologue
  unsigned long long lm_seen[kComputeWarps][kMaxB];  // per compute warp: best argmax key it has published
  uint32_t slot_t[kMaxSlots];  // trace: when the producer issued the slot's copies
  float alsum[kComputeWarps][4], amax[kComputeWarps][4];  // attention: each warp's exp-sum and maximum per head
  int gemm_last;  // wide batch, split K: this CTA's task was the tile's last segment
  int attn_last;  // attention: this CTA's task was its (sequence, kv head)'s last to finish
  int asplit;     // key chunks per attention task in this step (step_attn_split)
  int kv_ef;      // this step's K/V reads exceed half of L2: load them evict-first too
  // wide batch: this CTA's best argmax key per batch column, and what it published
  unsigned long long lm_cta[kMaxBatch], lm_pub[kMaxBatch];
  volatile int released;  // regular tasks the controller has handed to compute
  volatile int dq_head, dq_tail, fq_head, fq_tail, notifier_stop;
  int bad;
};
static_assert(sizeof(Smem) <= kSmemFixed, "fixed shared-memory area exceeds its reserve");
static_assert(kSmemFixed % 128 == 0, "the staging buffer needs 128-byte alignment");
static_assert(offsetof(Smem, full) % 8 == 0 && offsetof(Smem, fifo_full) % 8 == 0, "mbarriers need 8-byte alignment");
constexpr int BAR_COMP = 3;  // named barrier of the 8 compute warps

// ---------------------------------------------------------------- errors
__device__ __noinline__ void record_error(Control* ctl, int code, int fam, int idx, int ev) {
  if (atomicCAS(&ctl->status_code, 0, code) == 0) {
    ctl->status_family = fam;
    ctl->status_index = idx;
    ctl->status_event = ev;
    ctl->status_sm = blockIdx.x;
  }
  atomicExch(&ctl->abort, 1);
}

__device__ __forceinline__ bool aborted(Control* ctl) { return *(volatile int*)&ctl->abort != 0; }

// Bounded wait on an mbarrier phase; false if the kernel is aborting.  Inline
// (no call on the hot path: a call would save the caller's live registers).
__device__ __forceinline__ bool wait_mbar(uint64_t* bar, uint32_t parity, Control* ctl, long long timeout_ns, int fam,
                                          int idx) {
  if (mbar_try(bar, parity)) return true;
  unsigned long long t0 = global_ns();
  for (int it = 0;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63) == 63) {
      if (aborted(ctl)) return false;
      if ((long long)(global_ns() - t0) > timeout_ns) {
        record_error(ctl, MK_ERR_DEVICE_TIMEOUT, fam, idx, -1);
        return false;
      }
    }
  }
}

// A wait on an event inside the CTA that always completes (the controller's
// next release, the tensor cores' accumulator): bounded by three spin limits,
// but not ended by the abort flag, so that every compute warp sees the same
// sequence of tasks and no MMA is still running when its TMEM is read or
// freed (see compute).
__device__ __forceinline__ bool wait_local(uint64_t* bar, uint32_t parity, long long timeout_ns) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (int it = 0;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63) == 63 && (long long)(global_ns() - t0) > 3 * timeout_ns) return false;
  }
}

// ---------------------------------------------------------------- trace
// MK_DEBUG_TRACE: per CTA, records of 16 uint32 (low 32 bits of the global
// timer in ns); record 0 is the CTA's header.
enum TraceField : int {
  TR_FAM = 0, TR_IDX = 1, TR_POP = 2, TR_READY = 3, TR_GO = 4, TR_DONE = 5, TR_NOTIFIED = 6,
  TR_CSTART = 7, TR_CEND = 8, TR_ISSUE = 9, TR_DATA = 10,
  // GEMV tasks: activation staged, products done, partial tiles summed,
  // epilogue items written, the staging's first loads consumed
  TR_STAGED = 11, TR_MATH = 12, TR_RED = 13, TR_EPI = 14, TR_LOADS = 15,
  // header fields
  TRH_RECORDS = 0, TRH_BATCHES = 1, TRH_NOTIFIED = 2, TRH_FENCE_NS = 3
};
__device__ __forceinline__ uint32_t* trace_rec(const StepParams& S, int rec) {
  return (S.trace && rec >= 0 && rec < S.trace_cap) ? S.trace + ((size_t)blockIdx.x * S.trace_cap + rec) * 16
                                                    : nullptr;
}

// ---------------------------------------------------------------- plan helpers
__device__ __forceinline__ int ev_ctr(const DevPlan& P, int ev, int c0, int c1 = 0, int c2 = 0) {
  const EventTensorDesc& e = P.ev[ev];
  int lin = c0;
  if (e.ndim > 1) lin = lin * e.dims[1] + c1;
  if (e.ndim > 2) lin = lin * e.dims[2] + c2;
  return e.base + lin;
}
__device__ __forceinline__ int fam_of(const DevPlan& P, int op, int layer) {
  return layer < 0 ? P.fam_first_layer[op] : P.fam_first_layer[op] + layer * P.fam_stride;
}
// MoE: the scratch block and the weights of an MoE layer (layer -1: the
// MoE-layer plan's single layer)
__device__ __forceinline__ unsigned char* moe_block(const DevPlan& P, unsigned char* ws, int layer) {
  return ws + (layer > 0 ? (size_t)layer * (size_t)P.moe_stride : 0);
}
struct MoeW {
  const void* router; const float* bias; const void* gate; const void* up; const void* down;
};
__device__ __forceinline__ MoeW moe_weights(const DevPlan& P, const LayerPtrs* layers, int layer) {
  if (layer < 0) return MoeW{P.w_router, P.router_bias, P.w_egate, P.w_eup, P.w_edown};
  const LayerPtrs& l = layers[layer];
  return MoeW{l.w_router, l.router_bias, l.we_gate, l.we_up, l.we_down};
}
__device__ __forceinline__ int moe_li(int layer) { return layer > 0 ? layer : 0; }  // MoE event row

__device__ __forceinline__ bool is_followup(int op) {
  return op == OP_MERGE || op == OP_LMFIN || op == OP_MINDPTR || op == OP_MFIN;
}

// Counter a regular task waits on (-1: none).
template <int kKind>
__device__ int wait_counter(const DevPlan& P, const Smem& sm, const TaskDesc& t, int B) {
  constexpr bool kW = Kind<kKind>::wide, kMD = Kind<kKind>::moe_dec;
  switch (t.op) {
    case OP_NORM:  // (the MoE decoder's layers chain through the combine of the layer before)
      return (kMD && t.layer > 0) ? ev_ctr(P, EV_MCOMB, t.layer - 1)
                                                             : ev_ctr(P, EV_IN, t.layer);
    case OP_NORM2: return ev_ctr(P, EV_O, t.layer);
    case OP_NORMF:
      return kMD ? ev_ctr(P, EV_MCOMB, P.n_layers - 1) : ev_ctr(P, EV_IN, P.n_layers);
    case OP_QKV:
      if (kW) return ev_ctr(P, EV_N1, t.layer);
      return (kMD && t.layer > 0) ? ev_ctr(P, EV_MCOMB, t.layer - 1)
                                                             : ev_ctr(P, EV_IN, t.layer);
    case OP_ATTN: {
      if (kW) return ev_ctr(P, EV_QKV, t.layer, 0);
      AttnTask a = decode_attn(t.idx, B, P.n_kv_heads, sm.nch, sm.pre);
      return ev_ctr(P, EV_QKV, t.layer, a.g);
    }
    case OP_OPROJ: return ev_ctr(P, EV_ATTN, t.layer);
    case OP_GATEUP: return kW ? ev_ctr(P, EV_N2, t.layer) : ev_ctr(P, EV_O, t.layer);
    case OP_DOWN: return ev_ctr(P, EV_GU, t.layer, t.idx / P.n_dtiles);
    case OP_LM:
      if (kW) return ev_ctr(P, EV_NF, 0);
      return kMD ? ev_ctr(P, EV_MCOMB, P.n_layers - 1) : ev_ctr(P, EV_IN, P.n_layers);
    case OP_ROUTE: return kMD ? ev_ctr(P, EV_O, t.layer) : -1;
    case OP_EDOWN: return ev_ctr(P, EV_MH, moe_li(t.layer), t.idx / P.nt_d);
    case OP_COMBINE: return ev_ctr(P, EV_MY, moe_li(t.layer));
    default: return -1;  // EGU is pushed only once its tile table exists
  }
}

// ---------------------------------------------------------------- producer
// Copy geometry of the tasks of one family, set up once per family so that a
// slot costs the producer a handful of instructions (no divisions).
struct ProdFam {
  int fam, op, layer;
  const unsigned char* w[3];  // q/k/v (QKV) or the parts' base matrices
  uint32_t row_bytes;         // bytes of one row copy
  uint32_t row_stride;        // bytes between consecutive rows in memory
  uint32_t row_pitch;         // bytes between consecutive rows in a ring slot
  int rps;                    // rows per ring slot
  int slots_per_part;
  int parts;
  size_t task_stride;         // bytes between consecutive tasks' first rows
  const void* tm[4];          // tensor maps: GEMV parts (QKV: q, k, v); EGU: gate, up, routed rows (16-,
                              // 64-row boxes); EDOWN: down, SwiGLU rows (16-, 64-row boxes)
  const void* xg128;          // EGU / EDOWN: the 128-row boxes of the routed and the SwiGLU rows
  const void* hg128;
};

__device__ void prod_setup(const DevPlan& P, const LayerPtrs* layers, const unsigned char* tmaps, int fam, int op,
                           int layer, ProdFam& f) {
  const uint32_t H2 = (uint32_t)P.hidden * 2;
  f.fam = fam; f.op = op; f.layer = layer;
  auto tmap = [&](int l, int m) -> const void* { return tmaps + (size_t)tmap_index(l < 0 ? 0 : l, m) * kTmapBytes; };
  f.tm[0] = f.tm[1] = f.tm[2] = f.tm[3] = nullptr;
  // the RMSNorm gain this family's staging reads (one 2H-byte row, not
  // otherwise L2-resident after a step's weight stream) goes to L2 now, long
  // before the family's first task runs
  const void* gain = op == OP_QKV ? layers[layer].attn_norm
                     : op == OP_GATEUP ? layers[layer].ffn_norm
                     : op == OP_LM ? P.final_norm : nullptr;
  if (gain) bulk_prefetch_l2(gain, H2);
  switch (op) {
    case OP_QKV: f.tm[0] = tmap(layer, TM_WQ); f.tm[1] = tmap(layer, TM_WK); f.tm[2] = tmap(layer, TM_WV); break;
    case OP_OPROJ: f.tm[0] = tmap(layer, TM_WO); break;
    case OP_GATEUP: f.tm[0] = tmap(layer, TM_GATE); f.tm[1] = tmap(layer, TM_UP); break;
    case OP_DOWN: f.tm[0] = tmap(layer, TM_DOWN); break;
    case OP_LM: f.tm[0] = tmaps + (size_t)(P.n_layers * kTmapPerLayer + TMG_LM) * kTmapBytes; break;
    case OP_EGU:
      f.tm[0] = tmap(layer, TM_GATE); f.tm[1] = tmap(layer, TM_UP);
      f.tm[2] = tmap(layer, TM_XG16); f.tm[3] = tmap(layer, TM_XG64);
      break;
    case OP_EDOWN: f.tm[0] = tmap(layer, TM_DOWN); f.tm[1] = tmap(layer, TM_HG16); f.tm[2] = tmap(layer, TM_HG64); break;
    default: break;
  }
  f.xg128 = nullptr;
  f.hg128 = nullptr;
  switch (op) {
    case OP_EGU: f.xg128 = tmap(layer, TM_XG128); break;
    case OP_EDOWN: f.hg128 = tmap(layer, TM_HG128); break;
    default: break;
  }
  f.row_bytes = H2; f.row_stride = H2; f.row_pitch = H2; f.rps = P.slot_bytes / (int)H2; f.parts = 1;
  f.w[0] = f.w[1] = f.w[2] = nullptr;
  f.task_stride = 0;
  f.slots_per_part = 1;
  switch (op) {
    case OP_QKV: {
      const LayerPtrs& lp = layers[layer];
      f.w[0] = (const unsigned char*)lp.wq; f.w[1] = (const unsigned char*)lp.wk; f.w[2] = (const unsigned char*)lp.wv;
      f.parts = 2; f.slots_per_part = (P.tile_qkv / 2) / f.rps;
    } break;
    case OP_OPROJ:
      f.w[0] = (const unsigned char*)layers[layer].wo;
      f.slots_per_part = P.tile_o / f.rps; f.task_stride = (size_t)P.tile_o * H2;
      break;
    case OP_GATEUP:
      f.w[0] = (const unsigned char*)layers[layer].w_gate; f.w[1] = (const unsigned char*)layers[layer].w_up;
      f.parts = 2; f.slots_per_part = P.tile_gu / f.rps; f.task_stride = (size_t)P.tile_gu * H2;
      break;
    case OP_DOWN:
      f.w[0] = (const unsigned char*)layers[layer].w_down;
      f.row_bytes = (uint32_t)P.kseg * 2; f.row_stride = (uint32_t)P.ffn * 2; f.row_pitch = f.row_bytes;
      f.rps = P.slot_bytes / (int)f.row_bytes; f.slots_per_part = P.tile_down / f.rps;
      break;

    case OP_LM:
      f.w[0] = (const unsigned char*)P.lm_head;
      f.slots_per_part = ceil_div(P.tile_lm, f.rps); f.task_stride = (size_t)P.tile_lm * H2;
      break;
    default: break;  // ATTN: per task
  }
}

template <int kKind>
__device__ __forceinline__ int task_slots(const DevPlan& P, const ProdFam& f, int idx) {
  if (f.op == OP_ATTN) return P.attn_split;  // (at most; the task's chunks)
  if (Kind<kKind>::wide && (f.op == OP_QKV || f.op == OP_OPROJ || f.op == OP_LM)) return P.hidden / 64;
  if (Kind<kKind>::wide && f.op == OP_GATEUP) return 2 * (P.hidden / 64);
  if (Kind<kKind>::wide && f.op == OP_DOWN) return P.kseg / 64;
  if (f.op == OP_NORM || f.op == OP_NORM2 || f.op == OP_NORMF) return 0;
  if (f.op == OP_ROUTE || f.op == OP_COMBINE || f.op == OP_MINDPTR || f.op == OP_MFIN) return 0;
  if (f.op == OP_QKV || f.op == OP_OPROJ) return kGemvSlots;
  if (f.op == OP_GATEUP) return P.tile_gu > 16 ? 2 * kGemvSlots : kGemvSlots;
  if (f.op == OP_DOWN) return P.tile_down > 32 ? 2 * kGemvSlots : kGemvSlots;
  if (f.op == OP_LM) return P.tile_lm > 32 ? 2 * kGemvSlots : kGemvSlots;
  if (f.op == OP_EGU) return 3 * (P.hidden / 64);  // per 64-column chunk: gate rows, up rows, routed rows
  if (f.op == OP_EDOWN) return 2 * (P.eff / 64);   // per 64-column chunk: down rows, SwiGLU rows
  return f.parts * f.slots_per_part;
}

// A GroupGEMM tile's geometry: expert, m block, first compact row and row count.
struct MoeTile { int e, m, r0, nrows, tm; };
__device__ __forceinline__ MoeTile moe_tile(const DevPlan& P, const unsigned char* mb, int tile) {
  MoeTile t;
  t.e = __ldcg(reinterpret_cast<const int*>(mb + P.off_mtile_e) + tile);
  t.m = __ldcg(reinterpret_cast<const int*>(mb + P.off_mtile_m) + tile);
  const int h = __ldcg(reinterpret_cast<const int*>(mb + P.off_mhist) + t.e);
  const int tm = moe_tile_rows(h, P.moe_tm, P.moe_big);
  t.r0 = __ldcg(reinterpret_cast<const int*>(mb + P.off_mindptr) + t.e) + t.m * tm;
  t.tm = tm;
  t.nrows = min(tm, h - t.m * tm);
  return t;
}
// rows of the B operand a tile loads (its TMA box and the MMA's N): 16, 64 or 128
__device__ __forceinline__ int moe_tile_n(int nrows) { return nrows <= 16 ? 16 : nrows <= kMoeTileRows ? kMoeTileRows : kMoeBigTileRows; }

template <int kKind>
__device__ void producer(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                         unsigned char* ws, Control* ctl) {
  const LayerPtrs* layers = reinterpret_cast<const LayerPtrs*>(ws + P.off_layers);
  const long long tmo = P.spin_timeout_ns;
  uint32_t ring_seq = 0, fifo_seq = 0;
  int slot = 0;          // ring_seq % ring_slots
  uint32_t phase = 0;    // (ring_seq / ring_slots) & 1
  int emitted = 0;
  int qr = 0;  // dynamic queue: range cursor of this CTA
  QRange* Q = reinterpret_cast<QRange*>(ws + P.off_queue);
  bool ok = true;
  ProdFam f;
  f.fam = -2;
  const uint64_t wpol = l2_evict_first_policy();  // weight streams: first out of L2
  // K/V chunks: evict-first too when the step's K/V would not stay in L2 anyway
  const uint64_t kvpol = sm.kv_ef ? wpol : l2_evict_normal_policy();

  // acquire the next ring slot: wait until the compute warps released it
  auto next_slot = [&](int fam, int idx, unsigned char*& dst, uint64_t*& bar) -> bool {
    if (!wait_mbar(&sm.empty[slot], phase ^ 1, ctl, tmo, fam, idx)) return false;
    if (Kind<kKind>::trace && S.trace) sm.slot_t[slot] = (uint32_t)global_ns();
    dst = ring + (size_t)slot * P.slot_bytes;
    bar = &sm.full[slot];
    ring_seq++;
    if (++slot == P.ring_slots) { slot = 0; phase ^= 1; }
    return true;
  };
  // a GEMV task's rows by column slices: slot j gets columns [x0 + j cw,
  // x0 + (j + 1) cw) of part 0's rows (from row y0 of map tm0), then of part
  // 1's rows (row y1 of tm1), as one TMA box each
  auto stream_tiles = [&](int fam, int idx, int rows_part, int cw, int x0, const void* tm0, int y0, const void* tm1,
                          int y1) -> bool {
    const uint32_t part_bytes = (uint32_t)rows_part * cw * 2;
    for (int j = 0; j < kGemvSlots; ++j) {
      unsigned char* dst;
      uint64_t* bar;
      if (!next_slot(fam, idx, dst, bar)) return false;
      mbar_arrive_expect_tx(bar, tm1 ? 2 * part_bytes : part_bytes);
      if (cw >= 64) {  // swizzled [rows][cw / 64][64] boxes
        const int xc = (x0 + j * cw) >> 6;
        tma_load_3d_hint(dst, tm0, 0, xc, y0, bar, wpol);
        if (tm1) tma_load_3d_hint(dst + part_bytes, tm1, 0, xc, y1, bar, wpol);
      } else {
        tma_load_2d_hint(dst, tm0, x0 + j * cw, y0, bar, wpol);
        if (tm1) tma_load_2d_hint(dst + part_bytes, tm1, x0 + j * cw, y1, bar, wpol);
      }
    }
    return true;
  };

  // (always inlined: called from three places, the producer would otherwise
  // become a call whose frame holds its state; ptxas reported stack frames of
  // up to 2.3 KB for the MoE instances when it was not)
  auto emit = [&](int fam, int idx) __attribute__((always_inline)) -> bool {
    int op = OP_END, layer = -1;
    if (fam >= 0) {
      op = sm.fam_op[fam];
      layer = sm.fam_layer[fam];
      if (fam != f.fam) prod_setup(P, layers, ws + P.off_tmap, fam, op, layer, f);
    }
    TaskDesc d;
    d.fam = fam; d.idx = idx; d.op = op; d.layer = layer;
    const bool empty = (P.debug_flags & MK_DEBUG_EMPTY_TASKS) != 0;  // scheduling only: no copies
    d.nslots = (fam >= 0 && !empty) ? task_slots<kKind>(P, f, idx) : 0;
    d.slot_ph = slot | (int)(phase << 16);
    d.rec = 0;
    int k = fifo_seq % kFifo;
    if (!wait_mbar(&sm.fifo_empty[k], ((fifo_seq / kFifo) & 1) ^ 1, ctl, tmo, fam, idx)) return false;
    d.t_issue = (Kind<kKind>::trace && S.trace) ? (uint32_t)global_ns() : 0u;
    sm.fifo[k] = d;
    mbar_arrive(&sm.fifo_full[k]);
    fifo_seq++;
    if (fam < 0) return true;
    if (empty) { emitted++; return true; }
    if (Kind<kKind>::wide && (op == OP_QKV || op == OP_OPROJ || op == OP_GATEUP || op == OP_DOWN || op == OP_LM)) {
      // wide batch: the task's 128 weight rows in 64-column chunks, one slot
      // per chunk and part (gate/up: the gate rows, then the up rows); the
      // activation (the B operand) is loaded by the MMA-issuing thread once
      // the task's event has fired (see gemm_issue_wide)
      // (QKV, O and gate/up: K segment seg of tile idx / gseg)
      const int gseg = op == OP_QKV ? P.gseg_qkv : op == OP_OPROJ ? P.gseg_o : op == OP_GATEUP ? P.gseg_gu : 1;
      const int tile = idx / gseg, seg = idx - tile * gseg;
      const int K = op == OP_OPROJ ? P.n_q_heads * P.head_dim : P.hidden;
      int row = tile * kWideRows, x0 = seg * (K / gseg), nk = K / gseg / 64;
      const void* m0 = f.tm[0];
      if (op == OP_QKV) {
        const int nq = P.n_q_heads * P.head_dim / kWideRows, nkv = P.n_kv_heads * P.head_dim / kWideRows;
        const int kind = tile < nq ? 0 : tile < nq + nkv ? 1 : 2;
        m0 = f.tm[kind];
        row = (tile - (kind == 0 ? 0 : kind == 1 ? nq : nq + nkv)) * kWideRows;
      } else if (op == OP_DOWN) {
        const int kc = idx / P.n_dtiles;
        row = (idx - kc * P.n_dtiles) * kWideRows;
        x0 = kc * P.kseg;
        nk = P.kseg / 64;
      }
      for (int c = 0; c < nk; ++c)
        for (int part = 0; part < (op == OP_GATEUP ? 2 : 1); ++part) {
          unsigned char* dst;
          uint64_t* bar;
          if (!next_slot(fam, idx, dst, bar)) return false;
          mbar_arrive_expect_tx(bar, (uint32_t)kWideRows * 128u);
          tma_load_2d_hint(dst, part ? f.tm[1] : m0, x0 + c * 64, row, bar, wpol);
        }
      emitted++;
      return true;
    }
    switch (op) {
      case OP_QKV: {
        // rotate-half pairs: rows j0.. of the head, then rows j0 + D/2.. of it
        QkvTile q = decode_qkv(P, idx);
        const int y = q.head * P.head_dim + q.j0, half = P.tile_qkv / 2;
        if (!stream_tiles(fam, idx, half, P.hidden / kGemvSlots, 0, f.tm[q.kind], y, f.tm[q.kind],
                          y + P.head_dim / 2))
          return false;
      } break;
      case OP_OPROJ:
        if (!stream_tiles(fam, idx, P.tile_o, P.hidden / kGemvSlots, 0, f.tm[0], idx * P.tile_o, nullptr, 0))
          return false;
        break;
      case OP_GATEUP:
        if (P.tile_gu <= 16) {  // one half: 16 gate + 16 up rows per slot
          if (!stream_tiles(fam, idx, P.tile_gu, P.hidden / kGemvSlots, 0, f.tm[0], idx * P.tile_gu, f.tm[1],
                            idx * P.tile_gu))
            return false;
        } else {  // two halves of 8 slots: the gate rows, then the up rows
          if (!stream_tiles(fam, idx, P.tile_gu, P.hidden / kGemvSlots, 0, f.tm[0], idx * P.tile_gu, nullptr, 0) ||
              !stream_tiles(fam, idx, P.tile_gu, P.hidden / kGemvSlots, 0, f.tm[1], idx * P.tile_gu, nullptr, 0))
            return false;
        }
        break;
      case OP_DOWN: {
        const int kc = idx / P.n_dtiles, n = idx - kc * P.n_dtiles;
        for (int r0 = 0; r0 < P.tile_down; r0 += 32)  // halves of at most 32 rows
          if (!stream_tiles(fam, idx, min(32, P.tile_down), P.kseg / kGemvSlots, kc * P.kseg, f.tm[0],
                            n * P.tile_down + r0, nullptr, 0))
            return false;
      } break;
      case OP_LM:  // the last tile's rows past the vocabulary read as zeros
        for (int r0 = 0; r0 < P.tile_lm; r0 += 32)
          if (!stream_tiles(fam, idx, 32, P.hidden / kGemvSlots, 0, f.tm[0], idx * P.tile_lm + r0, nullptr, 0))
            return false;
        break;
      case OP_EGU:
      case OP_EDOWN: if constexpr (Kind<kKind>::moe) {
        // GroupGEMM tile (tcgen05): per 64-column chunk of K, the task's 128
        // weight rows (gate/up: the gate rows, then the up rows, one slot
        // each) and the tile's routed rows as the B operand, each a 2-D TMA
        // box under the 128-byte swizzle.  The tile's expert and rows come
        // from the tables the routing follow-up wrote, and the B rows were
        // written by other SMs' generic stores (routing tasks: the token rows;
        // gate/up tasks: the SwiGLU rows).  This task was popped after its
        // push, which followed those writes; the proxy fence orders them
        // before this thread's TMA reads.
        const unsigned char* mb = moe_block(P, ws, layer);
        const bool gu = op == OP_EGU;
        const int per = gu ? P.nt_gu : P.nt_d;
        const int tile = idx / per, n = idx - tile * per;
        const MoeTile mt = moe_tile(P, mb, tile);
        const int nb = moe_tile_n(mt.nrows);
        const uint32_t bbytes = (uint32_t)nb * 128;
        fence_proxy_async_global();
        const int wrow = mt.e * (gu ? P.eff : P.hidden) + n * kMoeTaskRows;
        const int brow = gu ? mt.e * P.moe_cap + mt.m * mt.tm : mt.r0;
        const void* bmap = gu ? (nb == 16 ? f.tm[2] : nb == kMoeTileRows ? f.tm[3] : f.xg128)
                              : (nb == 16 ? f.tm[1] : nb == kMoeTileRows ? f.tm[2] : f.hg128);
        const int nk = (gu ? P.hidden : P.eff) / 64;
        for (int c = 0; c < nk; ++c) {
          unsigned char* dst;
          uint64_t* bar;
          for (int part = 0; part < (gu ? 2 : 1); ++part) {
            if (!next_slot(fam, idx, dst, bar)) return false;
            mbar_arrive_expect_tx(bar, 128u * 128u);
            tma_load_2d_hint(dst, f.tm[part], c * 64, wrow, bar, wpol);
          }
          if (!next_slot(fam, idx, dst, bar)) return false;
          mbar_arrive_expect_tx(bar, bbytes);
          tma_load_2d(dst, bmap, c * 64, brow, bar);
        }
      } break;
      case OP_ATTN: {
        // the task's key chunks (the step's split of them at most), one slot each:
        // the chunk's 64 cache rows of K, then of V, as swizzled TMA boxes
        // (rows past max_ctx read as zeros; the task masks rows past ctx)
        AttnTask a = decode_attn(idx, S.B, P.n_kv_heads, sm.nch, sm.pre);
        const int p = sm.ctx[a.b];
        const int c0 = a.c * sm.asplit, c1 = min(c0 + sm.asplit, ceil_div(p + 1, P.chunk));
        const int plane = (layer * P.n_slots + sm.slot[a.b]) * P.n_kv_heads + a.g;
        const unsigned char* gm = ws + P.off_tmap + (size_t)P.n_layers * kTmapPerLayer * kTmapBytes;
        for (int cc = c0; cc < c1; ++cc) {
          unsigned char* dst;
          uint64_t* bar;
          if (!next_slot(fam, idx, dst, bar)) return false;
          mbar_arrive_expect_tx(bar, 2u * (uint32_t)P.chunk * 128u);
          tma_load_3d_hint(dst, gm + (size_t)TMG_KC * kTmapBytes, 0, cc * P.chunk, plane, bar, kvpol);
          tma_load_3d_hint(dst + (size_t)P.chunk * 128, gm + (size_t)TMG_VC * kTmapBytes, 0, cc * P.chunk, plane, bar,
                           kvpol);
        }
      } break;
      default: break;
    }
    emitted++;
    return true;
  };

  if (P.sched == MK_SCHED_STATIC) {
    const Instr* ins = reinterpret_cast<const Instr*>(ws + P.off_instr) + (size_t)blockIdx.x * P.n_instr_per_sm;
    for (int k = 0; k < P.n_instr_per_sm && ok; ++k) {
      Instr in = ins[k];
      if (in.family < 0) break;
      int lo, hi;
      instr_range(in, sm.fam_ext[in.family], lo, hi);
      for (int i = lo; i < hi && ok; ++i) ok = emit(in.family, i);
    }
  } else {
    for (;;) {
      // bounded lookahead: do not hoard ready tasks other SMs could run
      unsigned long long t0 = global_ns();
      while (emitted - sm.released > kDynLookahead) {
        __nanosleep(64);
        if (aborted(ctl)) { ok = false; break; }
        if ((long long)(global_ns() - t0) > tmo) { record_error(ctl, MK_ERR_DEVICE_TIMEOUT, -1, -1, -1); ok = false; break; }
      }
      if (!ok) break;
      unsigned long long ticket = atomicAdd(&ctl->q_head, 1ull);
      int fam = -1, idx = 0;
      bool found = false;
      t0 = global_ns();
      int it = 0;
      while (!found) {
        if (qr >= P.queue_ranges) { record_error(ctl, MK_ERR_DEVICE_BOUNDS, -1, qr, -1); ok = false; break; }
        if (ld_acquire_u32(&Q[qr].seq) == S.epoch) {
          unsigned long long st = __ldcg(&Q[qr].start);
          int cnt = __ldcg(&Q[qr].count);
          if (ticket < st + (unsigned long long)cnt) {
            fam = __ldcg(&Q[qr].family);
            idx = __ldcg(&Q[qr].lo) + (int)(ticket - st);
            found = true;
          } else {
            qr++;
          }
        } else if ((++it & 63) == 0) {
          if (aborted(ctl)) { ok = false; break; }
          if ((long long)(global_ns() - t0) > tmo) { record_error(ctl, MK_ERR_DEVICE_TIMEOUT, -1, qr, -1); ok = false; break; }
        }
      }
      if (!ok) break;
      if (fam < 0) break;  // END
      ok = emit(fam, idx);
      if (!ok) break;
    }
  }
  if (ok) ok = emit(-1, 0);
  // drain: every issued copy lands before the CTA may exit
  uint32_t lo = ring_seq > (uint32_t)P.ring_slots ? ring_seq - P.ring_slots : 0;
  for (uint32_t q = lo; q < ring_seq; ++q) {
    uint64_t* bar = &sm.full[q % P.ring_slots];
    uint32_t par = (q / P.ring_slots) & 1;
    unsigned long long t0 = global_ns();
    while (!mbar_try(bar, par)) {
      if ((long long)(global_ns() - t0) > tmo) break;
    }
  }
}

// ---------------------------------------------------------------- notifier
__device__ void push_range(const DevPlan& P, const StepParams& S, Control* ctl, unsigned char* ws, int fam,
                           int lo, int count) {
  if (count <= 0) return;
  QRange* Q = reinterpret_cast<QRange*>(ws + P.off_queue);
  unsigned long long old = atomicAdd(&ctl->q_tail, (1ull << 40) | (unsigned long long)count);
  int r = (int)(old >> 40);
  if (r >= P.queue_ranges) { record_error(ctl, MK_ERR_DEVICE_BOUNDS, fam, lo, r); return; }
  Q[r].family = fam;
  Q[r].lo = lo;
  Q[r].count = count;
  Q[r].start = old & ((1ull << 40) - 1);
  st_release_u32(&Q[r].seq, S.epoch);
}

// What notify() of a finished task does: the counter it decrements, whether
// the decrement's result is needed (a follow-up or a dynamic push hangs on
// it), and the follow-up it triggers when the counter reaches zero.
struct NotifyInfo {
  int ctr, ffam, fop, flayer, fidx, need_old;
};

template <int kKind>
__device__ NotifyInfo notify_info(const DevPlan& P, const StepParams& S, const Smem& sm, const TaskDesc& t) {
  const bool dyn = P.sched == MK_SCHED_DYNAMIC;
  NotifyInfo n;
  n.ctr = -1; n.ffam = -1; n.fop = 0; n.flayer = -1; n.fidx = 0; n.need_old = 0;
  switch (t.op) {
    case OP_NORM: n.ctr = ev_ctr(P, EV_N1, t.layer); break;
    case OP_NORM2: n.ctr = ev_ctr(P, EV_N2, t.layer); break;
    case OP_NORMF: n.ctr = ev_ctr(P, EV_NF, 0); break;
    case OP_QKV: n.ctr = ev_ctr(P, EV_QKV, t.layer, Kind<kKind>::wide ? 0 : decode_qkv(P, t.idx).group); break;
    case OP_ATTN: n.ctr = ev_ctr(P, EV_ATTN, t.layer); break;  // (every task; a pair's last one merged the pair)
    case OP_OPROJ: n.ctr = ev_ctr(P, EV_O, t.layer); break;
    case OP_GATEUP: n.ctr = ev_ctr(P, EV_GU, t.layer, t.idx / P.gseg_gu * P.tile_gu / P.kseg); break;
    case OP_DOWN: n.ctr = ev_ctr(P, EV_IN, t.layer + 1); break;
    case OP_LM:
      n.ctr = ev_ctr(P, EV_LM, 0);
      n.ffam = fam_of(P, OP_LMFIN, -1); n.fop = OP_LMFIN; n.fidx = 0;
      break;
    case OP_ROUTE:
      n.ctr = ev_ctr(P, EV_ROUTE, moe_li(t.layer));
      n.ffam = fam_of(P, OP_MINDPTR, t.layer); n.fop = OP_MINDPTR; n.flayer = t.layer; n.fidx = 0;
      break;
    case OP_MINDPTR: n.ctr = ev_ctr(P, EV_MIDX, moe_li(t.layer)); break;
    case OP_EGU: n.ctr = ev_ctr(P, EV_MH, moe_li(t.layer), t.idx / P.nt_gu); break;  // the tile's event: set by the routing
    case OP_EDOWN: n.ctr = ev_ctr(P, EV_MY, moe_li(t.layer)); break;
    case OP_COMBINE:
      n.ctr = ev_ctr(P, EV_MCOMB, moe_li(t.layer));
      if (Kind<kKind>::moe_layer) { n.ffam = fam_of(P, OP_MFIN, -1); n.fop = OP_MFIN; n.fidx = 0; }
      break;
    default: break;
  }
  n.need_old = (n.ctr >= 0 && (n.ffam >= 0 || dyn)) ? 1 : 0;
  return n;
}

// Dynamic mode: the notifier whose decrement took a counter to zero pushes
// the tasks that wait on it.
template <int kKind>
__device__ void push_successors(const DevPlan& P, const StepParams& S, const Smem& sm, Control* ctl,
                                unsigned char* ws, const TaskDesc& t) {
  const int Hkv = P.n_kv_heads;
  switch (t.op) {
    case OP_NORM: push_range(P, S, ctl, ws, fam_of(P, OP_QKV, t.layer), 0, P.n_qkv_tiles); break;
    case OP_NORM2: push_range(P, S, ctl, ws, fam_of(P, OP_GATEUP, t.layer), 0, P.n_gutiles); break;
    case OP_NORMF: push_range(P, S, ctl, ws, fam_of(P, OP_LM, -1), 0, P.n_lm_tiles); break;
    case OP_QKV: {
      if (Kind<kKind>::wide) {  // (one event per layer: every kv head's tasks of a sequence in one range)
        for (int b = 0; b < S.B; ++b)
          push_range(P, S, ctl, ws, fam_of(P, OP_ATTN, t.layer), Hkv * sm.pre[b], Hkv * sm.nch[b]);
        break;
      }
      int g = decode_qkv(P, t.idx).group;
      for (int b = 0; b < S.B; ++b)
        push_range(P, S, ctl, ws, fam_of(P, OP_ATTN, t.layer), Hkv * sm.pre[b] + g * sm.nch[b], sm.nch[b]);
    } break;
    case OP_ATTN: push_range(P, S, ctl, ws, fam_of(P, OP_OPROJ, t.layer), 0, P.n_otiles); break;
    case OP_OPROJ:
      if (Kind<kKind>::moe_dec) push_range(P, S, ctl, ws, fam_of(P, OP_ROUTE, t.layer), 0, ceil_div(S.B, 8));
      else if (Kind<kKind>::wide) push_range(P, S, ctl, ws, fam_of(P, OP_NORM2, t.layer), 0, S.B);
      else push_range(P, S, ctl, ws, fam_of(P, OP_GATEUP, t.layer), 0, P.n_gutiles);
      break;
    case OP_GATEUP: {
      int kc = t.idx / P.gseg_gu * P.tile_gu / P.kseg;
      push_range(P, S, ctl, ws, fam_of(P, OP_DOWN, t.layer), kc * P.n_dtiles, P.n_dtiles);
    } break;
    case OP_DOWN:
      if (Kind<kKind>::wide) {
        if (t.layer + 1 < P.n_layers) push_range(P, S, ctl, ws, fam_of(P, OP_NORM, t.layer + 1), 0, S.B);
        else push_range(P, S, ctl, ws, fam_of(P, OP_NORMF, -1), 0, S.B);
      } else if (t.layer + 1 < P.n_layers) {
        push_range(P, S, ctl, ws, fam_of(P, OP_QKV, t.layer + 1), 0, P.n_qkv_tiles);
      } else {
        push_range(P, S, ctl, ws, fam_of(P, OP_LM, -1), 0, P.n_lm_tiles);
      }
      break;
    // MoE: exp_indptr decides how many GroupGEMM tiles run (data-dependent task triggering)
    case OP_MINDPTR: if constexpr (Kind<kKind>::moe) {
      const int n_tiles = __ldcg(reinterpret_cast<const int*>(moe_block(P, ws, t.layer) + P.off_mtile) + P.n_experts);
      push_range(P, S, ctl, ws, fam_of(P, OP_EGU, t.layer), 0, n_tiles * P.nt_gu);
    } break;
    case OP_EGU: if constexpr (Kind<kKind>::moe) {
      const int tile = t.idx / P.nt_gu;
      push_range(P, S, ctl, ws, fam_of(P, OP_EDOWN, t.layer), tile * P.nt_d, P.nt_d);
    } break;
    case OP_EDOWN: push_range(P, S, ctl, ws, fam_of(P, OP_COMBINE, t.layer), 0, ceil_div(S.B, 8)); break;
    case OP_COMBINE:  // MoE decoder: the layer's residual is complete
      if (Kind<kKind>::moe_dec) {
        if (Kind<kKind>::wide) {
          if (t.layer + 1 < P.n_layers) push_range(P, S, ctl, ws, fam_of(P, OP_NORM, t.layer + 1), 0, S.B);
          else push_range(P, S, ctl, ws, fam_of(P, OP_NORMF, -1), 0, S.B);
        } else if (t.layer + 1 < P.n_layers) {
          push_range(P, S, ctl, ws, fam_of(P, OP_QKV, t.layer + 1), 0, P.n_qkv_tiles);
        } else {
          push_range(P, S, ctl, ws, fam_of(P, OP_LM, -1), 0, P.n_lm_tiles);
        }
      }
      break;
    default: break;
  }
}

// Notifier warp: drains up to kFollowQ entries of the done queue at a time
// and decrements their counters with gpu-scope release operations (one lane
// per distinct counter; decrements of the same counter are combined into one
// add).  The release covers every output of the batch's tasks: the compute
// warps' writes precede the done barrier, the controller's queue hand-off
// and this warp's reads in CTA order, and release is cumulative.
template <int kKind>
__device__ void notifier(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws, Control* ctl,
                         int* counters) {
  const int lane = threadIdx.x & 31;
  const bool trace = Kind<kKind>::trace && S.trace != nullptr;
  int tail = 0;
  unsigned long long n_batches = 0, fence_ns = 0;
  for (;;) {
    int head = sm.dq_head;
    if (head == tail) {
      if (sm.notifier_stop || aborted(ctl)) break;
      __nanosleep(20);
      continue;
    }
    __threadfence_block();
    const int n = min(head - tail, kFollowQ);  // at most kFollowQ follow-ups per batch
    TaskDesc t;
    NotifyInfo ni;
    ni.ctr = -1; ni.need_old = 0; ni.ffam = -1;
    if (lane < n) {
      t = sm.doneq[(tail + lane) % kDoneQ];
      ni = notify_info<kKind>(P, S, sm, t);
    }
    __syncwarp();
    if (trace) n_batches++;
    // one atomic per distinct counter of the batch: the lowest lane of each
    // group subtracts the group's size; when the old value is needed, the
    // counter reached zero iff it equalled that size (the follow-up and the
    // successors depend on the counter only, so the leader's task stands for
    // the group)
    const int key = (lane < n && ni.ctr >= 0) ? ni.ctr : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const bool leader = key >= 0 && lane == __ffs(peers) - 1;
    const int cnt = __popc(peers);
    bool fired = false;
    if (leader) {
      if (ni.need_old) {
        int old;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(counters + key), "r"(-cnt) : "memory");
        if (old < cnt) record_error(ctl, MK_ERR_DEVICE_BOUNDS, t.fam, t.idx, key);
        fired = old == cnt;
      } else {
        asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(counters + key), "r"(-cnt) : "memory");
      }
    }
    if (fired && P.sched == MK_SCHED_DYNAMIC) push_successors<kKind>(P, S, sm, ctl, ws, t);
    if (lane < n && (t.op == OP_LMFIN || t.op == OP_MFIN) && P.sched == MK_SCHED_DYNAMIC)
      push_range(P, S, ctl, ws, -1, 0, P.n_sm);  // one END per CTA
    unsigned fb = __ballot_sync(0xffffffffu, fired && ni.ffam >= 0);
    if (fb) {
      int fh = sm.fq_head;
      int rank = __popc(fb & ((1u << lane) - 1));
      int room_ok = 1;
      if (lane == 0) {
        unsigned long long t0 = global_ns();
        while (fh + __popc(fb) - sm.fq_tail > kFollowQ) {
          if (aborted(ctl) || (long long)(global_ns() - t0) > P.spin_timeout_ns) { room_ok = 0; break; }
        }
        if (!room_ok) record_error(ctl, MK_ERR_DEVICE_TIMEOUT, -1, -1, -1);
      }
      room_ok = __shfl_sync(0xffffffffu, room_ok, 0);
      if (room_ok && fired && ni.ffam >= 0) {
        TaskDesc f;
        f.fam = ni.ffam; f.op = ni.fop; f.layer = ni.flayer; f.idx = ni.fidx;
        f.slot_ph = 0; f.nslots = 0; f.rec = 0; f.t_issue = 0;
        sm.followq[(fh + rank) % kFollowQ] = f;
      }
      __syncwarp();
      __threadfence_block();
      if (lane == 0 && room_ok) sm.fq_head = fh + __popc(fb);
    }
    if (trace && lane < n && t.rec > 0) {
      uint32_t* r = trace_rec(S, t.rec);
      if (r) r[TR_NOTIFIED] = (uint32_t)global_ns();
    }
    __syncwarp();
    __threadfence_block();
    tail += n;
    if (lane == 0) sm.dq_tail = tail;
  }
  if (trace && lane == 0) {
    uint32_t* h = trace_rec(S, 0);
    h[TRH_BATCHES] = (uint32_t)n_batches;
    h[TRH_NOTIFIED] = (uint32_t)tail;
    h[TRH_FENCE_NS] = (uint32_t)fence_ns;
  }
}

// ---------------------------------------------------------------- controller
// Releases tasks to the compute warps in order, at most two at a time: task k
// goes to cur[k & 1] and completes phase k >> 1 of go_bar[k & 1]; the warps
// report it done on done_bar[k & 1].  Per-buffer barriers keep every barrier
// at most one phase ahead of any warp.
template <int kKind>
__device__ void controller(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws, Control* ctl,
                           int* counters) {
  const int lane = threadIdx.x & 31;
  const long long tmo = P.spin_timeout_ns;
  const FamilyDesc* fams = reinterpret_cast<const FamilyDesc*>(ws + P.off_families);
  uint32_t fifo_seq = 0, nrel = 0, ndone = 0;
  TaskDesc held, t;
  TaskDesc inflight[2];
  inflight[0].fam = inflight[1].fam = -1;
  inflight[0].idx = inflight[1].idx = -1;
  inflight[0].rec = inflight[1].rec = 0;
  bool have_held = false;
  int known = -1;
  int released = 0;
  int dq_head = 0, fq_tail = 0;
  bool dead = false;
  const bool trace = Kind<kKind>::trace && S.trace != nullptr;
  int nrec = 0;
  uint32_t t_pop = 0, t_ready = 0;
  auto stamp = [&](int rec, int field, uint32_t v) {
    if (trace && lane == 0 && rec > 0) {
      uint32_t* r = trace_rec(S, rec);
      if (r) r[field] = v;
    }
  };
  // hand a finished task to the notifier (lane 0; the caller broadcasts)
  auto enqueue = [&](const TaskDesc& e) -> bool {
    unsigned long long t0 = global_ns();
    while (dq_head - sm.dq_tail >= kDoneQ) {
      if (aborted(ctl) || (long long)(global_ns() - t0) > tmo) return false;
    }
    sm.doneq[dq_head % kDoneQ] = e;
    __threadfence_block();
    sm.dq_head = dq_head + 1;
    return true;
  };
  // completion of the oldest in-flight task: block (wait) or test only
  auto complete_oldest = [&](bool block) -> int {  // 1 completed, 0 not yet, -1 dead
    int st = 0;
    if (lane == 0) {
      uint64_t* bar = &sm.done_bar[ndone & 1];
      const uint32_t par = (ndone >> 1) & 1;
      bool ok = block ? wait_mbar(bar, par, ctl, tmo, inflight[ndone & 1].fam, inflight[ndone & 1].idx)
                      : mbar_test(bar, par);
      if (ok) {
        const TaskDesc& e = inflight[ndone & 1];
        if (trace && e.rec > 0) { uint32_t* r = trace_rec(S, e.rec); if (r) r[TR_DONE] = (uint32_t)global_ns(); }
        st = enqueue(e) ? 1 : -1;
      } else {
        st = block ? -1 : 0;
      }
    }
    st = __shfl_sync(0xffffffffu, st, 0);
    if (st == 1) { ndone++; dq_head++; }
    return st;
  };
  // spin helper: notify finished tasks as they complete; report follow-ups
  auto idle_poll = [&]() -> int {  // 2 follow-up pending, -1 dead, 0 otherwise
    if (nrel != ndone && complete_oldest(false) < 0) return -1;
    return sm.fq_head != fq_tail ? 2 : 0;
  };
  auto release = [&](TaskDesc& r) {
    r.rec = (trace && r.op != OP_END) ? ++nrec : 0;
    inflight[nrel & 1] = r;
    if (lane == 0) {
      sm.cur[nrel & 1] = r;
      if (r.op != OP_END && S.task_counts && (P.debug_flags & MK_DEBUG_TASK_COUNTS))
        atomicAdd(&S.task_counts[fams[r.fam].debug_base + r.idx], 1u);
      if (r.op != OP_END && !is_followup(r.op)) sm.released = ++released;
      mbar_arrive(&sm.go_bar[nrel & 1]);
    }
    __syncwarp();
    nrel++;
    if (r.rec > 0) {
      stamp(r.rec, TR_FAM, (uint32_t)r.fam);
      stamp(r.rec, TR_IDX, (uint32_t)r.idx);
      stamp(r.rec, TR_POP, t_pop);
      stamp(r.rec, TR_READY, t_ready);
      stamp(r.rec, TR_GO, (uint32_t)global_ns());
    }
  };

  for (;;) {
    if (aborted(ctl)) { dead = true; break; }
    if (sm.fq_head != fq_tail) {
      __threadfence_block();
      t = sm.followq[fq_tail % kFollowQ];
      __syncwarp();
      fq_tail++;
      if (lane == 0) sm.fq_tail = fq_tail;
    } else if (have_held) {
      t = held;
      have_held = false;
    } else {
      int k = fifo_seq % kFifo;
      const uint32_t par = (fifo_seq / kFifo) & 1;
      int st = 0;  // 1 ready, 2 follow-up, 3 dead
      unsigned long long t0 = global_ns();
      for (int it = 0;; ++it) {
        int ready = 0;
        if (lane == 0) ready = mbar_test(&sm.fifo_full[k], par);
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (ready) { st = 1; break; }
        int ip = idle_poll();
        if (ip < 0) { st = 3; break; }
        if (ip == 2) { st = 2; break; }
        if ((it & 15) == 15) {
          int bad = 0;
          if (lane == 0) {
            if (aborted(ctl)) bad = 1;
            else if ((long long)(global_ns() - t0) > tmo) { record_error(ctl, MK_ERR_DEVICE_TIMEOUT, -1, -1, -1); bad = 1; }
          }
          if (__shfl_sync(0xffffffffu, bad, 0)) { st = 3; break; }
        }
      }
      if (st == 3) { dead = true; break; }
      if (st == 2) continue;
      __syncwarp();
      t = sm.fifo[k];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.fifo_empty[k]);
      fifo_seq++;
    }
    if (trace) t_pop = (uint32_t)global_ns();
    if (t.op == OP_END) {
      // quiesce: every task finished and notified, no follow-up left
      while (nrel != ndone) {
        if (complete_oldest(true) < 0) { dead = true; break; }
      }
      if (dead) break;
      int st = 0;  // 1 quiet, 2 follow-up, 3 dead
      if (lane == 0) {
        unsigned long long t0 = global_ns();
        for (;;) {
          if (sm.fq_head != fq_tail) { st = 2; break; }
          if (sm.dq_tail == dq_head) {
            __threadfence_block();
            st = sm.fq_head != fq_tail ? 2 : 1;
            break;
          }
          if (aborted(ctl)) { st = 3; break; }
          if ((long long)(global_ns() - t0) > tmo) { record_error(ctl, MK_ERR_DEVICE_TIMEOUT, -1, -1, -1); st = 3; break; }
        }
      }
      st = __shfl_sync(0xffffffffu, st, 0);
      if (st == 3) { dead = true; break; }
      if (st == 2) { held = t; have_held = true; continue; }
      release(t);
      break;
    }
    if (!is_followup(t.op)) {
      int w = wait_counter<kKind>(P, sm, t, S.B);
      if (w >= 0 && w != known) {
        int st = 0;  // 1 fired, 2 follow-up, 3 dead
        unsigned long long t0 = global_ns();
        for (int it = 0;; ++it) {
          int zero = 0;
          if (lane == 0) zero = ld_acquire(&counters[w]) == 0;
          if (__shfl_sync(0xffffffffu, zero, 0)) { st = 1; break; }
          // never sit on finished tasks while waiting: their notify may be
          // what this event needs
          int ip = idle_poll();
          if (ip < 0) { st = 3; break; }
          if (ip == 2) { st = 2; break; }
          if ((it & 15) == 15) {
            int bad = 0;
            if (lane == 0) {
              if (aborted(ctl)) bad = 1;
              else if ((long long)(global_ns() - t0) > tmo) { record_error(ctl, MK_ERR_DEVICE_TIMEOUT, t.fam, t.idx, w); bad = 1; }
            }
            if (__shfl_sync(0xffffffffu, bad, 0)) { st = 3; break; }
          }
        }
        if (st == 3) { dead = true; break; }
        if (st == 2) { held = t; have_held = true; continue; }
        known = w;
      }
    }
    if (trace) t_ready = (uint32_t)global_ns();
    // at most two tasks in flight
    if (nrel - ndone == 2 && complete_oldest(true) < 0) { dead = true; break; }
    release(t);
  }
  if (trace && lane == 0) trace_rec(S, 0)[TRH_RECORDS] = (uint32_t)nrec;
  if (dead) {
    // shut the compute warps down: let them finish what they hold, then END
    while (nrel != ndone) {
      int st = 0;
      if (lane == 0) st = wait_mbar(&sm.done_bar[ndone & 1], (ndone >> 1) & 1, ctl, tmo, -1, -1) ? 1 : 0;
      st = __shfl_sync(0xffffffffu, st, 0);
      ndone++;
      if (!st) break;
    }
    TaskDesc e;
    e.fam = -1; e.op = OP_END; e.layer = -1; e.idx = 0; e.slot_ph = 0; e.nslots = 0; e.rec = 0; e.t_issue = 0;
    if (lane == 0) {
      sm.cur[nrel & 1] = e;
      sm.released = 1 << 30;
      mbar_arrive(&sm.go_bar[nrel & 1]);
    }
    __syncwarp();
  }
  if (lane == 0) sm.notifier_stop = 1;
}

// ---------------------------------------------------------------- compute
// Ring slot i of a task (its first slot and phase in slot_ph).
__device__ __forceinline__ int task_slot(const TaskDesc& d, int i, int R, uint32_t& parity) {
  const int pos = (d.slot_ph & 0xffff) + i, wrap = pos / R;
  parity = ((uint32_t)d.slot_ph >> 16) ^ ((uint32_t)wrap & 1u);
  return pos - wrap * R;
}

struct GemvSpec {
  int kind;           // 0: RMSNorm(x) * gamma, 1: attention output, 2: SwiGLU segment
  int gamma_sel;      // kind 0: 0 attention-norm gain of `layer`, 1 FFN-norm gain, 2 final-norm gain
  int layer;
  int kc;             // K segment (kind 2)
  int K;              // columns
  bool parts;         // kind 0: add the previous layer's down-projection partials to x
  int tag;            // identifies the activation; unchanged tag = reuse the registers
  int rows;           // valid rows of the task
};

__device__ __forceinline__ bool gemv_spec(const DevPlan& P, const TaskDesc& d, GemvSpec& g) {
  g.gamma_sel = 0; g.layer = d.layer; g.kc = 0; g.parts = false; g.K = P.hidden;
  switch (d.op) {
    case OP_QKV:
      g.kind = 0; g.gamma_sel = 0; g.parts = d.layer > 0 && P.kind == MK_MODEL_DENSE; g.tag = d.layer * 64;
      g.rows = P.tile_qkv;
      return true;
    case OP_OPROJ:
      g.kind = 1; g.tag = d.layer * 64 + 1; g.rows = P.tile_o;
      return true;
    case OP_GATEUP:
      g.kind = 0; g.gamma_sel = 1; g.tag = d.layer * 64 + 2; g.rows = 2 * P.tile_gu;
      return true;
    case OP_DOWN:
      g.kind = 2; g.kc = d.idx / P.n_dtiles; g.K = P.kseg; g.tag = d.layer * 64 + 8 + g.kc; g.rows = P.tile_down;
      return true;
    case OP_LM:
      g.kind = 0; g.gamma_sel = 2; g.parts = P.kind == MK_MODEL_DENSE; g.tag = 60 * 64;
      g.rows = min(P.tile_lm, P.vocab - d.idx * P.tile_lm);
      return true;
    default:
      return false;
  }
}


// TMEM address of lane quadrant q (lanes 32q .. 32q + 31), column 0.
__device__ __forceinline__ uint32_t S_tmem_lane(uint32_t base, int q) { return base + ((uint32_t)(32 * q) << 16); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Activation rows 0..B-1 of a GEMV family into shared memory, bf16 (the
// tensor-core operand type), row b at sm.xa() + b * kActPitch: the compute
// warps load them once for the CTA (adding the previous layer's down
// partials to x when asked), reduce each row's sum of squares and apply the
// RMSNorm.  Rows go in groups of four (one round trip to L2 per group: every
// load of a group is issued before the first use).  Called by all compute
// warps for the same task (the tag sequence is the same for all warps).
// Thread t stages columns [8t, 8t + 8).
__device__ __forceinline__ void stage_act(const DevPlan& P, unsigned char* ws, Smem& sm, const GemvSpec& g, int B,
                                          uint32_t* trec, float* cap) {
  const LayerPtrs* layers = reinterpret_cast<const LayerPtrs*>(ws + P.off_layers);
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const int K = g.K;  // at most 8 * kComputeThreads
  const int c = ct * 8;
  const bool has = c < K;
  const float* src;
  size_t rstride;
  if (g.kind == 0) { src = reinterpret_cast<const float*>(ws + P.off_x); rstride = P.hidden; }
  else if (g.kind == 1) { src = reinterpret_cast<const float*>(ws + P.off_attn); rstride = (size_t)P.n_q_heads * P.head_dim; }
  else { src = reinterpret_cast<const float*>(ws + P.off_h) + (size_t)g.kc * P.kseg; rstride = P.ffn; }
  const float* dp = reinterpret_cast<const float*>(ws + P.off_dpart);
  const int nq = g.parts ? P.n_kc : 0;
  // (the gain stays raw until its first use, so its load overlaps the rows')
  uint4 graw = make_uint4(0u, 0u, 0u, 0u);
  if (has && g.kind == 0) {
    const void* gp = g.gamma_sel == 2 ? P.final_norm
                                      : (g.gamma_sel == 1 ? layers[g.layer].ffn_norm : layers[g.layer].attn_norm);
    graw = __ldg(reinterpret_cast<const uint4*>(gp) + c / 8);
  }
  for (int b0 = 0; b0 < B; b0 += 4) {
    float4 u[4], v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int b = b0 + i;
      u[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      v[i] = u[i];
      if (has && b < B) {
        float4 t[5][2];
        const float4* p4 = reinterpret_cast<const float4*>(src + (size_t)b * rstride + c);
        t[0][0] = __ldcg(p4);
        t[0][1] = __ldcg(p4 + 1);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          t[q + 1][0] = t[q + 1][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (q < nq) {
            const float4* d4 = reinterpret_cast<const float4*>(dp + ((size_t)q * P.max_batch + b) * P.hidden + c);
            t[q + 1][0] = __ldcg(d4);
            t[q + 1][1] = __ldcg(d4 + 1);
          }
        }
        auto sum5 = [&](int h) {
          float4 r;
          r.x = t[0][h].x + ((t[1][h].x + t[2][h].x) + (t[3][h].x + t[4][h].x));
          r.y = t[0][h].y + ((t[1][h].y + t[2][h].y) + (t[3][h].y + t[4][h].y));
          r.z = t[0][h].z + ((t[1][h].z + t[2][h].z) + (t[3][h].z + t[4][h].z));
          r.w = t[0][h].w + ((t[1][h].w + t[2][h].w) + (t[3][h].w + t[4][h].w));
          return r;
        };
        u[i] = sum5(0);
        v[i] = sum5(1);
        for (int q = 4; q < nq; ++q) {  // (more than four K segments)
          const float4* d4 = reinterpret_cast<const float4*>(dp + ((size_t)q * P.max_batch + b) * P.hidden + c);
          const float4 a4 = __ldcg(d4), b4 = __ldcg(d4 + 1);
          u[i].x += a4.x; u[i].y += a4.y; u[i].z += a4.z; u[i].w += a4.w;
          v[i].x += b4.x; v[i].y += b4.y; v[i].z += b4.z; v[i].w += b4.w;
        }
        if (cap) {  // debug capture of the residual row this staging reduced
          float4* c4 = reinterpret_cast<float4*>(cap + (size_t)b * K + c);
          c4[0] = u[i];
          c4[1] = v[i];
        }
      }
    }
    float inv[4] = {1.f, 1.f, 1.f, 1.f};
    if (g.kind == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (b0 + i < B) {
          float ss = u[i].x * u[i].x + u[i].y * u[i].y + u[i].z * u[i].z + u[i].w * u[i].w + v[i].x * v[i].x +
                     v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
          ss = warp_sum(ss);
          if (lane == 0) sm.red8[b0 + i][w] = ss;
        }
    }
    if (trec && lane == 0 && b0 == 0) trec[TR_LOADS] = (uint32_t)global_ns();
    // (the first group's barrier also means every warp is done with the previous activation)
    bar_sync(BAR_COMP, kComputeThreads);
    if (g.kind == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (b0 + i < B) {
          float tot = 0.f;
#pragma unroll
          for (int q = 0; q < kComputeWarps; ++q) tot += sm.red8[b0 + i][q];
          inv[i] = 1.0f / sqrtf(tot / (float)K + P.eps);
        }
    }
    if (has) {
      float gf[8];
      bf16x8_to_f32(graw, gf);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (b0 + i < B) {
          const float f[8] = {u[i].x, u[i].y, u[i].z, u[i].w, v[i].x, v[i].y, v[i].z, v[i].w};
          __align__(16) __nv_bfloat16 o[8], lo[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float a = g.kind == 0 ? f[j] * inv[i] * gf[j] : f[j];
            o[j] = __float2bfloat16_rn(a);
            lo[j] = __float2bfloat16_rn(a - __bfloat162float(o[j]));  // what bf16 left out
          }
          if (2 * B <= kMaxB) {  // split rows: row 2b holds row b in bf16, row 2b + 1 what bf16 left out
            *reinterpret_cast<uint4*>(&sm.xa()[2 * (b0 + i) * kActPitch + c]) = *reinterpret_cast<const uint4*>(o);
            *reinterpret_cast<uint4*>(&sm.xa()[(2 * (b0 + i) + 1) * kActPitch + c]) = *reinterpret_cast<const uint4*>(lo);
          } else {
            *reinterpret_cast<uint4*>(&sm.xa()[(b0 + i) * kActPitch + c]) = *reinterpret_cast<const uint4*>(o);
          }
        }
    }
  }
  bar_sync(BAR_COMP, kComputeThreads);  // the activation is complete
}

// Ring slot release.  A slot's empty barrier expects one arrival per use,
// made after every read of the slot: by the slot's only reader (a GEMV
// product warp), by one thread after a barrier of all readers (attention),
// or by tcgen05.commit once the MMAs reading it completed (GroupGEMM tiles).
// Nobody arrives before it has waited for the slot's data, so no arrival can
// land in another use's phase (task k+1's slots can be physical slots that
// task k still reads).

// ---- tensor-core tiles
// Warp-level bf16 MMA m16n8k16 with fp32 accumulation.  K is walked in
// windows of 32: lane (g = lane / 4, q = lane % 4) loads one 16-byte chunk,
// columns [8q, 8q + 8) of the window, of each row it needs, and the two MMAs
// of the window take its halves.  The logical-k -> column map is the same
// for both operands, so each MMA pairs matching columns and the two MMAs
// together cover the window's 32 columns once.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_window(float (&c)[4], const uint4& ua, const uint4& ub, const uint4& wb) {
  mma_16816(c, ua.x, ub.x, ua.y, ub.y, wb.x, wb.y);
  mma_16816(c, ua.z, ub.z, ua.w, ub.w, wb.z, wb.w);
}

// Epilogue item i of a GEMV task: batch row b and row (pair ops: pair) r of
// the task; items are B x RI with RI the rows (pairs) of the task.
struct GemvItem { int b, r; bool on; };
__device__ __forceinline__ GemvItem gemv_item(const OpGeo& geo, int B, int i) {
  const int RI = geo.rows_part;
  GemvItem it;
  it.b = i / RI;
  it.r = i - it.b * RI;
  it.on = it.b < B;
  return it;
}

// Epilogue operands that do not depend on the task's products, loaded before
// them so that their round trip to L2 overlaps the staging and the math: a
// QKV item takes (cos, sin) of the rotary table for its column; an
// O-projection item the residual terms of its column (x and up to four of
// the previous layer's down-projection partials).
struct EpiAhead { float a[5]; };
__device__ __forceinline__ void gemv_epilogue_ahead(const DevPlan& P, const Smem& sm, unsigned char* ws,
                                                    const TaskDesc& d, const GemvItem& it, EpiAhead& e) {
#pragma unroll
  for (int i = 0; i < 5; ++i) e.a[i] = 0.f;
  if (!it.on) return;
  if (d.op == OP_QKV) {
    const QkvTile q = decode_qkv(P, d.idx);
    if (q.kind != 2) {
      const float2 cs = __ldg(reinterpret_cast<const float2*>(ws + P.off_rope) + (size_t)sm.ctx[it.b] * 32 +
                              q.j0 + it.r);
      e.a[0] = cs.x;
      e.a[1] = cs.y;
    }
  } else if (d.op == OP_OPROJ) {
    const size_t col = (size_t)d.idx * P.tile_o + it.r;
    const float* dp = reinterpret_cast<const float*>(ws + P.off_dpart) + (size_t)it.b * P.hidden + col;
    e.a[0] = __ldcg(reinterpret_cast<const float*>(ws + P.off_x) + (size_t)it.b * P.hidden + col);
    if (d.layer > 0 && P.kind == MK_MODEL_DENSE)
#pragma unroll
      for (int kc = 0; kc < 4; ++kc)
        if (kc < P.n_kc) e.a[1 + kc] = __ldcg(dp + (size_t)kc * P.max_batch * P.hidden);
  }
}

// A GEMV task on tensor cores: Y[rows x B] = W[rows x K] . A[B x K]^T, W
// the task's rows (16, 32 or 64) in its ring slots (bf16, by column slice),
// A the staged activation rows.  The rows arrive in halves of at most 32 rows
// and 8 slots each (pair ops with 32 + 32 rows: the part-0 half, then the
// part-1 half); product warp w reads slot w of each half: every 16-row block
// of the half over columns [w cw, (w + 1) cw), with the activation rows as
// the MMA's n = 8 columns (column n reads row min(n, B - 1)).  It waits for
// that slot alone and releases it (its only reader) as soon as its products
// are done.  Each warp leaves its partial tile in sm.gred() ([w][column][64
// rows]); after a barrier, the threads sum the 8 partials of their items
// (batch row b, row or pair r; 256 items at a time) and run the op's
// epilogue; a last barrier frees the partial tiles for the next task.
__device__ __forceinline__ void gemv_task(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                                          unsigned char* ws, Control* ctl, const TaskDesc& d, const GemvSpec& g,
                                          int B, const EpiAhead& ea0, uint32_t* trec) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const OpGeo geo = sm.geo[d.op];
  const int R = P.ring_slots;
  const int s0 = d.slot_ph & 0xffff;
  const uint32_t p0 = (uint32_t)d.slot_ph >> 16;
  const int rows_total = (geo.pairs ? 2 : 1) * geo.rows_part;
  const int nh = rows_total > 32 ? 2 : 1;        // halves of 8 slots
  const int nrb = (rows_total > 32 ? 32 : rows_total) >> 4;  // 16-row blocks per half: 1 or 2
  const int g8 = lane >> 2, q = lane & 3;
  const int pitch = geo.cw * 2;  // bytes per row in a slot
  // 16-byte chunk (window win, lane chunk q) of slot row r: with cw >= 64 the
  // rows are 128-byte lines under the 128-byte swizzle (chunk c of line n at
  // c ^ (n & 7)), which puts the 8 rows a quarter-warp reads on distinct banks
  const bool swz = geo.cw >= 64;
  // activation rows staged: B, or 2B when 2B <= 8 (row 2b + 1 carries the
  // bf16 remainder of row b, so the products see ~16-bit activations; lane q
  // then holds batch row q's two halves in its two columns and adds them)
  const bool split = 2 * B <= kMaxB;
  const int ncol = split ? 2 * B : B;
  const uint4* px = reinterpret_cast<const uint4*>(&sm.xa()[min(g8, ncol - 1) * kActPitch + w * geo.cw]) + q;
  const int nwin = geo.cw >> 5;
  float* red = sm.gred(P.act_bytes);
  auto put = [&](int row, float x0, float x1) {  // partial tile: [w][column][64 rows]
    if (split) {
      if (q < B) red[((size_t)w * kMaxB + q) * 64 + row] = x0 + x1;
    } else if (2 * q < ncol) {
      float* e = red + ((size_t)w * kMaxB + 2 * q) * 64 + row;
      e[0] = x0;
      e[64] = x1;
    }
  };
  for (int h = 0; h < nh; ++h) {
    const int j = kGemvSlots * h + w;  // this warp's slot of the task
    const int wrap = (s0 + j) / R;
    const int sw = s0 + j - wrap * R;
    if (j >= R) {
      // The ring position also held slot j - R of this task.  A parity wait
      // on the full barrier cannot tell that use's phase from this one's, so
      // first wait until slot j - R has been released (the empty barrier's
      // phase for that use: it cannot move on before this warp releases slot
      // j); the full barrier is then at most one phase behind slot j.
      const int wrap_prev = (s0 + j - R) / R;
      wait_mbar(&sm.empty[sw], p0 ^ ((uint32_t)wrap_prev & 1u), ctl, P.spin_timeout_ns, d.fam, d.idx);
    }
    wait_mbar(&sm.full[sw], p0 ^ ((uint32_t)wrap & 1u), ctl, P.spin_timeout_ns, d.fam, d.idx);
    if (trec && lane == 0 && h == 0) {
      trec[TR_DATA] = (uint32_t)global_ns();
      trec[TR_ISSUE] = sm.slot_t[s0];
    }
    const unsigned char* slot = ring + (size_t)sw * P.slot_bytes;
    auto chunk = [&](int r, int win) -> const uint4* {
      const int o = r * pitch + (win * 4 + q) * 16;
      return reinterpret_cast<const uint4*>(slot + (swz ? (o ^ (((o >> 7) & 7) << 4)) : o));
    };
    float c0[2][4], c1[2][4];  // row blocks 0 and 1, two accumulators each
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) c0[u][i] = c1[u][i] = 0.f;
    // windows in pairs, alternating accumulators (16-byte chunks: 4 per window)
    if (nrb == 2) {
      for (int win = 0; win < nwin; win += 2) {
        const uint4 xb = px[win * 4];
        mma_window(c0[0], *chunk(g8, win), *chunk(g8 + 8, win), xb);
        mma_window(c1[0], *chunk(g8 + 16, win), *chunk(g8 + 24, win), xb);
        if (win + 1 < nwin) {
          const uint4 xb1 = px[win * 4 + 4];
          mma_window(c0[1], *chunk(g8, win + 1), *chunk(g8 + 8, win + 1), xb1);
          mma_window(c1[1], *chunk(g8 + 16, win + 1), *chunk(g8 + 24, win + 1), xb1);
        }
      }
    } else {
      for (int win = 0; win < nwin; win += 2) {
        mma_window(c0[0], *chunk(g8, win), *chunk(g8 + 8, win), px[win * 4]);
        if (win + 1 < nwin) mma_window(c0[1], *chunk(g8, win + 1), *chunk(g8 + 8, win + 1), px[win * 4 + 4]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[sw]);  // the slot's only reader
    // lane (g8, q) holds rows g8, g8 + 8 (+ 16 for block 1) of the half at
    // batch columns 2q, 2q + 1
    const int rh = 32 * h;
    put(rh + g8, c0[0][0] + c0[1][0], c0[0][1] + c0[1][1]);
    put(rh + g8 + 8, c0[0][2] + c0[1][2], c0[0][3] + c0[1][3]);
    if (nrb == 2) {
      put(rh + g8 + 16, c1[0][0] + c1[1][0], c1[0][1] + c1[1][1]);
      put(rh + g8 + 24, c1[0][2] + c1[1][2], c1[0][3] + c1[1][3]);
    }
  }
  if (trec && lane == 0) trec[TR_MATH] = (uint32_t)global_ns();
  bar_sync(BAR_COMP, kComputeThreads);
  if (trec && lane == 0) trec[TR_RED] = (uint32_t)global_ns();
  const int n_items = B * geo.rows_part;
  for (int i0 = 0; i0 < n_items; i0 += kComputeThreads) {
    // item (b, r); v0 = row r (pair ops: part 0 row r), v1 = part 1 row r
    const GemvItem it = gemv_item(geo, B, i0 + ct);
    EpiAhead ea;
    if (i0 == 0) ea = ea0;
    else gemv_epilogue_ahead(P, sm, ws, d, it, ea);
    const int b = it.b, r = it.r;
    const bool mine = it.on && (geo.pairs || d.op != OP_LM || d.idx * P.tile_lm + r < P.vocab);
    float v0 = 0.f, v1 = 0.f;
    if (mine) {
#pragma unroll
      for (int k = 0; k < kComputeWarps; ++k) v0 += red[(k * kMaxB + b) * 64 + r];
      if (geo.pairs)
#pragma unroll
        for (int k = 0; k < kComputeWarps; ++k) v1 += red[(k * kMaxB + b) * 64 + geo.rows_part + r];
    }
    const int H = P.hidden;
    switch (d.op) {
      case OP_QKV: {
        // RoPE on q and k (rotate-half pairs j, j + D/2), then q -> buffer, k/v -> cache
        if (!mine) break;
        QkvTile qt = decode_qkv(P, d.idx);
        const int pos = sm.ctx[b];
        const int j = qt.j0 + r;
        if (qt.kind == 2) {
          size_t row = (((size_t)d.layer * P.n_slots + sm.slot[b]) * P.n_kv_heads + qt.head) * P.max_ctx + pos;
          __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(P.v_cache) + row * P.head_dim;
          vc[j] = __float2bfloat16_rn(v0);
          vc[j + 32] = __float2bfloat16_rn(v1);
        } else {
          const float cs = ea.a[0], sn = ea.a[1];  // (cos, sin) of (pos, j), loaded before the products
          const float x0 = v0 * cs - v1 * sn, x1 = v1 * cs + v0 * sn;
          if (qt.kind == 0) {
            float* qb = reinterpret_cast<float*>(ws + P.off_q) + (size_t)b * P.n_q_heads * P.head_dim +
                        qt.head * P.head_dim;
            qb[j] = x0;
            qb[j + 32] = x1;
          } else {
            size_t row = (((size_t)d.layer * P.n_slots + sm.slot[b]) * P.n_kv_heads + qt.head) * P.max_ctx + pos;
            __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(P.k_cache) + row * P.head_dim;
            kc[j] = __float2bfloat16_rn(x0);
            kc[j + 32] = __float2bfloat16_rn(x1);
          }
        }
      } break;
      case OP_OPROJ: {
        // residual: x = (x + previous layer's down partials) + o W_o^T
        if (!mine) break;
        const size_t col = (size_t)d.idx * P.tile_o + r;
        float* x = reinterpret_cast<float*>(ws + P.off_x) + (size_t)b * H;
        float acc = ea.a[0];
        if (d.layer > 0 && P.kind == MK_MODEL_DENSE) {
          acc += (ea.a[1] + ea.a[2]) + (ea.a[3] + ea.a[4]);
          const float* dp = reinterpret_cast<const float*>(ws + P.off_dpart) + (size_t)b * H + col;
          for (int kc = 4; kc < P.n_kc; ++kc) acc += __ldcg(dp + (size_t)kc * P.max_batch * H);
        }
        x[col] = acc + v0;
      } break;
      case OP_GATEUP: {
        if (!mine) break;
        float* h = reinterpret_cast<float*>(ws + P.off_h) + (size_t)b * P.ffn + (size_t)d.idx * P.tile_gu + r;
        *h = v0 / (1.0f + expf(-v0)) * v1;
      } break;
      case OP_DOWN: {
        if (!mine) break;
        const int nt = d.idx - g.kc * P.n_dtiles;
        float* dpart = reinterpret_cast<float*>(ws + P.off_dpart) + ((size_t)g.kc * P.max_batch + b) * H +
                       (size_t)nt * P.tile_down + r;
        *dpart = v0;
      } break;
      case OP_LM: {
        // logits, then the warp's best (logit, id) key (the warp's items share
        // one batch row); published with an atomic max only when it beats what
        // this warp published before (order independent)
        const int row = d.idx * P.tile_lm + r;
        unsigned long long key = 0ull;
        if (mine) {
          if (S.logits) S.logits[(size_t)b * P.vocab + row] = v0;
          key = argmax_key(v0, row);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
          key = other > key ? other : key;
        }
        if (lane == 0 && it.on && key > sm.lm_seen[w][b]) {
          sm.lm_seen[w][b] = key;
          atomicMax(reinterpret_cast<unsigned long long*>(ws + P.off_lmbest) + b, key);
        }
      } break;
      default: break;
    }
  }
  if (trec && lane == 0) trec[TR_EPI] = (uint32_t)global_ns();
  bar_sync(BAR_COMP, kComputeThreads);  // the partial tiles are free for the next task
}

// wide batch: store v at column c of batch row b of an activation buffer with
// ld columns (its bf16 value, and with the split its bf16 remainder)
__device__ __forceinline__ void store_act(const DevPlan& P, __nv_bfloat16* buf, size_t ld, int b, size_t c, float v) {
  const __nv_bfloat16 hv = __float2bfloat16_rn(v);
  buf[(size_t)act_buf_row(P.act_split, b, 0) * ld + c] = hv;
  if (P.act_split) buf[(size_t)act_buf_row(P.act_split, b, 1) * ld + c] = __float2bfloat16_rn(v - __bfloat162float(hv));
}

// wide batch: accumulator columns of batch rows 8 g8 .. 8 g8 + 7 from TMEM
// address ta (value plus remainder products with the split)
__device__ __forceinline__ void acc_rows8(uint32_t ta, int split, int g8, float (&v)[8]) {
  if (split) {
    float r[8];
    tmem_ld8(ta + 16u * (uint32_t)g8, v);
    tmem_ld8(ta + 16u * (uint32_t)g8 + 8u, r);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += r[i];
  } else {
    tmem_ld8(ta + 8u * (uint32_t)g8, v);
  }
}

// ldmatrix: four 8x8 b16 matrices from shared memory; lane l gives the
// address of row l % 8 of matrix l / 8 (16 bytes), register m receives the
// matrix-m elements of the mma fragment layout (plain or transposed).
__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
// (x0, x1) as a bf16 pair (x0 in the low half): the values, and the remainders x - value
__device__ __forceinline__ uint32_t bf16_pair(float x0, float x1) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x0, x1);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&v);
  lo = bf16_pair(x0 - __low2float(v), x1 - __high2float(v));
}
// 16-byte chunk c of row r of a 64-column bf16 tile under the 128-byte swizzle
__device__ __forceinline__ int sw128_off(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// Merge of the attention partials of one (sequence, GQA group), run by the
// pair's last attention task to finish: the output of
// head h is sum_c e^(m_c - M) o_c / sum_c e^(m_c - M) l_c.  Warp pair
// (2h, 2h + 1) takes head h, 32 output columns each; a batch of up to 16
// chunks is loaded in one round trip (lane c: m and l of chunk c; every lane:
// its column of all the batch's chunk outputs), with an online rescale across
// batches.
__device__ __forceinline__ void merge_pair(const DevPlan& P, const Smem& sm, unsigned char* ws, int b, int g) {
  const int lane = threadIdx.x & 31, w = (threadIdx.x - kComputeBase) >> 5;
  const int Hkv = P.n_kv_heads, qpg = P.n_q_heads / Hkv, D = P.head_dim;
  const int h = w >> 1, dd = (w & 1) * 32 + lane;
  if (h >= qpg) return;
  const int nch = sm.nch[b];
  const size_t cs = (size_t)qpg * (D + 2);
  const float* part = reinterpret_cast<const float*>(ws + P.off_apart) + ((size_t)b * Hkv + g) * P.max_chunks * cs +
                      h * (D + 2);
  float M = -INFINITY, L = 0.f, O = 0.f;
  for (int c0 = 0; c0 < nch; c0 += 16) {
    const int n = min(16, nch - c0);
    const int c = c0 + lane;
    const bool in = lane < n;  // lane c - c0 of the batch
    const float mc = in ? __ldcg(part + c * cs + D) : -INFINITY;
    const float lc = in ? __ldcg(part + c * cs + D + 1) : 0.f;
    float ov[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) ov[q] = q < n ? __ldcg(part + (c0 + q) * cs + dd) : 0.f;
    float mb = mc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float Mn = fmaxf(M, mb);
    const float sc = expf(M - Mn);  // 0 on the first batch (M = -inf, Mn finite)
    const float e = in ? expf(mc - Mn) : 0.f;
    L = L * sc + warp_sum(lc * e);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < 16; ++q) acc[q & 3] = fmaf(ov[q], __shfl_sync(0xffffffffu, e, q), acc[q & 3]);
    O = O * sc + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
    M = Mn;
  }
  float* out = reinterpret_cast<float*>(ws + P.off_attn) + (size_t)b * P.n_q_heads * D + (size_t)(g * qpg + h) * D;
  out[dd] = O / L;
  if (P.wide)  // the O projection's B operand
    store_act(P, reinterpret_cast<__nv_bfloat16*>(ws + P.off_attn_bf), (size_t)P.n_q_heads * D, b,
              (size_t)(g * qpg + h) * D + dd, O / L);
}

// One task of split-KV decode attention for the qpg query heads of a GQA
// group: up to the step's split (sm.asplit) of consecutive 64-key chunks of one sequence, one ring
// slot each (K rows, then V rows, as 128-byte-swizzled TMA boxes); compute
// warp w takes chunks w, w + 8, ... of the task (flash-decoding partials:
// unnormalised output, running maximum, exp-sum).  A (sequence, kv head)
// whose chunks all fit one task writes its finished output here and skips
// the merge.  A warp computes the chunk's scores S = Q K^T and
// O += P V with bf16 warp MMAs (m16n8k16, fp32 accumulation): MMA row h
// carries head h's query (or probabilities) as bf16 values and row h + 8 the
// bf16 remainders, so that the products see about 16 significant bits and
// the two rows' accumulators add up in the same lane; the softmax in between
// is fp32 in registers (lane (g, q) holds head g's scores of keys 2q, 2q + 1
// of each 8-key tile).  The warps' partials are combined through shared
// memory at the end.  The new key (position ctx) is read from the cache in
// global memory and written over its row of the slot, whose copy may predate
// this step's append; the slot's rows past the last key are masked (scores)
// and zeroed (values).
__device__ __forceinline__ void task_attn(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                                       unsigned char* ws, Control* ctl, const TaskDesc& d, uint32_t* trec) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const int Hkv = P.n_kv_heads, qpg = P.n_q_heads / Hkv, CH = P.chunk;
  constexpr int D = 64;  // head_dim (the plan builder accepts 64 only)
  const AttnTask a = decode_attn(d.idx, S.B, Hkv, sm.nch, sm.pre);
  const int p = sm.ctx[a.b];
  const int c0 = a.c * sm.asplit, c1 = min(c0 + sm.asplit, ceil_div(p + 1, CH));
  const int g = lane >> 2, q4 = lane & 3;
  const bool hv = g < qpg;  // this lane's MMA row is a head of the group
  float m_run = -INFINITY, l_run = 0.f;
  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  // query fragments (scaled by 1/sqrt(64)): dims 16t + 2q, +1 and +8, +9 of head g
  uint32_t qa[4][4];
  if (c0 + w < c1) {
    const float* qrow = reinterpret_cast<const float*>(ws + P.off_q) + (size_t)a.b * P.n_q_heads * D +
                        (size_t)(a.g * qpg + (hv ? g : 0)) * D;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 x01 = hv ? __ldcg(reinterpret_cast<const float2*>(qrow + 16 * t + 2 * q4)) : make_float2(0.f, 0.f);
      const float2 x89 = hv ? __ldcg(reinterpret_cast<const float2*>(qrow + 16 * t + 2 * q4 + 8)) : make_float2(0.f, 0.f);
      split_pair(x01.x * 0.125f, x01.y * 0.125f, qa[t][0], qa[t][1]);
      split_pair(x89.x * 0.125f, x89.y * 0.125f, qa[t][2], qa[t][3]);
    }
  }
  // this warp's chunks c0 + w, c0 + w + 8, ... (online softmax across them)
  for (int cc = c0 + w; cc < c1; cc += kComputeWarps) {
    const int n_old = max(0, min(CH, p - cc * CH));
    const bool has_new = (p - cc * CH) < CH;
    const int n_keys = n_old + (has_new ? 1 : 0);
    uint4 knew = make_uint4(0, 0, 0, 0);
    if (has_new && lane < 16) {
      const size_t row = (((size_t)d.layer * P.n_slots + sm.slot[a.b]) * Hkv + a.g) * P.max_ctx + p;
      const unsigned char* src = reinterpret_cast<const unsigned char*>(lane < 8 ? P.k_cache : P.v_cache) + row * D * 2;
      knew = __ldcg(reinterpret_cast<const uint4*>(src) + (lane & 7));
    }
    if (trec && lane == 0 && cc == c0 + w) trec[TR_STAGED] = (uint32_t)global_ns();
    uint32_t par;
    const int R = P.ring_slots, i = cc - c0;
    const int slot = task_slot(d, i, R, par);
    if (i >= R) {
      // The ring position also held chunk i - R of this task.  A parity wait
      // on the full barrier cannot tell that use's phase from this one's, so
      // first wait until chunk i - R has been released (its warp processes
      // its chunks in increasing order, none waiting on a later chunk).
      uint32_t par_prev;
      task_slot(d, i - R, R, par_prev);
      wait_mbar(&sm.empty[slot], par_prev, ctl, P.spin_timeout_ns, d.fam, d.idx);
    }
    wait_mbar(&sm.full[slot], par, ctl, P.spin_timeout_ns, d.fam, d.idx);
    if (trec && lane == 0 && cc == c0 + w) trec[TR_DATA] = (uint32_t)global_ns();
    unsigned char* kb = ring + (size_t)slot * P.slot_bytes;
    unsigned char* vb = kb + (size_t)CH * D * 2;
    if (has_new) {
      // the appended key and value over their row; value rows past it zeroed
      if (lane < 16) *reinterpret_cast<uint4*>((lane < 8 ? kb : vb) + sw128_off(n_old, lane & 7)) = knew;
      for (int i = lane; i < (CH - 1 - n_old) * 8; i += 32)
        *reinterpret_cast<uint4*>(vb + sw128_off(n_old + 1 + (i >> 3), i & 7)) = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
    // scores: 8 key tiles x 4 dim steps
    float sc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
      const int r = 8 * j + (lane & 7);
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + sw128_off(r, 4 * tt + (lane >> 3)), b0, b1, b2, b3);
        mma_16816(sc[j], qa[2 * tt][0], qa[2 * tt][1], qa[2 * tt][2], qa[2 * tt][3], b0, b1);
        mma_16816(sc[j], qa[2 * tt + 1][0], qa[2 * tt + 1][1], qa[2 * tt + 1][2], qa[2 * tt + 1][3], b2, b3);
      }
    }
    // softmax of head g over the chunk, joined to the running state
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float v = (8 * j + 2 * q4 + e < n_keys) ? sc[j][e] + sc[j][2 + e] : -INFINITY;
        sc[j][e] = v;
        mx = fmaxf(mx, v);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);  // finite: the chunk has a key
    const float scale = hv ? expf(m_run - m_new) : 0.f;
    float ls = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float pv = hv ? expf(sc[j][e] - m_new) : 0.f;
        sc[j][e] = pv;
        ls += pv;
      }
    ls += __shfl_xor_sync(0xffffffffu, ls, 1);
    ls += __shfl_xor_sync(0xffffffffu, ls, 2);
    l_run = l_run * scale + ls;
    m_run = m_new;
#pragma unroll
    for (int j = 0; j < 8; ++j) { o[j][0] *= scale; o[j][1] *= scale; o[j][2] *= scale; o[j][3] *= scale; }
    // O += P V: 4 key steps (key tiles 2t, 2t + 1) x 8 dim tiles
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t pa0, pa1, pa2, pa3;
      split_pair(sc[2 * t][0], sc[2 * t][1], pa0, pa1);
      split_pair(sc[2 * t + 1][0], sc[2 * t + 1][1], pa2, pa3);
      const int r = 16 * t + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + sw128_off(r, 2 * jj + (lane >> 4)), b0, b1, b2, b3);
        mma_16816(o[2 * jj], pa0, pa1, pa2, pa3, b0, b1);
        mma_16816(o[2 * jj + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
    }
    // (generic writes to the slot precede the producer's next TMA copy into it)
    if (has_new) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
  }
  if (trec && lane == 0) trec[TR_MATH] = (uint32_t)global_ns();
  // the warps' partials (value and remainder rows added), maxima and sums
  float* ob = sm.xs();
  if (hv) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float2*>(ob + (w * 4 + g) * D + 8 * j + 2 * q4) = make_float2(o[j][0] + o[j][2], o[j][1] + o[j][3]);
    if (q4 == 0) { sm.alsum[w][g] = l_run; sm.amax[w][g] = m_run; }
  }
  bar_sync(BAR_COMP, kComputeThreads);
  if (ct < qpg * D) {
    const int h = ct >> 6, dd = ct & 63;  // h is uniform in a warp
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kComputeWarps; ++ww) M = fmaxf(M, sm.amax[ww][h]);
    float O = 0.f, Ls = 0.f;
#pragma unroll
    for (int ww = 0; ww < kComputeWarps; ++ww) {
      const float mw = sm.amax[ww][h];
      if (mw != -INFINITY) {  // (warps without a chunk)
        const float f = expf(mw - M);
        O = fmaf(ob[(ww * 4 + h) * D + dd], f, O);
        Ls = fmaf(sm.alsum[ww][h], f, Ls);
      }
    }
    if (sm.nch[a.b] == 1) {
      // the pair's only task: the finished output (the merge of one partial)
      const size_t oc = (size_t)(a.g * qpg + h) * D + dd;
      reinterpret_cast<float*>(ws + P.off_attn)[(size_t)a.b * P.n_q_heads * D + oc] = O / Ls;
      if (P.wide) store_act(P, reinterpret_cast<__nv_bfloat16*>(ws + P.off_attn_bf), (size_t)P.n_q_heads * D, a.b, oc, O / Ls);
    } else {
      float* part = reinterpret_cast<float*>(ws + P.off_apart) +
                    (((size_t)a.b * Hkv + a.g) * P.max_chunks + a.c) * (size_t)(qpg * (D + 2)) + h * (D + 2);
      part[dd] = O;
      if (dd == 0) {
        part[D] = M;
        part[D + 1] = Ls;
      }
    }
  }
  if (sm.nch[a.b] > 1) {
    // the pair's tasks count in after writing their partials; the last one
    // to count in merges them (the same arithmetic whichever task that is).
    // The barrier orders every warp's partial stores before thread 0's fence,
    // which releases them with the count (as at the grid barrier).
    bar_sync(BAR_COMP, kComputeThreads);
    if (ct == 0) {
      int* cnt = reinterpret_cast<int*>(ws + P.off_actr) + a.b * Hkv + a.g;
      __threadfence();
      const int old = atomicAdd(cnt, 1);
      __threadfence();
      sm.attn_last = old == sm.nch[a.b] - 1;
      if (old == sm.nch[a.b] - 1) *cnt = 0;  // (no other task of this pair counts in again this layer)
    }
    bar_sync(BAR_COMP, kComputeThreads);
    if (sm.attn_last) merge_pair(P, sm, ws, a.b, a.g);
  }
  // every warp has read the partials before any of them writes the staging
  // buffer again (the next task may start without a barrier of its own)
  bar_sync(BAR_COMP, kComputeThreads);
  if (trec && lane == 0) trec[TR_RED] = (uint32_t)global_ns();
}


// ---------------------------------------------------------------- wide batch
// (max_batch > 8.)  The normalised activations are materialised in bf16 by
// NORM tasks, and every projection is a tcgen05 GEMM task: 128 weight rows
// (the MMA's M) x the batch (N = B rounded up to 16) over K in 64-column
// chunks.  The weight chunks stream through the ring from the producer, ahead
// of the task's event; the activation chunks are loaded by the MMA-issuing
// thread itself, after the event fired (the controller released the task),
// into kBStages stages of the staging buffer.

// NORM / NORM2 / NORMF (wide batch), batch row d.idx, all compute threads:
// the row's residual (x plus the previous layer's down partials, summed in a
// fixed order; kept in x by NORM) and its RMSNorm * gain as the GEMM tasks'
// bf16 activation row (value, and remainder with the split).  Thread t takes
// columns [8t, 8t + 8): every load of the row is issued before the first use.
__device__ __forceinline__ void task_norm(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws,
                                          const TaskDesc& d) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const int b = d.idx, H = P.hidden, c = 8 * ct;
  const bool on = c < H;
  const LayerPtrs* layers = reinterpret_cast<const LayerPtrs*>(ws + P.off_layers);
  const int lx = d.op == OP_NORMF ? P.n_layers : d.layer;
  const bool parts = P.kind == MK_MODEL_DENSE && d.op != OP_NORM2 && lx > 0;  // (an MoE decoder's x is complete)
  const void* gp = d.op == OP_NORM ? layers[d.layer].attn_norm : d.op == OP_NORM2 ? layers[d.layer].ffn_norm
                                                                                   : P.final_norm;
  float* x = reinterpret_cast<float*>(ws + P.off_x) + (size_t)b * H;
  const float* dp = reinterpret_cast<const float*>(ws + P.off_dpart) + (size_t)b * H;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), e = a;
  float ss = 0.f;
  if (on) {
    a = __ldcg(reinterpret_cast<const float4*>(x + c));
    e = __ldcg(reinterpret_cast<const float4*>(x + c) + 1);
    if (parts) {
      float4 pa[kMaxKc], pe[kMaxKc];
#pragma unroll
      for (int kc = 0; kc < kMaxKc; ++kc)
        if (kc < P.n_kc) {
          const float4* d4 = reinterpret_cast<const float4*>(dp + (size_t)kc * P.max_batch * H + c);
          pa[kc] = __ldcg(d4);
          pe[kc] = __ldcg(d4 + 1);
        }
#pragma unroll
      for (int kc = 0; kc < kMaxKc; ++kc)
        if (kc < P.n_kc) {
          a.x += pa[kc].x; a.y += pa[kc].y; a.z += pa[kc].z; a.w += pa[kc].w;
          e.x += pe[kc].x; e.y += pe[kc].y; e.z += pe[kc].z; e.w += pe[kc].w;
        }
      if (d.op == OP_NORM) {
        reinterpret_cast<float4*>(x + c)[0] = a;
        reinterpret_cast<float4*>(x + c)[1] = e;
      }
    }
    // debug capture: the residual after layer lx - 1 (what NORM and NORMF reduce)
    if (S.cap_resid && lx > 0 && d.op != OP_NORM2) {
      float4* c4 = reinterpret_cast<float4*>(S.cap_resid + ((size_t)(lx - 1) * S.B + b) * H + c);
      c4[0] = a;
      c4[1] = e;
    }
    ss = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + e.x * e.x + e.y * e.y + e.z * e.z + e.w * e.w;
  }
  ss = warp_sum(ss);
  if (lane == 0) sm.red8[0][w] = ss;
  bar_sync(BAR_COMP, kComputeThreads);
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kComputeWarps; ++k) tot += sm.red8[0][k];
  const float inv = 1.0f / sqrtf(tot / (float)H + P.eps);
  if (on) {
    float gf[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(gp) + c / 8), gf);
    const float v[8] = {a.x, a.y, a.z, a.w, e.x, e.y, e.z, e.w};
    __align__(16) __nv_bfloat16 o[8], rm[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float y = v[j] * inv * gf[j];
      o[j] = __float2bfloat16_rn(y);
      rm[j] = __float2bfloat16_rn(y - __bfloat162float(o[j]));
    }
    __nv_bfloat16* xn = reinterpret_cast<__nv_bfloat16*>(ws + P.off_xn);
    *reinterpret_cast<uint4*>(xn + (size_t)act_buf_row(P.act_split, b, 0) * H + c) = *reinterpret_cast<const uint4*>(o);
    if (P.act_split)
      *reinterpret_cast<uint4*>(xn + (size_t)act_buf_row(P.act_split, b, 1) * H + c) = *reinterpret_cast<const uint4*>(rm);
  }
  bar_sync(BAR_COMP, kComputeThreads);  // every warp has read the sums before the next task writes them
}

// MMA issue of a wide-batch GEMM task (one thread): per chunk c the task's
// weight slots (parts of them) from the ring and activation chunk c (all buffer
// rows x 64 columns, columns x0 + 64c of the activation buffer) from stage
// (bq + c) % kBStages of the staging buffer; the chunk for c + kBStages - 1
// is loaded once the MMAs of chunk c - 1 released its stage.
__device__ __forceinline__ void gemm_issue_wide(const DevPlan& P, Smem& sm, unsigned char* ring, Control* ctl,
                                                const TaskDesc& d, const void* bmap, int x0, int nk, int parts,
                                                int N, uint32_t& bq, uint32_t* trec) {
  const int R = P.ring_slots;
  const uint32_t idesc = umma_idesc_bf16(kWideRows, N);
  const uint32_t tm = sm.tmem_base;
  const uint32_t bbytes = (uint32_t)act_buf_rows(P.act_split, P.act_rows) * 128u;
  unsigned char* stages = sm.stage();
  const uint32_t u0 = bq;
  auto load_b = [&](int c) {
    const uint32_t u = u0 + (uint32_t)c;
    const int st = (int)(u % kBStages);
    if (u >= kBStages) wait_local(&sm.bempty[st], ((u / kBStages) - 1) & 1u, P.spin_timeout_ns);
    mbar_arrive_expect_tx(&sm.bfull[st], bbytes);
    tma_load_2d(stages + (size_t)st * bbytes, bmap, x0 + c * 64, 0, &sm.bfull[st]);
  };
  // the activation was written by other SMs' generic stores, ordered before
  // this thread by the task's event (the controller's acquire, then the
  // release to the compute warps); order that view before the TMA reads
  fence_proxy_async_global();
  for (int c = 0; c < min(kBStages - 1, nk); ++c) load_b(c);
  for (int c = 0; c < nk; ++c) {
    if (c + kBStages - 1 < nk) load_b(c + kBStages - 1);
    int sl[2];
    for (int q = 0; q < parts; ++q) {
      uint32_t par;
      sl[q] = task_slot(d, parts * c + q, R, par);
      wait_mbar(&sm.full[sl[q]], par, ctl, P.spin_timeout_ns, d.fam, d.idx);
    }
    if (trec && c == 0) { trec[TR_DATA] = (uint32_t)global_ns(); trec[TR_ISSUE] = sm.slot_t[d.slot_ph & 0xffff]; }
    const uint32_t u = u0 + (uint32_t)c;
    const int st = (int)(u % kBStages);
    wait_mbar(&sm.bfull[st], (u / kBStages) & 1u, ctl, P.spin_timeout_ns, d.fam, d.idx);
    if (trec && c == 0) trec[TR_LOADS] = (uint32_t)global_ns();
    tc_fence_after();
    const uint64_t b = umma_desc_sw128(stages + (size_t)st * bbytes);
    for (int q = 0; q < parts; ++q) {
      const uint64_t a = umma_desc_sw128(ring + (size_t)sl[q] * P.slot_bytes);
#pragma unroll
      for (int k = 0; k < 4; ++k) umma_bf16(tm + 128u * q, a + 2u * k, b + 2u * k, idesc, (c | k) ? 1u : 0u);
    }
    for (int q = 0; q < parts; ++q) umma_commit(&sm.empty[sl[q]]);
    umma_commit(&sm.bempty[st]);
  }
  bq = u0 + (uint32_t)nk;
  umma_commit(&sm.acc_bar);
  if (trec) trec[TR_STAGED] = (uint32_t)global_ns();  // (the last MMA issued)
}

// A wide-batch GEMM task: QKV (+ RoPE, KV append), O projection (+ residual),
// gate/up (+ SwiGLU), down (K segment partial) or LM head (+ logits and
// running argmax).  Lane quadrant q of the accumulator = weight rows 32q ..
// 32q + 31 of the tile; the two warps of a quadrant split the batch columns.
__device__ __forceinline__ void task_gemm_wide(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                                               unsigned char* ws, Control* ctl, const TaskDesc& d, uint32_t& tc_n,
                                               uint32_t& bq, uint32_t* trec) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const int B = S.B, H = P.hidden, D = P.head_dim;
  const int N = P.act_split ? 16 * ceil_div(B, 8) : ceil_div(B, 16) * 16;  // MMA N (see act_buf_row)
  const int sp = P.act_split;
  const unsigned char* gmaps = ws + P.off_tmap + (size_t)P.n_layers * kTmapPerLayer * kTmapBytes;
  const void* xn_map = gmaps + (size_t)TMG_XN * kTmapBytes;
  // QKV, O and gate/up: K segment seg of tile idx / gseg (split K)
  const int gseg = d.op == OP_QKV ? P.gseg_qkv : d.op == OP_OPROJ ? P.gseg_o : d.op == OP_GATEUP ? P.gseg_gu : 1;
  const int tile = d.idx / gseg, seg = d.idx - tile * gseg;
  const int K = d.op == OP_OPROJ ? P.n_q_heads * D : H;
  int x0 = seg * (K / gseg), nk = K / gseg / 64, parts = 1;
  const void* bmap = xn_map;
  if (d.op == OP_OPROJ) bmap = gmaps + (size_t)TMG_ATTN * kTmapBytes;
  if (d.op == OP_GATEUP) parts = 2;
  if (d.op == OP_DOWN) {
    bmap = gmaps + (size_t)TMG_H * kTmapBytes;
    x0 = (d.idx / P.n_dtiles) * P.kseg;
    nk = P.kseg / 64;
  }
  if (w == 0) {
    if (lane == 0) gemm_issue_wide(P, sm, ring, ctl, d, bmap, x0, nk, parts, N, bq, trec);
    __syncwarp();
  }
  wait_local(&sm.acc_bar, tc_n & 1u, P.spin_timeout_ns);
  tc_n++;
  tc_fence_after();
  if (trec && lane == 0) trec[TR_MATH] = (uint32_t)global_ns();
  const int q = (threadIdx.x >> 5) & 3;  // TMEM lane quadrant = weight rows 32q .. 32q + 31
  const int r = 32 * q + lane;           // this lane's row of the tile
  const uint32_t ta = S_tmem_lane(sm.tmem_base, q);
  const int ng = ceil_div(ceil_div(B, 8), 2);  // groups of 8 batch rows per warpgroup
  const int gb0 = (w >> 2) * ng, gb1 = min(gb0 + ng, ceil_div(B, 8));  // this warp's groups
  // split K: every segment's task writes its partial tile (value + remainder
  // products added) and counts in; the last one to count in sums the
  // partials in segment order (the same order whichever task is last) and
  // runs the tile's epilogue, the others stop here
  float* gpart = reinterpret_cast<float*>(ws + P.off_gpart);
  auto gp_at = [&](int sg, int part, int g8) -> float* {
    return gpart + ((((size_t)tile * gseg + sg) * parts + part) * kWideRows + r) * P.act_rows + 8 * g8;
  };
  bool run_epi = true;
  if (gseg > 1) {
    for (int part = 0; part < parts; ++part)
      for (int g8 = gb0; g8 < gb1; ++g8) {
        float v[8];
        acc_rows8(ta + 128u * (uint32_t)part, sp, g8, v);
        float4* dst = reinterpret_cast<float4*>(gp_at(seg, part, g8));
        __stcg(dst, make_float4(v[0], v[1], v[2], v[3]));
        __stcg(dst + 1, make_float4(v[4], v[5], v[6], v[7]));
      }
    __threadfence();
    tc_fence_before();
    bar_sync(BAR_COMP, kComputeThreads);
    if (ct == 0) {
      int* ctr = reinterpret_cast<int*>(ws + P.off_gctr) + (d.op == OP_QKV ? 0 : d.op == OP_OPROJ ? 1 : 2) * kGctrPerOp + tile;
      const int old = atomicAdd(ctr, 1);
      __threadfence();
      sm.gemm_last = old == gseg - 1;
      if (old == gseg - 1) *ctr = 0;  // (no other task of this tile counts in again in this step)
    }
    bar_sync(BAR_COMP, kComputeThreads);
    run_epi = sm.gemm_last != 0;
  }
  // the tile's values at this lane's row for batch rows 8 g8 .. 8 g8 + 7
  // (part: gate 0 / up 1): from TMEM, or (split K) the segments' partials
  // summed in segment order (their loads issued together)
  auto rows8 = [&](int part, int g8, float (&v)[8]) {
    if (gseg == 1) {
      acc_rows8(ta + 128u * (uint32_t)part, sp, g8, v);
      return;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    for (int sg = 0; sg < gseg; ++sg) {
      const float4* src = reinterpret_cast<const float4*>(gp_at(sg, part, g8));
      const float4 a = __ldcg(src), b = __ldcg(src + 1);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w; v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
  };
  if (run_epi) switch (d.op) {
    case OP_QKV: {
      // a tile is two heads (q, k or v rows); rotate-half pairs (j, j + 32)
      // of a head sit in quadrants (0, 1) and (2, 3): the odd quadrants hand
      // their values over through the staging buffer
      const int nq = P.n_q_heads * D / kWideRows, nkv = P.n_kv_heads * D / kWideRows;
      const int kind = tile < nq ? 0 : tile < nq + nkv ? 1 : 2;
      const int h0 = 2 * (tile - (kind == 0 ? 0 : kind == 1 ? nq : nq + nkv));
      float* xch = sm.xs();  // [64][act_rows]
      if (q & 1)
        for (int g8 = gb0; g8 < gb1; ++g8) {
          float v[8];
          rows8(0, g8, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) xch[((q >> 1) * 32 + lane) * P.act_rows + 8 * g8 + i] = v[i];
        }
      tc_fence_before();
      bar_sync(BAR_COMP, kComputeThreads);
      if (!(q & 1)) {
        const int hh = h0 + (q >> 1), j = lane;
        for (int g8 = gb0; g8 < gb1; ++g8) {
          const int c8 = 8 * g8;
          float2 cs[8];  // (cos, sin) of (position, j): read-only, loaded ahead of the group's stores
#pragma unroll
          for (int i = 0; i < 8; ++i)
            cs[i] = (kind != 2 && c8 + i < B)
                        ? __ldg(reinterpret_cast<const float2*>(ws + P.off_rope) + (size_t)sm.ctx[c8 + i] * 32 + j)
                        : make_float2(1.f, 0.f);
          float v[8];
          rows8(0, g8, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int b = c8 + i;
            if (b >= B) break;
            const float v0 = v[i], v1 = xch[((q >> 1) * 32 + lane) * P.act_rows + b];
            const int pos = sm.ctx[b];
            if (kind == 2) {
              const size_t row = (((size_t)d.layer * P.n_slots + sm.slot[b]) * P.n_kv_heads + hh) * P.max_ctx + pos;
              __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(P.v_cache) + row * D;
              vc[j] = __float2bfloat16_rn(v0);
              vc[j + 32] = __float2bfloat16_rn(v1);
            } else {
              const float x0r = v0 * cs[i].x - v1 * cs[i].y, x1r = v1 * cs[i].x + v0 * cs[i].y;
              if (kind == 0) {
                float* qb = reinterpret_cast<float*>(ws + P.off_q) + (size_t)b * P.n_q_heads * D + hh * D;
                qb[j] = x0r;
                qb[j + 32] = x1r;
              } else {
                const size_t row = (((size_t)d.layer * P.n_slots + sm.slot[b]) * P.n_kv_heads + hh) * P.max_ctx + pos;
                __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(P.k_cache) + row * D;
                kc[j] = __float2bfloat16_rn(x0r);
                kc[j + 32] = __float2bfloat16_rn(x1r);
              }
            }
          }
        }
      }
    } break;
    case OP_OPROJ: {
      // residual: x += o W_o^T, one fire-and-forget add per element (the
      // tile's only writer, so the sum is x + o exactly as a load and store)
      float* x = reinterpret_cast<float*>(ws + P.off_x);
      const int col = tile * kWideRows + r;
      for (int g8 = gb0; g8 < gb1; ++g8) {
        float v[8];
        rows8(0, g8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (8 * g8 + i < B) atomicAdd(x + (size_t)(8 * g8 + i) * H + col, v[i]);
      }
    } break;
    case OP_GATEUP: {
      __nv_bfloat16* hb = reinterpret_cast<__nv_bfloat16*>(ws + P.off_h_bf);
      const int col = tile * kWideRows + r;
      for (int g8 = gb0; g8 < gb1; ++g8) {
        const int c8 = 8 * g8;
        float g[8], u[8];
        rows8(0, g8, g);
        rows8(1, g8, u);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (c8 + i < B) store_act(P, hb, P.ffn, c8 + i, col, g[i] / (1.0f + expf(-g[i])) * u[i]);
      }
    } break;
    case OP_DOWN: {
      const int kc = d.idx / P.n_dtiles, col = (d.idx - kc * P.n_dtiles) * kWideRows + r;
      float* dp = reinterpret_cast<float*>(ws + P.off_dpart) + (size_t)kc * P.max_batch * H;
      for (int g8 = gb0; g8 < gb1; ++g8) {
        const int c8 = 8 * g8;
        float v[8];
        rows8(0, g8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (c8 + i < B) dp[(size_t)(c8 + i) * H + col] = v[i];
      }
    } break;
    case OP_LM: {
      // logits of vocabulary row `row`; per batch column the warp's best
      // (logit, id) key joins this CTA's running best in shared memory; after
      // the task, a column's key is published with one global atomic max
      // when it beats what this CTA published before (order independent)
      const int row = d.idx * kWideRows + r;
      const bool in = row < P.vocab;
      for (int g8 = gb0; g8 < gb1; ++g8) {
        const int c8 = 8 * g8;
        float v[8];
        rows8(0, g8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int b = c8 + i;
          if (b >= B) break;
          if (S.logits && in) S.logits[(size_t)b * P.vocab + row] = v[i];
          unsigned long long key = in ? argmax_key(v[i], row) : 0ull;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
            key = other > key ? other : key;
          }
          if (lane == 0) atomicMax(&sm.lm_cta[b], key);
        }
      }
      tc_fence_before();
      bar_sync(BAR_COMP, kComputeThreads);
      unsigned long long* best = reinterpret_cast<unsigned long long*>(ws + P.off_lmbest);
      for (int b = ct; b < B; b += kComputeThreads)
        if (sm.lm_cta[b] > sm.lm_pub[b]) {
          sm.lm_pub[b] = sm.lm_cta[b];
          atomicMax(best + b, sm.lm_cta[b]);
        }
    } break;
    default: break;
  }
  if (trec && lane == 0) trec[TR_EPI] = (uint32_t)global_ns();
  tc_fence_before();
  bar_sync(BAR_COMP, kComputeThreads);  // the accumulator and the staging buffer are free for the next task
}

// ---------------------------------------------------------------- MoE layer
// (The MoE task bodies are compiled into the MoE instances of the kernel only:
// see megakernel<kKind>.)
// Mixture-of-experts FFN on T tokens ("Event Tensor: A Unified Abstraction for
// Compiling Dynamic Megakernel", section "Core method": data-dependent event
// update and data-dependent task triggering).  Rows of the grouped problem
// are the (token, slot) pairs; expert e owns rows [indptr[e], indptr[e+1]).

// ROUTE: tokens 8*idx .. 8*idx+7.  Phase 1: warp w computes the router
// logits of experts w, w+8, ... for the 8 tokens, each in one fixed order
// (lane l sums its products over hidden index 256*i + 8*l + j, i outer, j
// inner, from +0; then an xor butterfly 16, 8, 4, 2, 1; then the bias), so
// that the top-k is exact.  Phase 2: warp w takes token w: top-k by logit
// (ties -> lower expert), softmax over the selected logits, and one
// histogram atomic per selection whose old value is the pair's rank inside
// its expert's rows.
__device__ __forceinline__ void task_route(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws,
                                           const TaskDesc& d) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const int E = P.n_experts, K = P.top_k, H = P.hidden, T = S.B, nblk = H >> 8;
  unsigned char* mb = moe_block(P, ws, d.layer);
  const MoeW mw = moe_weights(P, reinterpret_cast<const LayerPtrs*>(ws + P.off_layers), d.layer);
  const bool dec = P.kind == MK_MODEL_MOE_DECODER;
  __nv_bfloat16* xhat = reinterpret_cast<__nv_bfloat16*>(mb + P.off_mxhat);
  float* lg = sm.xs();  // [8][64] logits of this task's tokens
  // this task's token rows, bf16 [8][H] after the logits: read by every warp
  // for every expert (the staging buffer holds route_stage_bytes(H))
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<unsigned char*>(lg) + kRouteLogitBytes);
  bar_sync(BAR_COMP, kComputeThreads);  // the staging buffer is free
  {
    const int t = d.idx * 8 + w;
    if (t < T && dec) {
      // the layer's FFN input: RMSNorm(x) * ffn_norm of each token's residual row, in bf16
      const float* xr32 = reinterpret_cast<const float*>(ws + P.off_x) + (size_t)t * H;
      const uint4* gam = reinterpret_cast<const uint4*>(reinterpret_cast<const LayerPtrs*>(ws + P.off_layers)[d.layer].ffn_norm);
      float v[kMaxBlk][8];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxBlk; ++i)
        if (i < nblk) {
          const float4* p4 = reinterpret_cast<const float4*>(xr32 + 256 * i + 8 * lane);
          const float4 a = __ldcg(p4), b = __ldcg(p4 + 1);
          v[i][0] = a.x; v[i][1] = a.y; v[i][2] = a.z; v[i][3] = a.w;
          v[i][4] = b.x; v[i][5] = b.y; v[i][6] = b.z; v[i][7] = b.w;
#pragma unroll
          for (int j = 0; j < 8; ++j) ss += v[i][j] * v[i][j];
        }
      const float inv = 1.0f / sqrtf(warp_sum(ss) / (float)H + P.eps);
#pragma unroll
      for (int i = 0; i < kMaxBlk; ++i)
        if (i < nblk) {
          float gf[8];
          bf16x8_to_f32(__ldg(gam + (256 * i + 8 * lane) / 8), gf);
          __align__(16) __nv_bfloat16 o[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) o[j] = __float2bfloat16_rn(v[i][j] * inv * gf[j]);
          const uint4 ov = *reinterpret_cast<const uint4*>(o);
          *reinterpret_cast<uint4*>(xhat + (size_t)t * H + 256 * i + 8 * lane) = ov;
          *reinterpret_cast<uint4*>(xs + (size_t)w * H + 256 * i + 8 * lane) = ov;
          if (S.cap_moe_in)
            *reinterpret_cast<uint4*>(S.cap_moe_in + ((size_t)d.layer * T + t) * H + 256 * i + 8 * lane) = ov;
        }
    } else if (t < T) {
      const uint4* xr = reinterpret_cast<const uint4*>(S.moe_x) + (size_t)t * H / 8;
#pragma unroll
      for (int i = 0; i < kMaxBlk; ++i)
        if (i < nblk) *reinterpret_cast<uint4*>(xs + (size_t)w * H + 256 * i + 8 * lane) = __ldcg(xr + 32 * i + lane);
    }
  }
  bar_sync(BAR_COMP, kComputeThreads);  // the token rows are staged (and the FFN inputs written)
  // logits: warp w takes experts w, w + 8, ...; the token rows come from
  // shared memory, so an expert costs one round trip (its router row) for all
  // the task's tokens; each logit is summed in the fixed order (lane l:
  // columns 256 i + 8 l + j in increasing i, j, then the xor butterfly)
  const uint4* wr = reinterpret_cast<const uint4*>(mw.router);
  const int nt = min(8, T - d.idx * 8);
  for (int e = w; e < E; e += kComputeWarps) {
    uint4 wv[kMaxBlk];
#pragma unroll
    for (int i = 0; i < kMaxBlk; ++i)
      if (i < nblk) wv[i] = __ldg(wr + ((size_t)e * H + 256 * i + 8 * lane) / 8);
    const float bias = mw.bias ? __ldg(mw.bias + e) : 0.f;
    for (int tt = 0; tt < nt; ++tt) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxBlk; ++i)
        if (i < nblk) {
          float wf[8], xf[8];
          bf16x8_to_f32(wv[i], wf);
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(xs + (size_t)tt * H + 256 * i + 8 * lane), xf);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc = fmaf(wf[j], xf[j], acc);  // the product is exact in fp32
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc = acc + __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) lg[tt * 64 + e] = acc + bias;
    }
  }
  bar_sync(BAR_COMP, kComputeThreads);
  const int t = d.idx * 8 + w;
  if (t >= T) return;
  const bool has0 = lane < E, has1 = lane + 32 < E;
  const float v0 = has0 ? lg[w * 64 + lane] : 0.f, v1 = has1 ? lg[w * 64 + lane + 32] : 0.f;
  // debug outputs: the MoE decoder's hold one block per layer
  const size_t lblk = dec ? (size_t)d.layer : 0;
  if (S.dbg_logits) {
    if (has0) S.dbg_logits[(lblk * T + t) * E + lane] = v0;
    if (has1) S.dbg_logits[(lblk * T + t) * E + lane + 32] = v1;
  }
  bool av0 = has0, av1 = has1;
  int sel_e = 0;
  float sel_v = 0.f;
  for (int j = 0; j < K; ++j) {
    const unsigned long long k0 = av0 ? argmax_key(v0, lane) : 0ull, k1 = av1 ? argmax_key(v1, lane + 32) : 0ull;
    unsigned long long best = k0 > k1 ? k0 : k1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    const int e = argmax_key_index(best);
    const float v = __shfl_sync(0xffffffffu, e < 32 ? v0 : v1, e & 31);
    if (lane == (e & 31)) { if (e < 32) av0 = false; else av1 = false; }
    if (lane == j) { sel_e = e; sel_v = v; }
  }
  const float mx = __shfl_sync(0xffffffffu, sel_v, 0);  // the first selection is the largest
  const float ex = lane < K ? expf(sel_v - mx) : 0.f;
  const float sum = warp_sum(ex);
  int rank = 0;
  if (lane < K) {
    const float wt = ex / sum;
    const size_t pi = (size_t)t * K + lane;
    rank = atomicAdd(reinterpret_cast<int*>(mb + P.off_mhist) + sel_e, 1);
    reinterpret_cast<int*>(mb + P.off_mrank)[pi] = rank;
    reinterpret_cast<int*>(mb + P.off_midx)[pi] = sel_e;
    reinterpret_cast<float*>(mb + P.off_mw)[pi] = wt;
    if (S.dbg_idx) S.dbg_idx[lblk * T * K + pi] = sel_e;
    if (S.dbg_w) S.dbg_w[lblk * T * K + pi] = wt;
  }
  // grouping: the token's row goes to each selected expert's rows of the
  // routed-row buffer, at the pair's rank there (each GroupGEMM tile then
  // loads its B operand as one box of consecutive rows)
  uint4* xg = reinterpret_cast<uint4*>(mb + P.off_mxg);
  const size_t dst_row = lane < K ? ((size_t)sel_e * P.moe_cap + rank) * (H / 8) : 0;  // lane j: pair j's row
  for (int i = 0; i < nblk; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(xs + (size_t)w * H + 256 * i + 8 * lane);  // (token t's staged row)
    for (int j = 0; j < K; ++j) xg[__shfl_sync(0xffffffffu, dst_row, j) + 32 * i + lane] = v;
  }
}

// MINDPTR (follow-up of the routing event, all compute warps): exp_indptr =
// exclusive prefix sum of the histogram; tile_ptr = exclusive prefix sum of
// ceil(hist[e] / tm) and the tile -> (expert, m) table the GroupGEMM tasks
// decode; the run-time count of EV_MY (one per down task); and the row map
// (pair -> row, row -> pair).
__device__ __forceinline__ void task_mindptr(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws,
                                             const TaskDesc& d) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  const int E = P.n_experts, K = P.top_k, TMt = P.moe_tm;
  unsigned char* mb = moe_block(P, ws, d.layer);
  int* sx = reinterpret_cast<int*>(sm.xs());  // exp_indptr [E + 1], then the tile count
  const size_t lblk = P.kind == MK_MODEL_MOE_DECODER ? (size_t)d.layer : 0;
  int* dbg_hist = S.dbg_hist ? S.dbg_hist + lblk * E : nullptr;
  int* dbg_indptr = S.dbg_indptr ? S.dbg_indptr + lblk * (E + 1) : nullptr;
  bar_sync(BAR_COMP, kComputeThreads);
  if (w == 0) {
    const int* hist = reinterpret_cast<const int*>(mb + P.off_mhist);
    int* indptr = reinterpret_cast<int*>(mb + P.off_mindptr);
    int* tptr = reinterpret_cast<int*>(mb + P.off_mtile);
    int* tile_e = reinterpret_cast<int*>(mb + P.off_mtile_e);
    int* tile_m = reinterpret_cast<int*>(mb + P.off_mtile_m);
    const int h0 = lane < E ? __ldcg(hist + lane) : 0, h1 = lane + 32 < E ? __ldcg(hist + lane + 32) : 0;
    // tiles per expert, from its routed rows (routing-aware tile heights)
    const int t0 = moe_tile_rows(h0, TMt, P.moe_big), t1 = moe_tile_rows(h1, TMt, P.moe_big);
    const int c0 = (h0 + t0 - 1) / t0, c1 = (h1 + t1 - 1) / t1;
    int s0 = h0, s1 = h1, u0 = c0, u1 = c1;  // inclusive scans over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a0 = __shfl_up_sync(0xffffffffu, s0, o), a1 = __shfl_up_sync(0xffffffffu, s1, o);
      const int b0 = __shfl_up_sync(0xffffffffu, u0, o), b1 = __shfl_up_sync(0xffffffffu, u1, o);
      if (lane >= o) { s0 += a0; s1 += a1; u0 += b0; u1 += b1; }
    }
    const int tot_h0 = __shfl_sync(0xffffffffu, s0, 31), tot_c0 = __shfl_sync(0xffffffffu, u0, 31);
    const int ex0 = s0 - h0, ex1 = tot_h0 + s1 - h1;
    const int tx0 = u0 - c0, tx1 = tot_c0 + u1 - c1;
    if (lane < E) {
      indptr[lane] = ex0; sx[lane] = ex0; tptr[lane] = tx0;
      for (int m = 0; m < c0; ++m) { tile_e[tx0 + m] = lane; tile_m[tx0 + m] = m; }
      if (dbg_hist) dbg_hist[lane] = h0;
      if (dbg_indptr) dbg_indptr[lane] = ex0;
    }
    if (lane + 32 < E) {
      indptr[lane + 32] = ex1; sx[lane + 32] = ex1; tptr[lane + 32] = tx1;
      for (int m = 0; m < c1; ++m) { tile_e[tx1 + m] = lane + 32; tile_m[tx1 + m] = m; }
      if (dbg_hist) dbg_hist[lane + 32] = h1;
      if (dbg_indptr) dbg_indptr[lane + 32] = ex1;
    }
    if (lane == 31) {
      const int rows = tot_h0 + s1, tiles = tot_c0 + u1;
      indptr[E] = rows; sx[E] = rows; tptr[E] = tiles; sx[E + 1] = tiles;
      if (dbg_indptr) dbg_indptr[E] = rows;
      // data-dependent event count: every down task of every tile notifies EV_MY
      atomicExch(reinterpret_cast<int*>(ws + P.off_counters) + ev_ctr(P, EV_MY, moe_li(d.layer)), tiles * P.nt_d);
    }
  }
  bar_sync(BAR_COMP, kComputeThreads);
  // data-dependent event update: the tiles the routing created wait for their
  // gate/up tasks (the elements past them stay armed at zero); the GroupGEMM
  // tasks are pushed only after this task's notify, which releases these writes
  {
    int* ctr = reinterpret_cast<int*>(ws + P.off_counters);
    for (int t = ct; t < sx[E + 1]; t += kComputeThreads) atomicExch(ctr + ev_ctr(P, EV_MH, moe_li(d.layer), t), P.nt_gu);
  }
  const int* midx = reinterpret_cast<const int*>(mb + P.off_midx);
  const int* mrank = reinterpret_cast<const int*>(mb + P.off_mrank);
  int* mrow = reinterpret_cast<int*>(mb + P.off_mrow);
  int* mperm = reinterpret_cast<int*>(mb + P.off_mperm);
  const int npairs = S.B * K;
  for (int p = ct; p < npairs; p += kComputeThreads) {
    const int row = sx[__ldcg(midx + p)] + __ldcg(mrank + p);
    mrow[p] = row;
    mperm[row] = p;
  }
}

// ---- GroupGEMM tiles on tcgen05 (5th-generation tensor cores, TMEM accumulators)
// A tile is up to kMoeTileRows routed rows of one expert; a task multiplies
// kMoeTaskRows weight rows of that expert (the MMA's M = 128) by the tile's
// rows (N = 16 or 64, the B operand) over K in 64-column chunks that the
// producer streams into the ring (see emit).  Compute warp 0's lane 0 issues
// the MMAs (M 128 x N x 16, bf16 in, fp32 accumulate in TMEM) as the chunks
// land and releases each slot with tcgen05.commit; the accumulator's
// completion arrives on acc_bar.  The epilogue reads TMEM: warp quadrant q
// (hardware warp % 4) owns lanes 32q .. 32q + 31, i.e. weight rows; the two
// compute warps of a quadrant split the N columns (routed rows).

// Issue the MMAs of one GroupGEMM task (one thread).  Per chunk c of K the
// task's slots are [A0, (A1,) B]: A0 (and A1 for gate/up, its up rows) are
// 128 weight rows x 64 columns, B is the tile's N rows x 64 columns.  D0 at
// TMEM column 0 accumulates A0 . B^T, D1 at column 128 accumulates A1 . B^T.
__device__ __forceinline__ void moe_issue_mma(const DevPlan& P, Smem& sm, unsigned char* ring, Control* ctl,
                                              const TaskDesc& d, int nk, int parts, int N) {
  const int R = P.ring_slots;
  const uint32_t idesc = umma_idesc_bf16(kMoeTaskRows, N);
  const uint32_t tm = sm.tmem_base;
  for (int c = 0; c < nk; ++c) {
    int sl[3];
    for (int q = 0; q <= parts; ++q) {
      uint32_t par;
      sl[q] = task_slot(d, (parts + 1) * c + q, R, par);
      wait_mbar(&sm.full[sl[q]], par, ctl, P.spin_timeout_ns, d.fam, d.idx);
    }
    tc_fence_after();
    const uint64_t b = umma_desc_sw128(ring + (size_t)sl[parts] * P.slot_bytes);
    for (int q = 0; q < parts; ++q) {
      const uint64_t a = umma_desc_sw128(ring + (size_t)sl[q] * P.slot_bytes);
#pragma unroll
      for (int k = 0; k < 4; ++k) umma_bf16(tm + 128u * q, a + 2u * k, b + 2u * k, idesc, (c | k) ? 1u : 0u);
    }
    for (int q = 0; q <= parts; ++q) umma_commit(&sm.empty[sl[q]]);
  }
  umma_commit(&sm.acc_bar);
}

// EGU task (tile, n): gate rows and up rows n*128 .. n*128 + 127 of the
// tile's expert against its routed rows (gathered by the routing tasks into
// the expert's rows of the routed-row buffer) -> SwiGLU, stored as bf16 at the
// tile's compact rows of the SwiGLU buffer.
__device__ __forceinline__ void task_egu(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                                         unsigned char* ws, Control* ctl, const TaskDesc& d, uint32_t& tc_n) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  unsigned char* mb = moe_block(P, ws, d.layer);
  const int tile = d.idx / P.nt_gu, n = d.idx - tile * P.nt_gu;
  const MoeTile mt = moe_tile(P, mb, tile);
  const int N = moe_tile_n(mt.nrows);
  if (w == 0) {
    if (lane == 0) moe_issue_mma(P, sm, ring, ctl, d, P.hidden / 64, 2, N);
    __syncwarp();
  }
  wait_local(&sm.acc_bar, tc_n & 1u, P.spin_timeout_ns);
  tc_n++;
  tc_fence_after();
  const int q = (threadIdx.x >> 5) & 3;  // TMEM lane quadrant of this warp
  const int col = n * kMoeTaskRows + 32 * q + lane;  // this lane's gate/up row = SwiGLU column
  const bool ok = col < P.eff;
  __nv_bfloat16* mh = reinterpret_cast<__nv_bfloat16*>(mb + P.off_mh);
  const uint32_t ta = S_tmem_lane(sm.tmem_base, q);
  for (int c8 = (w >> 2) * (N / 2); c8 < ((w >> 2) + 1) * (N / 2); c8 += 8) {
    float g[8], u[8];
    tmem_ld8(ta + (uint32_t)c8, g);
    tmem_ld8(ta + 128u + (uint32_t)c8, u);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (ok && c8 + i < mt.nrows)
        mh[(size_t)(mt.r0 + c8 + i) * P.eff + col] = __float2bfloat16_rn(g[i] / (1.0f + expf(-g[i])) * u[i]);
  }
  tc_fence_before();
  bar_sync(BAR_COMP, kComputeThreads);  // the accumulator is free for the next task
}

// EDOWN task (tile, n): down rows n*128 .. n*128 + 127 of the tile's expert
// against the tile's SwiGLU rows -> fp32 at the tile's compact rows, columns
// n*128 .. n*128 + 127, of the expert-output buffer.
__device__ __forceinline__ void task_edown(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                                           unsigned char* ws, Control* ctl, const TaskDesc& d, uint32_t& tc_n) {
  const int ct = threadIdx.x - kComputeBase, lane = ct & 31, w = ct >> 5;
  unsigned char* mb = moe_block(P, ws, d.layer);
  const int tile = d.idx / P.nt_d, n = d.idx - tile * P.nt_d;
  const MoeTile mt = moe_tile(P, mb, tile);
  const int N = moe_tile_n(mt.nrows);
  if (w == 0) {
    if (lane == 0) moe_issue_mma(P, sm, ring, ctl, d, P.eff / 64, 1, N);
    __syncwarp();
  }
  wait_local(&sm.acc_bar, tc_n & 1u, P.spin_timeout_ns);
  tc_n++;
  tc_fence_after();
  const int q = (threadIdx.x >> 5) & 3;
  const int col = n * kMoeTaskRows + 32 * q + lane;  // output column (< hidden)
  float* my = reinterpret_cast<float*>(mb + P.off_my);
  const uint32_t ta = S_tmem_lane(sm.tmem_base, q);
  for (int c8 = (w >> 2) * (N / 2); c8 < ((w >> 2) + 1) * (N / 2); c8 += 8) {
    float v[8];
    tmem_ld8(ta + (uint32_t)c8, v);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (c8 + i < mt.nrows) my[(size_t)(mt.r0 + c8 + i) * P.hidden + col] = v[i];
  }
  tc_fence_before();
  bar_sync(BAR_COMP, kComputeThreads);
}

// COMBINE: warp w takes token 8*idx + w: out[t] = sum_j w[t, j] * y[row(t, j)]
// in slot order j = 0..k-1, written as bf16.
__device__ __forceinline__ void task_combine(const DevPlan& P, const StepParams& S, unsigned char* ws,
                                             const TaskDesc& d) {
  const int lane = threadIdx.x & 31, w = (threadIdx.x - kComputeBase) >> 5;
  const int H = P.hidden, K = P.top_k, nblk = H >> 8;
  const int nt = min(8, S.B - d.idx * 8);  // this task's tokens
  const unsigned char* mb = moe_block(P, ws, d.layer);
  const int* mrow = reinterpret_cast<const int*>(mb + P.off_mrow);
  const float* mw = reinterpret_cast<const float*>(mb + P.off_mw);
  const float* my = reinterpret_cast<const float*>(mb + P.off_my);
  const bool dec = P.kind == MK_MODEL_MOE_DECODER;
  // items (token tt, 256-column block i) over the 8 warps, token fastest:
  // with 8 tokens warp w takes token w's blocks (as one warp per token), with
  // one token each warp takes one block (its loads in one round trip); each
  // element sums its expert rows in the token's top-k order whichever warp
  // takes it
  int rows[8], cur = -1;
  float wts[8];
  for (int it = w; it < nt * nblk; it += kComputeWarps) {
    const int tt = it % nt, i = it / nt;
    const int t = d.idx * 8 + tt;
    float* xres = reinterpret_cast<float*>(ws + P.off_x) + (size_t)t * H;
    if (tt != cur) {
      cur = tt;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < K) { rows[j] = __ldcg(mrow + (size_t)t * K + j); wts[j] = __ldcg(mw + (size_t)t * K + j); }
    }
    const int c = 256 * i + 8 * lane;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < K) {
        const float4* y4 = reinterpret_cast<const float4*>(my + (size_t)rows[j] * H + c);
        const float4 a = __ldcg(y4), b = __ldcg(y4 + 1);
        acc[0] = fmaf(wts[j], a.x, acc[0]); acc[1] = fmaf(wts[j], a.y, acc[1]);
        acc[2] = fmaf(wts[j], a.z, acc[2]); acc[3] = fmaf(wts[j], a.w, acc[3]);
        acc[4] = fmaf(wts[j], b.x, acc[4]); acc[5] = fmaf(wts[j], b.y, acc[5]);
        acc[6] = fmaf(wts[j], b.z, acc[6]); acc[7] = fmaf(wts[j], b.w, acc[7]);
      }
    if (dec) {
      // MoE decoder: the FFN output joins the fp32 residual
      float4* x4 = reinterpret_cast<float4*>(xres + c);
      float4 a = __ldcg(x4), b = __ldcg(x4 + 1);
      a.x += acc[0]; a.y += acc[1]; a.z += acc[2]; a.w += acc[3];
      b.x += acc[4]; b.y += acc[5]; b.z += acc[6]; b.w += acc[7];
      x4[0] = a;
      x4[1] = b;
    } else {
      __align__(16) __nv_bfloat16 o[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) o[q] = __float2bfloat16_rn(acc[q]);
      *reinterpret_cast<uint4*>(S.moe_out + (size_t)t * H + c) = *reinterpret_cast<const uint4*>(o);
    }
  }
}

// Kernel instances: the plan kinds (MK_MODEL_*), and the dense decoder's
// wide-batch path as an instance of its own.
template <int kKind>
__device__ void compute(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring, unsigned char* ws,
                        Control* ctl) {
  const int lane = threadIdx.x & 31, w = (threadIdx.x - kComputeBase) >> 5;
  const int B = S.B;
  int a_tag = -1;
  uint32_t tc_n = 0;  // tcgen05 tasks run (the phase of acc_bar)
  uint32_t bq = 0;    // wide batch: activation chunks the MMA issuer loaded (stage and phase)
  constexpr bool kWide = Kind<kKind>::wide;
  constexpr bool kMoe = Kind<kKind>::moe;
  constexpr bool tc = Kind<kKind>::base != MK_MODEL_DENSE;
  if constexpr (tc) {
    // tensor memory for the tcgen05 accumulators, held for the kernel's lifetime
    if (w == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    bar_sync(BAR_COMP, kComputeThreads);
    tc_fence_after();
  }
  for (uint32_t k = 0;; ++k) {
    // task k: released into cur[k & 1] as phase k >> 1 of go_bar[k & 1].  An
    // abort does not end this wait: the controller always releases either
    // the task or an END (its own waits are bounded), and every compute warp
    // must see the same sequence, since the task bodies meet at barriers.
    if (!wait_local(&sm.go_bar[k & 1], (k >> 1) & 1, P.spin_timeout_ns)) break;
    const TaskDesc d = sm.cur[k & 1];
    if (d.op == OP_END) break;
    uint32_t* trec = (Kind<kKind>::trace && d.rec > 0 && w == 0) ? trace_rec(S, d.rec) : nullptr;
    if (trec && lane == 0) trec[TR_CSTART] = (uint32_t)global_ns();
    GemvSpec g;
    bool moe_task = false;
    if (P.debug_flags & MK_DEBUG_EMPTY_TASKS) {  // interpreter measurement: no body
      if (trec && lane == 0) trec[TR_CEND] = (uint32_t)global_ns();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.done_bar[k & 1]);
      continue;
    }
    if constexpr (kMoe) {
      moe_task = d.op >= OP_ROUTE && d.op <= OP_MFIN;
      if (d.op == OP_ROUTE) {
        task_route(P, S, sm, ws, d);
      } else if (d.op == OP_MINDPTR) {
        task_mindptr(P, S, sm, ws, d);
      } else if (d.op == OP_EGU) {
        task_egu(P, S, sm, ring, ws, ctl, d, tc_n);
      } else if (d.op == OP_EDOWN) {
        task_edown(P, S, sm, ring, ws, ctl, d, tc_n);
      } else if (d.op == OP_COMBINE) {
        task_combine(P, S, ws, d);
      }
    }
    if (Kind<kKind>::moe_layer || moe_task) {
      a_tag = -1;  // MoE tasks use the staging buffer as scratch
    } else if (kWide && (d.op == OP_QKV || d.op == OP_OPROJ || d.op == OP_GATEUP || d.op == OP_DOWN ||
                         d.op == OP_LM)) {
      if constexpr (kWide) task_gemm_wide(P, S, sm, ring, ws, ctl, d, tc_n, bq, trec);
    } else if (kWide && (d.op == OP_NORM || d.op == OP_NORM2 || d.op == OP_NORMF)) {
      if constexpr (kWide) task_norm(P, S, sm, ws, d);
    } else if (!kWide && gemv_spec(P, d, g)) {
      // all B activation rows are staged together; an unchanged tag reuses them
      const GemvItem it = gemv_item(sm.geo[d.op], B, threadIdx.x - kComputeBase);
      EpiAhead ea;
      gemv_epilogue_ahead(P, sm, ws, d, it, ea);
      if (g.tag != a_tag) {
        // debug capture: the residual after layer l is what QKV of layer l + 1
        // (the LM head after the last layer) reduces; task 0 of the family writes it
        float* cap = nullptr;
        if (S.cap_resid && d.idx == 0 && ((d.op == OP_QKV && d.layer > 0) || d.op == OP_LM))
          cap = S.cap_resid + (size_t)(d.op == OP_LM ? P.n_layers - 1 : d.layer - 1) * B * P.hidden;
        stage_act(P, ws, sm, g, B, trec, cap);
        a_tag = g.tag;
      }
      if (trec && lane == 0) trec[TR_STAGED] = (uint32_t)global_ns();
      gemv_task(P, S, sm, ring, ws, ctl, d, g, B, ea, trec);
    } else if (d.op == OP_ATTN) {
      task_attn(P, S, sm, ring, ws, ctl, d, trec);
      a_tag = -1;  // the staging buffer held the warps' partial outputs
    } else if (d.op == OP_LMFIN) {
      for (int b = threadIdx.x - kComputeBase; b < B; b += kComputeThreads) {
        unsigned long long k = __ldcg(reinterpret_cast<const unsigned long long*>(ws + P.off_lmbest) + b);
        S.next_tokens[b] = argmax_key_index(k);
      }
    }
    if (trec && lane == 0) trec[TR_CEND] = (uint32_t)global_ns();
    // every lane of the warp has finished its writes before lane 0 arrives
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.done_bar[k & 1]);
  }
  if constexpr (tc) {
    // every MMA completed (each task waited for its accumulator): free the TMEM
    tc_fence_before();
    bar_sync(BAR_COMP, kComputeThreads);
    tc_fence_after();
    if (w == 0) tmem_dealloc(sm.tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- kernel
// Prologue: every family's extent for this step's symbols (into shared
// memory), and every Event Tensor counter armed with its wait count (this
// thread's share of the grid-wide range).
__device__ __forceinline__ void arm_events(const DevPlan& P, Smem& sm, const FamilyDesc* fams, const int32_t* code,
                                        int* counters, int B) {
  const int tid = threadIdx.x;
  for (int f = tid; f < P.n_families; f += blockDim.x) {
    ExprEnv env{B, sm.ctx, {0, 0, 0}, sm.asplit};
    sm.fam_ext[f] = expr_eval(code, fams[f].extent_expr, env);
    sm.fam_op[f] = (signed char)fams[f].op;
    sm.fam_layer[f] = (signed char)fams[f].layer;
  }
  const int gtid = blockIdx.x * blockDim.x + tid, gthreads = gridDim.x * blockDim.x;
  for (int i = gtid; i < P.n_counters; i += gthreads) {
    // the event tensor holding counter i (tensors a plan does not use are empty)
    int e = 0;
    for (; e < EV_COUNT; ++e) {
      const EventTensorDesc& d = P.ev[e];
      const int size = d.ndim < 1 ? 0 : d.dims[0] * (d.ndim > 1 ? d.dims[1] : 1) * (d.ndim > 2 ? d.dims[2] : 1);
      if (i >= d.base && i < d.base + size) break;
    }
    if (e == EV_COUNT) continue;
    int lin = i - P.ev[e].base;
    ExprEnv env{B, sm.ctx, {0, 0, 0}, sm.asplit};
    for (int dd = P.ev[e].ndim - 1; dd >= 0; --dd) { env.coord[dd] = lin % P.ev[e].dims[dd]; lin /= P.ev[e].dims[dd]; }
    counters[i] = expr_eval(code, P.ev[e].count_expr, env) + (i == P.fault_ctr ? 1 : 0);
  }
}

// One persistent kernel per plan kind: the instances share the interpreter
// (producer, controller, notifier) and differ in the task bodies compiled in
// (dense decoder, MoE layer, or both for the MoE decoder), so each gets its
// own register allocation.
template <int kKind>
__global__ void __launch_bounds__(kThreads, 1) megakernel(const DevPlan P, const StepParams S, unsigned char* ws) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = smem_raw;
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (size_t)P.ring_slots * P.slot_bytes);
  Control* ctl = reinterpret_cast<Control*>(ws + P.off_control);
  int* counters = reinterpret_cast<int*>(ws + P.off_counters);
  const FamilyDesc* fams = reinterpret_cast<const FamilyDesc*>(ws + P.off_families);
  const int32_t* code = reinterpret_cast<const int32_t*>(ws + P.off_expr);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int B = S.B;

  // ---- prologue: resolve the symbols, arm the Event Tensors, gather embeddings
  const bool moe = P.kind == MK_MODEL_MOE_LAYER;
  if (tid == 0) {
    int* seq = reinterpret_cast<int*>(sm.stage() + P.act_bytes + P.gred_bytes);
    const int mb = P.max_batch > 0 ? P.max_batch : 1;
    sm.ctx = seq; sm.slot = seq + mb; sm.tok = seq + 2 * mb; sm.nch = seq + 3 * mb; sm.pre = seq + 4 * mb;
    sm.bad = moe ? (B < 1 || B > P.max_tokens) : (B < 1 || B > P.max_batch || B > (P.wide ? kMaxBatch : kMaxB));
    // the ring's slots hold 128-byte-swizzled TMA boxes and tcgen05 operands,
    // whose swizzle pattern assumes 1024-byte-aligned slots
    if (smem_u32(smem_raw) & 1023u) sm.bad = 1;
    sm.released = 0;
    sm.dq_head = sm.dq_tail = sm.fq_head = sm.fq_tail = sm.notifier_stop = 0;
  }
  if (tid < kComputeWarps * kMaxB) sm.lm_seen[tid / kMaxB][tid % kMaxB] = 0ull;
  if (tid < kMaxBatch) sm.lm_cta[tid] = sm.lm_pub[tid] = 0ull;
  if (P.kind != MK_MODEL_MOE_LAYER && blockIdx.x == 0)  // attention pair counters
    for (int i = tid; i < P.max_batch * P.n_kv_heads; i += blockDim.x) reinterpret_cast<int*>(ws + P.off_actr)[i] = 0;
  if (P.wide && blockIdx.x == 0)  // split-K tile counters
    for (int i = tid; i < 3 * kGctrPerOp; i += blockDim.x) reinterpret_cast<int*>(ws + P.off_gctr)[i] = 0;
  __syncthreads();
  if (!moe && !sm.bad && tid < B) {
    int c = S.ctx[tid], s = S.slots[tid], t = S.tokens[tid];
    sm.ctx[tid] = c; sm.slot[tid] = s; sm.tok[tid] = t;
    if (c < 0 || c >= P.max_ctx || s < 0 || s >= P.n_slots || t < 0 || t >= P.vocab) atomicOr(&sm.bad, 1);
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0) {
      if (blockIdx.x == 0) record_error(ctl, MK_ERR_DEVICE_BOUNDS, -1, -1, -1);
      atomicAdd(&ctl->grid_bar, 1u);  // keep the barrier count in step with the launch count
    }
    return;
  }
  if (tid == 0) {
    // GEMV geometry of each op (see OpGeo)
    auto set_geo = [&](int op, int K, int rows_part, int pairs) {
      OpGeo& gg = sm.geo[op];
      gg.rows_part = rows_part;
      gg.cw = K / kGemvSlots;
      gg.pairs = pairs;
    };
    if (!moe && !P.wide) {
      set_geo(OP_QKV, P.hidden, P.tile_qkv / 2, 1);
      set_geo(OP_OPROJ, P.hidden, P.tile_o, 0);
      set_geo(OP_GATEUP, P.hidden, P.tile_gu, 1);
      set_geo(OP_DOWN, P.kseg, P.tile_down, 0);
      set_geo(OP_LM, P.hidden, P.tile_lm, 0);
    }
    sm.asplit = moe ? P.attn_split : step_attn_split(P, B, sm.ctx);
    // K/V the step reads; below half of L2 it is kept at normal priority, so
    // that it stays in L2 from one step to the next
    long long kv = 0;
    for (int b = 0; !moe && b < B; ++b) kv += sm.ctx[b] + 1;
    sm.kv_ef = kv * P.n_layers * P.n_kv_heads * P.head_dim * 4 > kKvL2Bytes;
    if (!moe) {
      int run = 0;
      for (int b = 0; b < B; ++b) {  // attention tasks of sequence b: its key chunks, asplit at a time
        sm.pre[b] = run;
        sm.nch[b] = ceil_div(ceil_div(sm.ctx[b] + 1, P.chunk), sm.asplit);
        run += sm.nch[b];
      }
      sm.pre[B] = run;
    }
  }
  __syncthreads();
  arm_events(P, sm, fams, code, counters, B);
  const int gtid = blockIdx.x * blockDim.x + tid, gthreads = gridDim.x * blockDim.x;
  if (P.kind != MK_MODEL_DENSE && blockIdx.x == 0) {
    // every MoE layer's expert histogram starts at zero
    const int n_moe = P.kind == MK_MODEL_MOE_DECODER ? P.n_layers : 1;
    for (int i = tid; i < n_moe * P.n_experts; i += blockDim.x)
      reinterpret_cast<int*>(moe_block(P, ws, i / P.n_experts) + P.off_mhist)[i % P.n_experts] = 0;
  }
  if (!moe) {
    float* x = reinterpret_cast<float*>(ws + P.off_x);
    const int cpr = P.hidden / 8;
    for (int i = gtid; i < B * cpr; i += gthreads) {
      int b = i / cpr, c = i % cpr;
      uint4 v = __ldg(reinterpret_cast<const uint4*>(P.embed) + ((size_t)sm.tok[b] * P.hidden) / 8 + c);
      float f[8];
      bf16x8_to_f32(v, f);
      float4* dst = reinterpret_cast<float4*>(x + (size_t)b * P.hidden + c * 8);
      dst[0] = make_float4(f[0], f[1], f[2], f[3]);
      dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
  if (blockIdx.x == 0 && tid < P.max_batch)
    reinterpret_cast<unsigned long long*>(ws + P.off_lmbest)[tid] = 0ull;  // running argmax keys
  if (blockIdx.x == 0 && tid == 0 && P.sched == MK_SCHED_DYNAMIC) {
    ctl->q_head = 0;
    ctl->q_tail = 0;
    if (moe) push_range(P, S, ctl, ws, fam_of(P, OP_ROUTE, -1), 0, ceil_div(B, 8));
    else if (P.wide) push_range(P, S, ctl, ws, fam_of(P, OP_NORM, 0), 0, B);  // EV_IN[0] armed at zero
    else push_range(P, S, ctl, ws, fam_of(P, OP_QKV, 0), 0, P.n_qkv_tiles);  // EV_IN[0] is armed at zero
  }
  if (tid == 0) {
    for (int s = 0; s < P.ring_slots; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], 1); }
    for (int j = 0; j < 2; ++j) { mbar_init(&sm.go_bar[j], 1); mbar_init(&sm.done_bar[j], kComputeWarps); }
    mbar_init(&sm.acc_bar, 1);
    for (int j = 0; j < kBStages; ++j) { mbar_init(&sm.bfull[j], 1); mbar_init(&sm.bempty[j], 1); }
    for (int k = 0; k < kFifo; ++k) { mbar_init(&sm.fifo_full[k], 1); mbar_init(&sm.fifo_empty[k], 1); }
    fence_proxy_async_smem();
  }
  // ---- grid barrier: every counter is armed before any task runs
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(&ctl->grid_bar, 1u);
    const unsigned target = S.epoch * gridDim.x;
    unsigned long long t0 = global_ns();
    for (int it = 0;; ++it) {
      if ((int)(ld_acquire_u32(&ctl->grid_bar) - target) >= 0) break;
      if ((it & 15) == 15) {
        if (aborted(ctl)) break;
        if ((long long)(global_ns() - t0) > P.spin_timeout_ns) { record_error(ctl, MK_ERR_DEVICE_TIMEOUT, -1, -1, -1); break; }
      }
    }
  }
  __syncthreads();

  // ---- interpreter roles
  if (warp == 0) {
    if ((tid & 31) == 0) producer<kKind>(P, S, sm, ring, ws, ctl);
  } else if (warp == 1) {
    controller<kKind>(P, S, sm, ws, ctl, counters);
  } else if (warp == 2) {
    notifier<kKind>(P, S, sm, ws, ctl, counters);
  } else {
    compute<kKind>(P, S, sm, ring, ws, ctl);
  }
}

}  // namespace mk

// ---------------------------------------------------------------- host glue
#include "launch.hpp"

namespace mk {

template <int kFlags>
static const void* kernel_of(const DevPlan& P) {
  switch (P.kind) {
    case MK_MODEL_MOE_LAYER: return (const void*)megakernel<MK_MODEL_MOE_LAYER | kFlags>;
    case MK_MODEL_MOE_DECODER:
      return P.wide ? (const void*)megakernel<kKindMoeDecWide | kFlags>
                    : (const void*)megakernel<MK_MODEL_MOE_DECODER | kFlags>;
    default:
      return P.wide ? (const void*)megakernel<kKindDenseWide | kFlags> : (const void*)megakernel<MK_MODEL_DENSE | kFlags>;
  }
}
static const void* kernel_for(const DevPlan& P) {
  return (P.debug_flags & MK_DEBUG_TRACE) ? kernel_of<kTraced>(P) : kernel_of<0>(P);
}

mk_status dev_query(int* n_sm, int* smem_optin, int* device, std::string& err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) { err = std::string("CUDA device query failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) { err = "this library is built for sm_100a (B200) only"; return MK_ERR_UNSUPPORTED; }
  *device = dev;
  return MK_OK;
}

int smem_fixed_bytes() { return kSmemFixed; }

// The driver's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// Tensor maps of the dense weight matrices, written into the plan image: a
// bf16 [rows][cols] matrix with a row stride, read in boxes of (cols / 8)
// columns x box_rows rows (one box per ring slot and part); rows past the
// end read as zeros.
static bool encode_weight_maps(const DevPlan& P, const unsigned char* ws, std::vector<unsigned char>& image,
                               std::string& err) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) { err = "cuTensorMapEncodeTiled is not available"; return false; }
  const LayerPtrs* layers = reinterpret_cast<const LayerPtrs*>(image.data() + (P.off_layers - P.off_families));
  // a bf16 [rows][cols] row-major matrix read in boxes of 64 columns x box_rows
  // rows under the 128-byte swizzle (the K-major layout of a tcgen05 operand);
  // rows past the end read as zeros
  auto put_sw128 = [&](int index, const void* w, long long rows, long long cols, int box_rows,
                       const char* what) -> bool {
    if (reinterpret_cast<uintptr_t>(w) & 15) { err = std::string(what) + " must be 16-byte aligned"; return false; }
    CUtensorMap m;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) { err = std::string("tensor map of ") + what + " rejected by the driver"; return false; }
    std::memcpy(image.data() + (P.off_tmap - P.off_families) + (size_t)index * kTmapBytes, &m, sizeof(m));
    return true;
  };
  if (P.kind != MK_MODEL_DENSE) {
    // GroupGEMM operands of every MoE layer: the expert matrices and the
    // layer's routed-row and SwiGLU buffers in the workspace
    const int Lm = P.kind == MK_MODEL_MOE_DECODER ? P.n_layers : 1;
    const long long E = P.n_experts, F = P.eff, H = P.hidden, cap = P.moe_cap, K = P.top_k;
    for (int l = 0; l < Lm; ++l) {
      const bool dec = P.kind == MK_MODEL_MOE_DECODER;
      const void* g = dec ? layers[l].we_gate : P.w_egate;
      const void* u = dec ? layers[l].we_up : P.w_eup;
      const void* dn = dec ? layers[l].we_down : P.w_edown;
      if (!g || !u || !dn) { err = "MoE expert weights missing"; return false; }
      const unsigned char* blk = ws + P.off_mxg + (size_t)l * P.moe_stride;
      const unsigned char* hblk = ws + P.off_mh + (size_t)l * P.moe_stride;
      if (!put_sw128(tmap_index(l, TM_GATE), g, E * F, H, kMoeTaskRows, "expert w_gate") ||
          !put_sw128(tmap_index(l, TM_UP), u, E * F, H, kMoeTaskRows, "expert w_up") ||
          !put_sw128(tmap_index(l, TM_DOWN), dn, E * H, F, kMoeTaskRows, "expert w_down") ||
          !put_sw128(tmap_index(l, TM_XG16), blk, E * cap, H, 16, "routed rows") ||
          !put_sw128(tmap_index(l, TM_XG64), blk, E * cap, H, kMoeTileRows, "routed rows") ||
          !put_sw128(tmap_index(l, TM_HG16), hblk, cap * K, F, 16, "SwiGLU rows") ||
          !put_sw128(tmap_index(l, TM_HG64), hblk, cap * K, F, kMoeTileRows, "SwiGLU rows") ||
          !put_sw128(tmap_index(l, TM_XG128), blk, E * cap, H, kMoeBigTileRows, "routed rows") ||
          !put_sw128(tmap_index(l, TM_HG128), hblk, cap * K, F, kMoeBigTileRows, "SwiGLU rows"))
        return false;
    }
    if (P.kind == MK_MODEL_MOE_LAYER) return true;
  }
  auto put = [&](int index, const void* w, long long rows, long long cols, long long stride_elems, int box_cols,
                 int box_rows, const char* what) -> bool {
    if (!w) return true;  // (an MoE decoder has no dense FFN)
    if (reinterpret_cast<uintptr_t>(w) & 15) { err = std::string(what) + " must be 16-byte aligned"; return false; }
    CUtensorMap m;
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r;
    if (box_cols >= 64) {
      // [rows][cols / 64][64] with the 128-byte swizzle: a box lands as rows of
      // box_cols / 64 128-byte lines, 16-byte chunk c of line n at c ^ (n & 7)
      const cuuint64_t dims[3] = {64, (cuuint64_t)cols / 64, (cuuint64_t)rows};
      const cuuint64_t strides[2] = {128, (cuuint64_t)stride_elems * 2};
      const cuuint32_t box[3] = {64, (cuuint32_t)box_cols / 64, (cuuint32_t)box_rows};
      r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
      const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
      const cuuint64_t strides[1] = {(cuuint64_t)stride_elems * 2};
      const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
      r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) { err = std::string("tensor map of ") + what + " rejected by the driver"; return false; }
    std::memcpy(image.data() + (P.off_tmap - P.off_families) + (size_t)index * kTmapBytes, &m, sizeof(m));
    return true;
  };
  static_assert(sizeof(CUtensorMap) == kTmapBytes, "tensor map size");
  // the norm gains are prefetched into L2 with bulk copies: 16-byte aligned
  for (int l = 0; l < P.n_layers; ++l)
    if ((reinterpret_cast<uintptr_t>(layers[l].attn_norm) | reinterpret_cast<uintptr_t>(layers[l].ffn_norm)) & 15)
      { err = "norm gains must be 16-byte aligned"; return false; }
  if (reinterpret_cast<uintptr_t>(P.final_norm) & 15) { err = "final_norm must be 16-byte aligned"; return false; }
  const int H = P.hidden, D = P.head_dim, Hq = P.n_q_heads, Hkv = P.n_kv_heads, F = P.ffn;
  {
    // the K and V caches as [layer, slot, kv head][max_ctx][64]: one box per
    // 64-key chunk of a (layer, slot, head), under the 128-byte swizzle (the
    // attention tasks' ldmatrix reads are then conflict-free)
    const void* caches[2] = {P.k_cache, P.v_cache};
    for (int kv = 0; kv < 2; ++kv) {
      if (reinterpret_cast<uintptr_t>(caches[kv]) & 15) { err = "the KV caches must be 16-byte aligned"; return false; }
      CUtensorMap m;
      const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)P.max_ctx,
                                  (cuuint64_t)P.n_layers * P.n_slots * Hkv};
      const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)P.max_ctx * D * 2};
      const cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)P.chunk, 1};
      const cuuint32_t estr[3] = {1, 1, 1};
      CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(caches[kv]), dims, strides, box,
                       estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) { err = "tensor map of the KV cache rejected by the driver"; return false; }
      const int index = P.n_layers * kTmapPerLayer + (kv ? TMG_VC : TMG_KC);
      std::memcpy(image.data() + (P.off_tmap - P.off_families) + (size_t)index * kTmapBytes, &m, sizeof(m));
    }
  }
  if (P.wide) {
    // wide batch: every matrix in boxes of 64 columns x 128 rows (a tcgen05
    // A operand per box), the activations in boxes of 64 columns x all their rows
    const int g0 = P.n_layers * kTmapPerLayer;
    for (int l = 0; l < P.n_layers; ++l) {
      const LayerPtrs& lp = layers[l];
      if (!put_sw128(tmap_index(l, TM_WQ), lp.wq, (long long)Hq * D, H, kWideRows, "wq") ||
          !put_sw128(tmap_index(l, TM_WK), lp.wk, (long long)Hkv * D, H, kWideRows, "wk") ||
          !put_sw128(tmap_index(l, TM_WV), lp.wv, (long long)Hkv * D, H, kWideRows, "wv") ||
          !put_sw128(tmap_index(l, TM_WO), lp.wo, H, (long long)Hq * D, kWideRows, "wo"))
        return false;
      if (P.kind == MK_MODEL_DENSE &&  // (an MoE decoder's entries hold its expert maps)
          (!put_sw128(tmap_index(l, TM_GATE), lp.w_gate, F, H, kWideRows, "w_gate") ||
           !put_sw128(tmap_index(l, TM_UP), lp.w_up, F, H, kWideRows, "w_up") ||
           !put_sw128(tmap_index(l, TM_DOWN), lp.w_down, H, F, kWideRows, "w_down")))
        return false;
    }
    const int ar = act_buf_rows(P.act_split, P.act_rows);  // (value and remainder rows with the split)
    return put_sw128(g0 + TMG_LM, P.lm_head, P.vocab, H, kWideRows, "lm_head") &&
           put_sw128(g0 + TMG_XN, ws + P.off_xn, ar, H, ar, "normalised activations") &&
           put_sw128(g0 + TMG_ATTN, ws + P.off_attn_bf, ar, H, ar, "attention output") &&
           (P.kind != MK_MODEL_DENSE || put_sw128(g0 + TMG_H, ws + P.off_h_bf, ar, F, ar, "SwiGLU output"));
  }
  for (int l = 0; l < P.n_layers; ++l) {
    const LayerPtrs& lp = layers[l];
    const int bh = H / kGemvSlots;  // columns per slot of a hidden-wide row
    if (!put(tmap_index(l, TM_WQ), lp.wq, (long long)Hq * D, H, H, bh, P.tile_qkv / 2, "wq") ||
        !put(tmap_index(l, TM_WK), lp.wk, (long long)Hkv * D, H, H, bh, P.tile_qkv / 2, "wk") ||
        !put(tmap_index(l, TM_WV), lp.wv, (long long)Hkv * D, H, H, bh, P.tile_qkv / 2, "wv") ||
        !put(tmap_index(l, TM_WO), lp.wo, H, (long long)Hq * D, (long long)Hq * D, bh, P.tile_o, "wo"))
      return false;
    if (P.kind == MK_MODEL_DENSE &&
        (!put(tmap_index(l, TM_GATE), lp.w_gate, F, H, H, bh, std::min(32, P.tile_gu), "w_gate") ||
         !put(tmap_index(l, TM_UP), lp.w_up, F, H, H, bh, std::min(32, P.tile_gu), "w_up") ||
         !put(tmap_index(l, TM_DOWN), lp.w_down, H, F, F, P.kseg / kGemvSlots, std::min(32, P.tile_down), "w_down")))
      return false;
  }
  return put(tmap_index(P.n_layers, 0), P.lm_head, P.vocab, H, H, H / kGemvSlots, 32, "lm_head");
}

// The dynamic shared-memory limit is an attribute of the kernel function, and
// plans of one kernel instance may need different sizes (the staging buffer
// depends on max_batch): set it for the plan being launched when another plan
// left a different value (one table entry per device and instance).
static cudaError_t ensure_smem_attr(int device, const void* kern, int smem) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<int, const void*>, int>> set;
  std::lock_guard<std::mutex> lock(mu);
  for (auto& e : set)
    if (e.first.first == device && e.first.second == kern) {
      if (e.second == smem) return cudaSuccess;
      cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (r == cudaSuccess) e.second = smem;
      return r;
    }
  cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (r == cudaSuccess) set.push_back({{device, kern}, smem});
  return r;
}

mk_status dev_bind(Plan& p, void* ws, size_t bytes, void* stream, const std::vector<unsigned char>& image_in,
                   std::string& err) {
  cudaStream_t s = (cudaStream_t)stream;
  std::vector<unsigned char> image = image_in;
  if (!encode_weight_maps(p.dp, (const unsigned char*)ws, image, err)) return MK_ERR_INVALID_ARG;
  size_t smem = (size_t)p.dp.ring_slots * p.dp.slot_bytes + kSmemFixed + p.dp.act_bytes + p.dp.gred_bytes +
                seq_table_bytes(p.dp);
  const void* kern = kernel_for(p.dp);
  cudaError_t e = ensure_smem_attr(p.device, kern, (int)smem);
  if (e == cudaSuccess) {
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, smem);
    if (e == cudaSuccess && nb < 1) { err = "megakernel does not fit on an SM"; return MK_ERR_UNSUPPORTED; }
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync((unsigned char*)ws + p.dp.off_families, image.data(), image.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync((unsigned char*)ws + p.dp.off_control, 0, sizeof(Control), s);
  // a queue entry counts as published when its tag equals the launch epoch, and
  // epochs restart at 1 here: clear whatever the memory held before
  if (e == cudaSuccess)
    e = cudaMemsetAsync((unsigned char*)ws + p.dp.off_queue, 0, sizeof(QRange) * (size_t)p.dp.queue_ranges, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) { err = std::string("bind failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.dp.smem_bytes = (int)smem;
  p.epoch = 0;
  return MK_OK;
}

// the decode step's debug captures (the MoE decoder's routing captures use the
// MoE layer's debug outputs, one block per layer)
static void set_captures(StepParams& sp, const mk_step_args* a) {
  sp.cap_resid = a->capture_resid;
  sp.cap_moe_in = reinterpret_cast<__nv_bfloat16*>(a->capture_moe_in);
  sp.dbg_idx = a->capture_topk;
  sp.dbg_hist = a->capture_hist;
  sp.dbg_indptr = a->capture_indptr;
}

mk_status dev_launch(Plan& p, const mk_step_args* a, void* stream, std::string& err) {
  StepParams sp = StepParams();
  sp.B = a->batch;
  sp.tokens = a->token_ids;
  sp.slots = a->slot_ids;
  sp.ctx = a->ctx_lens;
  sp.logits = a->logits;
  sp.next_tokens = a->next_tokens;
  sp.task_counts = a->task_counts;
  sp.trace = (p.dp.debug_flags & MK_DEBUG_TRACE) ? (uint32_t*)a->trace : nullptr;
  sp.trace_cap = a->trace_cap;
  if (sp.trace && sp.trace_cap < 2) sp.trace = nullptr;
  set_captures(sp, a);
  sp.epoch = p.epoch + 1;
  unsigned char* ws = (unsigned char*)p.ws;
  DevPlan dp = p.dp;
  void* args[] = {(void*)&dp, (void*)&sp, (void*)&ws};
  cudaError_t e = ensure_smem_attr(p.device, kernel_for(p.dp), p.dp.smem_bytes);
  if (e == cudaSuccess)
    e = cudaLaunchCooperativeKernel(kernel_for(p.dp), dim3(p.dp.n_sm), dim3(kThreads), args,
                                    (size_t)p.dp.smem_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) { err = std::string("launch failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.epoch++;
  p.launches++;
  return MK_OK;
}

// ---------------------------------------------------------------- static scratch
// Scratch of mk_decode_step_static: a module-scope device array, so that the
// step needs no device allocation at all.  Each CUDA context (one per device)
// holds its own copy of it.  The array is shared by every plan and call on the
// device and keeps the last call's contents; g_static records whose plan
// arrays it holds, so they are uploaded again only when the plan changes.
static __device__ __align__(256) unsigned char g_static_scratch[MK_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxStaticDevices = 64;
struct StaticScratchState {
  unsigned char* addr = nullptr;  // device address of g_static_scratch in this device's context
  unsigned long long owner = 0;   // uid of the plan whose arrays it holds (0: none)
};
std::mutex g_static_mu;
StaticScratchState g_static[kMaxStaticDevices];
}  // namespace

mk_status dev_launch_static(Plan& p, const mk_step_args* a, void* stream, std::string& err) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) { err = std::string("cudaGetDevice failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  if (dev != p.device) { err = "the current device is not the one the plan was built on"; return MK_ERR_INVALID_ARG; }
  if (dev < 0 || dev >= kMaxStaticDevices) { err = "device ordinal beyond the static-scratch table"; return MK_ERR_UNSUPPORTED; }
  const DevPlan& P0 = p.dp;
  if ((unsigned long long)P0.ws_bytes > (unsigned long long)MK_STATIC_SCRATCH_BYTES) {
    err = "plan scratch exceeds MK_STATIC_SCRATCH_BYTES";
    return MK_ERR_WORKSPACE;
  }

  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticScratchState& st = g_static[dev];
  // the array's address in this device's context, resolved on every call (a
  // reset of the context reloads the module, possibly at another address, and
  // then the plan arrays must be uploaded again)
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_static_scratch);
  if (e != cudaSuccess) {
    err = std::string("cudaGetSymbolAddress of the static scratch failed: ") + cudaGetErrorString(e);
    return MK_ERR_CUDA;
  }
  if (st.addr != static_cast<unsigned char*>(ptr)) {
    st.addr = static_cast<unsigned char*>(ptr);
    st.owner = 0;
  }
  cudaStream_t s = (cudaStream_t)stream;
  unsigned char* ws = st.addr;
  const size_t smem = (size_t)P0.ring_slots * P0.slot_bytes + kSmemFixed + P0.act_bytes + P0.gred_bytes +
                      seq_table_bytes(P0);
  if (st.owner != p.uid) {
    st.owner = 0;
    e = ensure_smem_attr(p.device, kernel_for(P0), (int)smem);
    if (e == cudaSuccess) {
      int nb = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel_for(P0), kThreads, smem);
      if (e == cudaSuccess && nb < 1) { err = "megakernel does not fit on an SM"; return MK_ERR_UNSUPPORTED; }
    }
    // the read-only plan arrays and the weights' tensor maps (host memory only)
    std::vector<unsigned char> image;
    lower_plan(p, image);
    if (!encode_weight_maps(P0, ws, image, err)) return MK_ERR_INVALID_ARG;
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(ws + P0.off_families, image.data(), image.size(), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) { err = std::string("plan upload failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
    st.owner = p.uid;
  }
  // every call starts at epoch 1 from a cleared control block and queue; the
  // counters, activations and argmax keys are set by the kernel's prologue
  e = cudaMemsetAsync(ws + P0.off_control, 0, sizeof(Control), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws + P0.off_queue, 0, sizeof(QRange) * (size_t)P0.queue_ranges, s);
  if (e != cudaSuccess) { err = std::string("scratch clear failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }

  StepParams sp = StepParams();
  sp.B = a->batch;
  sp.tokens = a->token_ids;
  sp.slots = a->slot_ids;
  sp.ctx = a->ctx_lens;
  sp.logits = a->logits;
  sp.next_tokens = a->next_tokens;
  sp.task_counts = a->task_counts;
  sp.trace = (P0.debug_flags & MK_DEBUG_TRACE) ? (uint32_t*)a->trace : nullptr;
  sp.trace_cap = a->trace_cap;
  if (sp.trace && sp.trace_cap < 2) sp.trace = nullptr;
  set_captures(sp, a);
  sp.epoch = 1;
  DevPlan dp = P0;
  dp.smem_bytes = (int)smem;
  void* args[] = {(void*)&dp, (void*)&sp, (void*)&ws};
  e = ensure_smem_attr(p.device, kernel_for(p.dp), (int)smem);
  if (e == cudaSuccess) e = cudaLaunchCooperativeKernel(kernel_for(p.dp), dim3(dp.n_sm), dim3(kThreads), args, smem, s);
  if (e != cudaSuccess) { err = std::string("launch failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.launches++;
  return MK_OK;
}

mk_status dev_launch_moe(Plan& p, const mk_moe_args* a, void* stream, std::string& err) {
  StepParams sp = StepParams();
  sp.B = a->n_tokens;
  sp.moe_x = reinterpret_cast<const __nv_bfloat16*>(a->x);
  sp.moe_out = reinterpret_cast<__nv_bfloat16*>(a->out);
  sp.dbg_idx = a->topk_idx;
  sp.dbg_w = a->topk_w;
  sp.dbg_hist = a->hist;
  sp.dbg_indptr = a->indptr;
  sp.dbg_logits = a->logits;
  sp.task_counts = a->task_counts;
  sp.epoch = p.epoch + 1;
  unsigned char* ws = (unsigned char*)p.ws;
  DevPlan dp = p.dp;
  void* args[] = {(void*)&dp, (void*)&sp, (void*)&ws};
  cudaError_t e = ensure_smem_attr(p.device, kernel_for(p.dp), p.dp.smem_bytes);
  if (e == cudaSuccess)
    e = cudaLaunchCooperativeKernel(kernel_for(p.dp), dim3(p.dp.n_sm), dim3(kThreads), args,
                                              (size_t)p.dp.smem_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) { err = std::string("launch failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.epoch++;
  p.launches++;
  return MK_OK;
}

mk_status dev_status(Plan& p, mk_device_status* st, std::string& err) {
  Control c;
  cudaError_t e = cudaMemcpy(&c, (unsigned char*)p.ws + p.dp.off_control, sizeof(c), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) { err = std::string("status read failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  st->code = c.status_code;
  st->family = c.status_code ? c.status_family : -1;
  st->index = c.status_code ? c.status_index : -1;
  st->event = c.status_code ? c.status_event : -1;
  st->sm = c.status_code ? c.status_sm : -1;
  return c.status_code;
}

mk_status dev_reset(Plan& p, void* stream, std::string& err) {
  cudaError_t e = cudaMemsetAsync((unsigned char*)p.ws + p.dp.off_control, 0, sizeof(Control), (cudaStream_t)stream);
  // epochs restart at 1: entries tagged by the old epochs must not read as published
  if (e == cudaSuccess)
    e = cudaMemsetAsync((unsigned char*)p.ws + p.dp.off_queue, 0, sizeof(QRange) * (size_t)p.dp.queue_ranges,
                        (cudaStream_t)stream);
  if (e != cudaSuccess) { err = std::string("reset failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.epoch = 0;
  return MK_OK;
}

}  // namespace mk
