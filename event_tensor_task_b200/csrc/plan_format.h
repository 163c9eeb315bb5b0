// plan_format.h — the lowered plan as the megakernel reads it, plus the
// symbolic-expression bytecode and the task-index decoding that the host
// compiler and the device interpreter share.
//
// Symbolic extents follow "Event Tensor: A Unified Abstraction for Compiling
// Dynamic Megakernel", section "Core method" (shape dynamism: event-tensor
// dimensions may be symbolic, e.g. the batch size B, and one runtime is
// instantiated from the actual values) and "Lecture 112: Production
// Megakernels for Real-World Inference", section "Symbolic Representation of
// Work" (extents and barriers are expressions in the runtime sizes, so the
// work queue is never rebuilt).  Every extent and every wait count is a small
// postfix program over the symbols B (batch), ctx[b] (per-sequence context)
// and the coordinates of the event element being armed.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define MK_HD __host__ __device__ __forceinline__
#else
#define MK_HD inline
#endif

namespace mk {

// ---------------------------------------------------------------- ops
enum Op : int32_t {
  OP_END = 0,
  OP_QKV = 1,     // RMSNorm -> Q/K/V rows -> RoPE -> KV append
  OP_ATTN = 2,    // one key chunk of one (sequence, kv head) -> softmax partials
  OP_MERGE = 3,   // (reserved: a pair's last attention task merges its partials)
  OP_OPROJ = 4,   // output projection rows + residual
  OP_GATEUP = 5,  // RMSNorm -> gate and up rows -> SwiGLU
  OP_DOWN = 6,    // down projection rows over one K segment -> partial
  OP_NORM = 7,    // wide batch, one row: residual (x + down partials) -> x, RMSNorm(x) * attn gain -> bf16
  OP_LM = 8,      // final RMSNorm -> vocabulary rows -> logits + running argmax
  OP_NORM2 = 9,   // wide batch, one row: RMSNorm(x) * FFN gain -> bf16
  OP_LMFIN = 10,  // follow-up: the running argmax -> next token
  // mixture-of-experts FFN layer (data-dependent task graph, dynamic schedule)
  OP_ROUTE = 11,    // 8 tokens: router logits -> top-k, weights, per-expert ranks
  OP_MINDPTR = 12,  // follow-up: exp_indptr, tile table, row map, data-dependent counts
  OP_EGU = 13,      // GroupGEMM tile: an expert's gate/up rows x its routed rows -> SwiGLU
  OP_EDOWN = 14,    // GroupGEMM tile: an expert's down rows x its routed rows
  OP_COMBINE = 15,  // 8 tokens: weighted sum of their top-k expert outputs
  OP_MFIN = 16,     // follow-up: end of the layer
  OP_NORMF = 17,    // wide batch, one row: final residual, RMSNorm * final gain -> bf16
  OP_COUNT = 18
};

// ---------------------------------------------------------------- expressions
// Postfix bytecode; every program ends with X_RET.  X_SUM_B len sums the
// next `len` words (a program without X_SUM_B, ended by X_RET) over
// b = 0..B-1 with X_VAR pushing b.
enum XOp : int32_t {
  X_RET = 0,
  X_PUSH = 1,     // operand follows
  X_B = 2,        // batch size
  X_COORD = 3,    // operand d: coordinate d of the element being evaluated
  X_CTX_AT = 4,   // pop i; push ctx[i] (0 when i >= B)
  X_VAR = 5,      // loop variable of the enclosing X_SUM_B
  X_ADD = 6, X_SUB = 7, X_MUL = 8,
  X_CEILDIV = 9,  // pop d, a; push ceil(a / d)
  X_MIN = 10, X_MAX = 11,
  X_LT = 12,      // pop b, a; push a < b
  X_SUM_B = 13,   // operand len; body of len words follows
  X_ASPLIT = 14,  // the step's key chunks per attention task (step_attn_split)
};

struct ExprEnv {
  int B;
  const int* ctx;   // [B]
  int coord[3];
  int asplit;       // key chunks per attention task in this step
};

MK_HD int expr_flat(const int32_t* code, int pc, const ExprEnv& env, int var) {
  int st[12];
  int sp = 0;
  for (;;) {
    int op = code[pc++];
    switch (op) {
      case X_RET: return sp > 0 ? st[sp - 1] : 0;
      case X_PUSH: st[sp++] = code[pc++]; break;
      case X_B: st[sp++] = env.B; break;
      case X_COORD: st[sp++] = env.coord[code[pc++]]; break;
      case X_CTX_AT: { int i = st[sp - 1]; st[sp - 1] = (i >= 0 && i < env.B) ? env.ctx[i] : 0; } break;
      case X_VAR: st[sp++] = var; break;
      case X_ASPLIT: st[sp++] = env.asplit; break;
      case X_ADD: sp--; st[sp - 1] = st[sp - 1] + st[sp]; break;
      case X_SUB: sp--; st[sp - 1] = st[sp - 1] - st[sp]; break;
      case X_MUL: sp--; st[sp - 1] = st[sp - 1] * st[sp]; break;
      case X_CEILDIV: sp--; st[sp - 1] = (st[sp - 1] + st[sp] - 1) / st[sp]; break;
      case X_MIN: sp--; st[sp - 1] = st[sp - 1] < st[sp] ? st[sp - 1] : st[sp]; break;
      case X_MAX: sp--; st[sp - 1] = st[sp - 1] > st[sp] ? st[sp - 1] : st[sp]; break;
      case X_LT: sp--; st[sp - 1] = st[sp - 1] < st[sp] ? 1 : 0; break;
      default: return -1;
    }
  }
}

MK_HD int expr_eval(const int32_t* code, int pc, const ExprEnv& env) {
  int st[12];
  int sp = 0;
  for (;;) {
    int op = code[pc++];
    switch (op) {
      case X_RET: return sp > 0 ? st[sp - 1] : 0;
      case X_PUSH: st[sp++] = code[pc++]; break;
      case X_B: st[sp++] = env.B; break;
      case X_COORD: st[sp++] = env.coord[code[pc++]]; break;
      case X_CTX_AT: { int i = st[sp - 1]; st[sp - 1] = (i >= 0 && i < env.B) ? env.ctx[i] : 0; } break;
      case X_ASPLIT: st[sp++] = env.asplit; break;
      case X_ADD: sp--; st[sp - 1] = st[sp - 1] + st[sp]; break;
      case X_SUB: sp--; st[sp - 1] = st[sp - 1] - st[sp]; break;
      case X_MUL: sp--; st[sp - 1] = st[sp - 1] * st[sp]; break;
      case X_CEILDIV: sp--; st[sp - 1] = (st[sp - 1] + st[sp] - 1) / st[sp]; break;
      case X_MIN: sp--; st[sp - 1] = st[sp - 1] < st[sp] ? st[sp - 1] : st[sp]; break;
      case X_MAX: sp--; st[sp - 1] = st[sp - 1] > st[sp] ? st[sp - 1] : st[sp]; break;
      case X_LT: sp--; st[sp - 1] = st[sp - 1] < st[sp] ? 1 : 0; break;
      case X_SUM_B: {
        int len = code[pc++];
        int s = 0;
        for (int b = 0; b < env.B; ++b) s += expr_flat(code, pc, env, b);
        st[sp++] = s;
        pc += len;
      } break;
      default: return -1;
    }
  }
}

// ---------------------------------------------------------------- lowered plan
// Event-tensor slots of the dense decoder (index into DevPlan::ev).
enum EvId : int32_t {
  EV_IN = 0,     // [L+1]        layer input ready (element l+1 notified by layer l's down tiles)
  EV_QKV = 1,    // [L][Hkv]     Q/K/V rows of one kv-head group written
  EV_CHUNK = 2,  // (unused: armed at one element of count zero)
  EV_ATTN = 3,   // [L]          every attention task done (each pair merged by its last task)
  EV_O = 4,      // [L]          output projection done
  EV_GU = 5,     // [L][n_kc]    SwiGLU outputs of one K segment written
  EV_LM = 6,     // [1]          all LM tiles done
  // MoE layer
  // (one element per MoE layer: [1] for the MoE-layer plan, [L] for the MoE decoder)
  EV_ROUTE = 7,  // [Lm]            all ROUTE tasks done
  EV_MIDX = 8,   // [Lm]            exp_indptr and the tile table written
  EV_MH = 9,     // [Lm][max_tiles] SwiGLU rows of one GroupGEMM tile written (all its gate/up tasks)
  EV_MY = 10,    // [Lm]            all down tasks done (count set at run time from exp_indptr)
  EV_MCOMB = 11, // [Lm]            all COMBINE tasks done (the layer's residual is updated)
  // wide batch (max_batch > 8): the normalised activations are materialised
  EV_N1 = 12,    // [L]  layer input normalised (bf16) and the residual materialised
  EV_N2 = 13,    // [L]  FFN input normalised
  EV_NF = 14,    // [1]  final norm done
  EV_COUNT = 15
};

struct EventTensorDesc {
  int32_t base;        // first counter of this tensor in the counter array
  int32_t ndim;
  int32_t dims[3];     // maximum extents
  int32_t count_expr;  // wait count of an element, a program over its coordinates
};

struct FamilyDesc {
  int32_t op;
  int32_t layer;       // -1 for the LM families
  int32_t extent_expr; // number of tasks, a program over B and ctx
  int32_t max_extent;
  int32_t debug_base;
  int32_t followup;    // 1: executed by the last notifier of its trigger event
  int32_t pad[2];
};

// One static-schedule instruction: this SM runs the contiguous block
// [v*ext/n, (v+1)*ext/n) of a family's tasks, ext being the family's
// evaluated extent (a contiguous block keeps a CTA's activation registers
// valid across its tasks).
struct Instr {
  int32_t family;
  int32_t v;  // this SM's virtual index for the family
  int32_t n;  // number of virtual SMs
  int32_t pad;
};

MK_HD void instr_range(const Instr& in, int ext, int& lo, int& hi) {
  lo = (int)(((long long)in.v * ext) / in.n);
  hi = (int)(((long long)(in.v + 1) * ext) / in.n);
}

struct LayerPtrs {
  const void* attn_norm; const void* wq; const void* wk; const void* wv; const void* wo;
  const void* ffn_norm; const void* w_gate; const void* w_up; const void* w_down;
  // MoE decoder: this layer's MoE FFN
  const void* w_router; const float* router_bias; const void* we_gate; const void* we_up; const void* we_down;
};

constexpr int kMaxFamilies = 256;
struct DevPlan;
// bytes of the per-sequence tables (ctx, slot, token, attention tasks and
// their prefix; max_batch ints each, one more for the prefix)
MK_HD int seq_table_bytes_for(int max_batch) { return ((5 * (max_batch > 0 ? max_batch : 1) + 1) * 4 + 127) / 128 * 128; }
// Dynamic shared memory of a CTA: the ring (ring_slots x slot_bytes), the
// kernel's fixed control area (at most kSmemFixed bytes), the staging buffer
// (act_bytes: the GEMV activation rows in bf16, kActPitch elements per batch
// row, or 8 KB of fp32 scratch for the other task bodies) and the GEMV
// partial tiles (gred_bytes: 8 warps x gbatch = 8 columns x 64 rows of fp32).
constexpr int kSmemFixed = 9 * 1024;
constexpr int kActPitch = 2048 + 8;  // bf16 elements per staged activation row (16-byte bank offset per row)
constexpr int kMaxBatchRows = 8;     // batch rows of a narrow step (the GEMV's MMA n = 8 columns)
constexpr int kMaxWideBatch = 64;    // batch rows of a wide step (tcgen05 GEMM tiles, N up to 64)
// wide batch: GEMM tasks of kWideRows weight rows (the tcgen05 MMA's M); the
// global tensor maps after the per-layer ones: the LM head, then the
// normalised activations, the attention output and the SwiGLU output (bf16)
constexpr int kWideRows = 128;
constexpr int kBStages = 3;  // wide batch: activation-chunk stages of the MMA issuer (in the staging buffer)
// global tensor maps: the LM head, the wide-batch activation buffers, and the
// K and V caches as [layer, slot, kv head][max_ctx][64] (one 64-key chunk per
// box, 128-byte swizzle)
enum TmapGlobal : int { TMG_LM = 0, TMG_XN, TMG_ATTN, TMG_H, TMG_KC, TMG_VC, kTmapGlobal };
// A GEMV task's weights arrive in kGemvSlots ring slots, slot j holding columns
// [j K / 8, (j + 1) K / 8) of all the task's rows (one 2-D TMA box per part),
// through one tensor map per dense weight matrix: matrix m of layer l at
// index l * kTmapPerLayer + m, the LM head after the last layer.
constexpr int kGemvSlots = 8;
constexpr int kTmapBytes = 128;
// Per layer: the dense matrices; in MoE plans TM_GATE / TM_UP / TM_DOWN map
// the layer's expert matrices ([E * F][H] and [E * H][F], boxes of 64 columns
// x 128 rows) and TM_XG / TM_HG the GroupGEMM activation buffers (the routed
// token rows per expert, the SwiGLU rows) in boxes of 64 columns x 16 or 64
// rows (the MoE-layer plan uses layer 0's entries).
enum TmapMatrix : int {
  TM_WQ = 0, TM_WK, TM_WV, TM_WO, TM_GATE, TM_UP, TM_DOWN, TM_XG16, TM_XG64, TM_HG16, TM_HG64,
  TM_XG128, TM_HG128, kTmapPerLayer
};
MK_HD int tmap_index(int layer, int m) { return layer * kTmapPerLayer + m; }
constexpr int kMaxBatch = 128;
// MoE GroupGEMM on tcgen05: a tile is kMoeTileRows routed rows of one expert;
// a task covers kMoeTaskRows weight rows (gate/up: that many gate rows and as
// many up rows; down: that many output rows), the MMA's M
constexpr int kMoeTileRows = 64;
constexpr int kMoeTaskRows = 128;
constexpr int kMoeBigTileRows = 128;  // routing-aware tiles: experts with more rows than kMoeTileRows
// Rows per GroupGEMM tile of an expert with h routed rows: with routing-aware
// tiles (moe_big), an expert holding more than kMoeTileRows rows gets tiles of
// kMoeBigTileRows, so its weights stream once per 128 rows instead of 64.
// wide batch: buffer row of batch row b's bf16 value (part 0) or of its bf16
// remainder v - value (part 1).  With the split, rows come in groups of 16:
// the values of batch rows 8g .. 8g + 7, then their remainders, so that one
// MMA with N = 16 * ceil(B / 8) columns multiplies both and the epilogue adds
// column pairs (8g + i, 16g + 8 + i -> batch row 8g + i).
MK_HD int act_buf_row(int split, int b, int part) { return split ? (b >> 3) * 16 + part * 8 + (b & 7) : b; }
// rows of an activation buffer (and of its TMA box)
MK_HD int act_buf_rows(int split, int act_rows) { return split ? 2 * act_rows : act_rows; }

MK_HD int moe_tile_rows(int h, int tm, int big) { return (big && h > tm) ? kMoeBigTileRows : tm; }

// A ROUTE task's use of the staging buffer: the router logits of its 8
// tokens ([8][64] fp32), then the tokens' bf16 input rows ([8][hidden]), read
// by every warp for every expert.  Plans with ROUTE tasks size the staging
// buffer to hold it.
constexpr int kRouteLogitBytes = 8 * 64 * 4;
MK_HD int route_stage_bytes(int hidden) { return kRouteLogitBytes + 8 * hidden * 2; }
constexpr int kTmemCols = 256;  // TMEM columns a CTA of an MoE plan allocates

// Fixed header of the plan; passed to the kernel by value.  Offsets are in
// bytes from the workspace base.
struct DevPlan {
  int32_t sched, n_sm, n_families, n_instr_per_sm;
  int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  int32_t max_batch, max_ctx, n_slots;
  float eps;
  int32_t tile_qkv, tile_o, tile_gu, tile_down, kseg, tile_lm, chunk;
  int32_t n_qkv_tiles, n_otiles, n_gutiles, n_dtiles, n_kc, n_lm_tiles, max_chunks;
  int32_t ring_slots, slot_bytes, smem_bytes;
  int32_t act_bytes, gred_bytes, gbatch, pad3;  // shared-memory staging buffer and partial tiles
  int32_t n_counters, debug_slots, queue_ranges;
  uint32_t debug_flags;
  int32_t fault_ctr;  // fault injection: this counter is armed one above its count (-1: none)
  int64_t spin_timeout_ns;
  EventTensorDesc ev[EV_COUNT];
  int32_t fam_first_layer[OP_COUNT];  // family index of (op, layer 0), or of the op for LM families
  int32_t fam_stride;                 // families per layer
  int32_t pad1;
  // workspace offsets
  int64_t off_control, off_counters, off_families, off_expr, off_instr, off_layers, off_rope;
  int64_t off_queue, off_x, off_q, off_apart, off_attn, off_h, off_dpart, off_lmbest;
  int64_t off_tmap;  // TMA tensor maps of the dense weights (kTmapBytes each, see tmap_index)
  int64_t ws_bytes;
  // global weights (device)
  const void* embed; const void* lm_head; const void* final_norm;
  void* k_cache; void* v_cache;
  // MoE layer (kind MK_MODEL_MOE_LAYER) and MoE decoder (MK_MODEL_MOE_DECODER)
  int32_t kind;
  int32_t n_experts, top_k, eff, max_tokens;
  int32_t moe_tm;     // routed rows per GroupGEMM tile
  int32_t moe_tn;     // gate/up row pairs per EGU task
  int32_t moe_td;     // down rows per EDOWN task
  int32_t nt_gu, nt_d, max_tiles;
  int32_t pad2;
  const void* w_router; const float* router_bias;
  const void* w_egate; const void* w_eup; const void* w_edown;
  // MoE scratch: one block per MoE layer, moe_stride bytes apart; the offsets
  // below are those of layer 0's block (the MoE-layer plan has one block)
  int64_t moe_stride;
  int64_t off_mhist, off_mrank, off_midx, off_mw, off_mindptr, off_mtile, off_mtile_e, off_mtile_m;
  int64_t off_mperm, off_mrow, off_mh, off_my, off_mxhat;
  int64_t off_mxg;  // routed token rows, bf16 [E][moe_cap][H] (row = the pair's rank in its expert)
  int32_t moe_cap;  // rows per expert in off_mxg (the plan's token maximum)
  int32_t moe_big;  // routing-aware tiles (see moe_tile_rows)
  int32_t pad5;
  // wide batch: tcgen05 GEMM tasks on materialised bf16 activations
  int32_t wide;       // 1: max_batch > kMaxBatchRows
  int32_t attn_split; // key chunks per attention task (adaptive plans: at most; see step_attn_split)
  int32_t act_rows;   // batch rows of the activation buffers (max_batch rounded up to 16)
  int32_t act_split;  // 1: each activation row stored as its bf16 value and its bf16 remainder (see act_buf_row)
  int64_t off_xn, off_attn_bf, off_h_bf;  // bf16 [max_batch][H], [max_batch][H], [max_batch][F]
  // wide batch, split K: QKV, O-projection and gate/up tiles run as gseg_*
  // tasks over consecutive K segments; each writes its fp32 partial tile to
  // off_gpart and counts in at the tile's counter (off_gctr, [3][64]); the
  // last to count in sums the partials in segment order and runs the
  // tile's epilogue (the counters are zeroed at launch and by that task)
  int32_t gseg_qkv, gseg_o, gseg_gu;
  int32_t attn_auto;  // 1: the attention split follows each step's B and contexts (step_attn_split; wide plans: steps of at most kMaxBatchRows rows)
  int64_t off_gpart, off_gctr;
  // attention: per (sequence, kv head) count of finished tasks; the last of a
  // pair's tasks merges their partials (zeroed at launch and by that task)
  int64_t off_actr;
};
constexpr int kGctrPerOp = 64;  // split-K tile counters per GEMM op (tiles of 128 rows)

MK_HD int seq_table_bytes(const DevPlan& P) { return seq_table_bytes_for(P.max_batch); }

// Control block at off_control (first 256 bytes of the workspace).
struct Control {
  int32_t status_code, status_family, status_index, status_event, status_sm;
  int32_t abort;
  uint32_t grid_bar;        // monotonic grid-barrier arrivals
  uint32_t pad0;
  unsigned long long q_tail;  // dynamic queue: (ranges << 40) | tasks reserved
  unsigned long long q_head;  // dynamic queue: tasks popped
  int32_t pad[52];
};

// Dynamic queue entry: a contiguous range of tasks of one family.
struct QRange {
  int32_t family;
  int32_t lo;          // first task index
  int32_t count;
  uint32_t seq;        // (epoch << 20 | range index) + 1 once published
  unsigned long long start;  // ticket of the first task of the range
};

// ---------------------------------------------------------------- task decoding
// QKV tile i covers rows j0..j0+R/2-1 and j0+D/2.. of head hh (q heads, then
// k heads, then v heads); R = tile_qkv, rotate-half pairs stay in one tile.
struct QkvTile { int hh; int kind; int head; int group; int j0; };
MK_HD QkvTile decode_qkv(const DevPlan& P, int i) {
  QkvTile t;
  int per_head = P.head_dim / P.tile_qkv;
  t.hh = i / per_head;
  t.j0 = (i % per_head) * (P.tile_qkv / 2);
  int qpg = P.n_q_heads / P.n_kv_heads;
  if (t.hh < P.n_q_heads) { t.kind = 0; t.head = t.hh; t.group = t.hh / qpg; }
  else if (t.hh < P.n_q_heads + P.n_kv_heads) { t.kind = 1; t.head = t.hh - P.n_q_heads; t.group = t.head; }
  else { t.kind = 2; t.head = t.hh - P.n_q_heads - P.n_kv_heads; t.group = t.head; }
  return t;
}

// ATTN task i -> (b, g, c) given per-sequence task counts nch[] (key chunks
// grouped attn_split at a time) and their exclusive prefix pre[] (index =
// Hkv * pre[b] + g * nch[b] + c).
struct AttnTask { int b, g, c; };
MK_HD AttnTask decode_attn(int i, int B, int Hkv, const int* nch, const int* pre) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {  // largest b with Hkv * pre[b] <= i
    int mid = (lo + hi + 1) >> 1;
    if (Hkv * pre[mid] <= i) lo = mid; else hi = mid - 1;
  }
  AttnTask t;
  t.b = lo;
  int r = i - Hkv * pre[lo];
  t.g = r / nch[lo];
  t.c = r % nch[lo];
  return t;
}

MK_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Key chunks per attention task in one step.  A plan with a fixed split
// (attn_auto = 0) returns attn_split, and so does a wide-batch plan at a step
// of more than kMaxBatchRows rows.  Otherwise the step's
// C = Hkv * sum_b ceil((ctx_b + 1) / chunk) chunk units are cut into about two
// thirds of n_sm tasks: s = ceil(C / ceil(2 n_sm / 3)), clamped to
// [min(kAttnSplitMin, attn_split), attn_split].  (Measured on the 1B shape at
// B = 1..8: fewer, longer tasks leave SMs idle; more tasks than that pay a
// second wave and more merging; below 3 chunks a task's fixed costs dominate.)
constexpr int kAttnSplitMin = 3;
MK_HD int step_attn_split(const DevPlan& P, int B, const int* ctx) {
  if (!P.attn_auto || (P.wide && B > kMaxBatchRows)) return P.attn_split;
  long long c = 0;
  for (int b = 0; b < B; ++b) c += ceil_div(ctx[b] + 1, P.chunk);
  c *= P.n_kv_heads;
  const long long target = ceil_div(2 * P.n_sm, 3);
  const long long s = (c + target - 1) / target;
  const int lo = P.attn_split < kAttnSplitMin ? P.attn_split : kAttnSplitMin;
  return s < lo ? lo : s > P.attn_split ? P.attn_split : (int)s;
}

}  // namespace mk
