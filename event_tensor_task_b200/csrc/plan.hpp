// plan.hpp — host task-graph compiler for the decode megakernel.
//
// Builds, from a model description, the task families (tiles of every op,
// with symbolic extents), the Event Tensors (shapes and symbolic wait
// counts), the static per-SM instruction queues and the dynamic successor
// rules, and lowers them into the flat arrays the device interpreter reads
// ("Event Tensor: A Unified Abstraction for Compiling Dynamic Megakernel",
// section "Core method": event tensors as first-class compiler objects,
// static and dynamic scheduling transformations, lowering of events to plain
// integer counters).
#pragma once
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "plan_format.h"

namespace mk {

// Host-side record of one task for one binding of the symbols.
enum Buf : int {
  BUF_X = 0, BUF_Q, BUF_KC, BUF_VC, BUF_APART, BUF_ATTN, BUF_H, BUF_DPART,
  BUF_LOGITS, BUF_NEXT,
  // MoE scratch, one block per MoE layer: the layer input rows (bf16), the
  // per-pair routing records (expert, weight, rank), the tables the routing
  // follow-up writes (exp_indptr, tile table, row map), the SwiGLU rows and
  // the expert output rows of the grouped problem, the layer output
  BUF_MXHAT, BUF_MPAIR, BUF_MTAB, BUF_MH, BUF_MY, BUF_MOUT,
  BUF_MXG,  // the routed token rows per expert (row = the pair's rank in its expert)
  BUF_XN,   // wide batch: the normalised activation rows (bf16)
  BUF_COUNT
};

struct Region {
  int buf;
  long long lo, hi;  // element range [lo, hi)
};

struct TaskRec {
  int fam = -1;
  int idx = -1;
  int wait_ev = -1;       // counter index waited on (-1: none)
  int notify_ev = -1;     // counter index decremented at completion (-1: none)
  int follow_fam = -1;    // follow-up family run by the notifier that reaches zero
  int follow_idx = -1;
  bool exists = true;     // false: an index of the family this binding does not run (a merge of a
                          // (sequence, kv head) whose chunks fit one attention task)
  std::vector<Region> reads, writes;
};

// Routing of one MoE layer call for the host model: the top-k experts of
// every (token, slot) pair, and what the routing follow-up derives from them.
struct MoeRoute {
  std::vector<int> idx;      // [T * k]
  std::vector<int> hist;     // [E]
  std::vector<int> indptr;   // [E + 1], exclusive prefix sum of hist
  std::vector<int> tile_e, tile_m;  // GroupGEMM tile -> (expert, m block)
  std::vector<int> rank;     // [T * k]: the pair's row among its expert's rows (ascending (t, j) here)
  int tiles = 0;
};

struct Binding {
  int B;
  std::vector<int> ctx;
  std::vector<MoeRoute> route;  // one per MoE layer (empty for a dense plan)
};

struct Plan {
  mk_model_desc m{};
  std::vector<mk_layer_weights> layer_w;
  mk_plan_opts o{};
  DevPlan dp{};
  std::vector<FamilyDesc> fams;
  std::vector<std::string> fam_names;
  std::vector<int32_t> code;
  std::vector<Instr> instr;         // [n_sm][n_instr_per_sm]
  std::vector<LayerPtrs> layers;
  std::vector<float> rope;          // [max_ctx][head_dim/2][2] cos, sin
  int device = -1;
  unsigned long long uid = 0;       // unique per plan built in this process
  void* ws = nullptr;
  size_t ws_bound = 0;
  unsigned epoch = 0;
  long long launches = 0;
  double build_ms = 0.0;             // host time of mk_plan_build

  // host model of the task graph
  int fam_index(int op, int layer) const;
  int counter(int ev, int c0, int c1 = 0, int c2 = 0) const;
  int event_count(int ev, int c0, int c1, int c2, const Binding& bd) const;
  int family_extent(int f, const Binding& bd) const;
  // extent of a family in a step: the symbolic extent, or for the GroupGEMM
  // families the number of tasks the binding's routing creates
  int actual_extent(int f, const Binding& bd) const;
  void task(int f, int idx, const Binding& bd, TaskRec& t) const;
  // dynamic successors of a counter that reached zero: (family, lo, count) ranges
  void successors(int counter_index, const Binding& bd, std::vector<int>& out3) const;
  int total_counters() const { return dp.n_counters; }
};

// Build; returns MK_OK or an error with `err` set.
mk_status build_plan(const mk_model_desc* m, const mk_plan_opts* o, int n_sm, int smem_bytes,
                     Plan& p, std::string& err);
mk_status validate_plan(const Plan& p, const Binding& bd, std::string& err);
mk_status simulate_plan(const Plan& p, const Binding& bd, int n_orders, unsigned seed, int fault,
                        int fault_family, mk_sim_report* rep);
double step_bytes(const Plan& p, const Binding& bd, bool with_logits);
// A seeded routing for every MoE layer of the plan on the binding's B tokens
// (k distinct experts per token; `skew` > 0 draws experts with weights
// (rank + 1)^-skew over a seeded expert order), with its histogram,
// exp_indptr and GroupGEMM tiles.
void draw_routing(const Plan& p, Binding& bd, unsigned seed, double skew);

// Lowered plan image (families, expressions, instructions, layer pointers,
// rope table) with the offsets recorded in p.dp.
void lower_plan(Plan& p, std::vector<unsigned char>& image);

}  // namespace mk
