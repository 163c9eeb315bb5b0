// plan.cpp — host task-graph compiler, validator and plan simulator.
//
// The graph of one dense decode step, per layer l (events in brackets):
//   QKV tiles        wait EV_IN[l]        notify EV_QKV[l][g]
//   ATTN chunks      wait EV_QKV[l][g]    notify EV_ATTN[l] (the pair's last task merges)
//   OPROJ tiles      wait EV_ATTN[l]      notify EV_O[l]
//   GATEUP tiles     wait EV_O[l]         notify EV_GU[l][kc]
//   DOWN tiles       wait EV_GU[l][kc]    notify EV_IN[l+1]
// The residual after layer l's FFN is never materialised: it is the residual
// after the attention block (X, updated in place by OPROJ) plus the sum of
// layer l's K-segment partials of the down projection, and every reader of
// the layer input (QKV and OPROJ of layer l+1, the LM head) adds the partials
// itself.  This removes a reduction hop from every layer.
// then LM tiles (wait EV_IN[L], notify EV_LM -> LMFIN) and LMFIN.  The LM
// tiles fold their best (logit, id) key into a running maximum with an
// atomic max; the order of those updates does not change the result.  Fine-grained events let a consumer
// start on the subset of producer output it reads ("Event Tensor: A Unified
// Abstraction for Compiling Dynamic Megakernel", section "Problem": coarse
// kernel-boundary synchronisation; "Lecture 112: Production Megakernels for
// Real-World Inference", section "Dependency Tracking (Barriers)": partition
// tensor dimensions by dependency to maximise the number of barriers).
#include "plan.hpp"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <random>
#include <set>
#include <unordered_map>

namespace mk {

static const char* kOpNames[OP_COUNT] = {"end", "qkv", "attn", "merge", "oproj", "gateup", "down", "norm", "lm",
                                         "norm2", "lmfin", "route", "mindptr", "egu", "edown", "combine", "mfin",
                                         "normf"};
static const int kLayerOps[] = {OP_QKV, OP_ATTN, OP_OPROJ, OP_GATEUP, OP_DOWN};
static const int kLmOps[] = {OP_LM, OP_LMFIN};
static constexpr int kFamPerLayer = 5;

// ---------------------------------------------------------------- expressions
namespace {
struct Emit {
  std::vector<int32_t>& c;
  int start;
  explicit Emit(std::vector<int32_t>& code) : c(code), start((int)code.size()) {}
  Emit& push(int v) { c.push_back(X_PUSH); c.push_back(v); return *this; }
  Emit& op(int o) { c.push_back(o); return *this; }
  Emit& coord(int d) { c.push_back(X_COORD); c.push_back(d); return *this; }
  int ret() { c.push_back(X_RET); return start; }
};
int emit_const(std::vector<int32_t>& code, int v) { return Emit(code).push(v).ret(); }
}  // namespace

int Plan::fam_index(int op, int layer) const {
  // (as the device's fam_of: the family of (op, layer 0) plus the layer stride)
  const int f0 = dp.fam_first_layer[op];
  if (f0 < 0) return -1;
  return layer < 0 ? f0 : f0 + layer * dp.fam_stride;
}

int Plan::actual_extent(int f, const Binding& bd) const {
  const int op = fams[f].op;
  if (op == OP_EGU || op == OP_EDOWN) {
    const int li = fams[f].layer < 0 ? 0 : fams[f].layer;
    if (li >= (int)bd.route.size()) return 0;
    return bd.route[li].tiles * (op == OP_EGU ? dp.nt_gu : dp.nt_d);
  }
  return family_extent(f, bd);
}

void draw_routing(const Plan& p, Binding& bd, unsigned seed, double skew) {
  const DevPlan& P = p.dp;
  bd.route.clear();
  if (P.kind == MK_MODEL_DENSE) return;
  const int Lm = P.kind == MK_MODEL_MOE_DECODER ? P.n_layers : 1;
  const int E = P.n_experts, K = P.top_k, T = bd.B;
  std::mt19937 rng(seed * 2654435761u + 17u);
  for (int l = 0; l < Lm; ++l) {
    MoeRoute r;
    std::vector<int> perm(E);
    for (int e = 0; e < E; ++e) perm[e] = e;
    std::shuffle(perm.begin(), perm.end(), rng);
    std::vector<double> wt(E);
    for (int i = 0; i < E; ++i) wt[perm[i]] = skew > 0 ? std::pow((double)(i + 1), -skew) : 1.0;
    r.idx.resize((size_t)T * K);
    for (int t = 0; t < T; ++t) {
      std::vector<double> w = wt;
      for (int j = 0; j < K; ++j) {  // k distinct experts, drawn by weight without replacement
        std::discrete_distribution<int> pick(w.begin(), w.end());
        const int e = pick(rng);
        r.idx[(size_t)t * K + j] = e;
        w[e] = 0.0;
      }
    }
    r.hist.assign(E, 0);
    r.rank.resize(r.idx.size());
    for (size_t q = 0; q < r.idx.size(); ++q) r.rank[q] = r.hist[r.idx[q]]++;
    r.indptr.assign(E + 1, 0);
    for (int e = 0; e < E; ++e) r.indptr[e + 1] = r.indptr[e] + r.hist[e];
    for (int e = 0; e < E; ++e) {
      const int tm = moe_tile_rows(r.hist[e], P.moe_tm, P.moe_big);
      for (int m = 0; m < ceil_div(r.hist[e], tm); ++m) { r.tile_e.push_back(e); r.tile_m.push_back(m); }
    }
    r.tiles = (int)r.tile_e.size();
    bd.route.push_back(std::move(r));
  }
}

int Plan::counter(int ev, int c0, int c1, int c2) const {
  const EventTensorDesc& e = dp.ev[ev];
  int lin = c0;
  if (e.ndim > 1) lin = lin * e.dims[1] + c1;
  if (e.ndim > 2) lin = lin * e.dims[2] + c2;
  return e.base + lin;
}

int Plan::event_count(int ev, int c0, int c1, int c2, const Binding& bd) const {
  ExprEnv env{bd.B, bd.ctx.data(), {c0, c1, c2}, step_attn_split(dp, bd.B, bd.ctx.data())};
  return expr_eval(code.data(), dp.ev[ev].count_expr, env);
}

int Plan::family_extent(int f, const Binding& bd) const {
  ExprEnv env{bd.B, bd.ctx.data(), {0, 0, 0}, step_attn_split(dp, bd.B, bd.ctx.data())};
  return expr_eval(code.data(), fams[f].extent_expr, env);
}

// ---------------------------------------------------------------- task model
void Plan::task(int f, int idx, const Binding& bd, TaskRec& t) const {
  const DevPlan& P = dp;
  t = TaskRec();
  t.fam = f;
  t.idx = idx;
  int op = fams[f].op, l = fams[f].layer;
  int B = bd.B, H = P.hidden, D = P.head_dim, Hq = P.n_q_heads, Hkv = P.n_kv_heads;
  int qpg = Hkv > 0 ? Hq / Hkv : 0, F = P.ffn;  // (no attention in an MoE layer plan)
  long long QD = (long long)Hq * D;
  auto kv_row = [&](int layer, int slot, int g, int pos) -> long long {
    return ((((long long)layer * P.n_slots + slot) * Hkv + g) * P.max_ctx + pos) * D;
  };
  // sequence b uses slot b in the host model (slots are distinct by contract)
  const bool mdec = P.kind == MK_MODEL_MOE_DECODER;
  // MoE: this family's layer block, its routing and a tile's rows
  const int li = l < 0 ? 0 : l;
  const long long maxT = P.max_tokens, Kk = P.top_k;
  const MoeRoute* rt = (P.kind != MK_MODEL_DENSE && li < (int)bd.route.size()) ? &bd.route[li] : nullptr;
  auto tile_rows = [&](int tile, int& r0, int& nr) {
    const int e = rt->tile_e[tile], m = rt->tile_m[tile];
    const int tm = moe_tile_rows(rt->hist[e], P.moe_tm, P.moe_big);
    r0 = rt->indptr[e] + m * tm;
    nr = std::min(tm, rt->hist[e] - m * tm);
  };
  const bool wide = P.wide != 0;
  const int asplit = step_attn_split(P, bd.B, bd.ctx.data());  // key chunks per attention task this step
  auto nsplit = [&](int b) { return ceil_div(ceil_div(bd.ctx[b] + 1, P.chunk), asplit); };
  if (wide && op == OP_QKV) {
    // a 128-row tile of [Wq; Wk; Wv]: two heads of q, k or v rows.  Of a
    // tile's K-segment tasks, the last to finish runs the epilogue (a counter
    // inside the tasks orders them, not an event): segment 0 stands for it
    // here and writes the tile's outputs, the others only read their inputs
    const int nq = Hq * D / kWideRows, nk = Hkv * D / kWideRows, tile = idx / P.gseg_qkv;
    const bool epi = idx % P.gseg_qkv == 0;
    const int kind = tile < nq ? 0 : tile < nq + nk ? 1 : 2;
    const int h0 = 2 * (tile - (kind == 0 ? 0 : kind == 1 ? nq : nq + nk));
    t.wait_ev = counter(EV_N1, l);
    t.notify_ev = counter(EV_QKV, l, 0);
    for (int b = 0; b < B; ++b) {
      t.reads.push_back({BUF_XN, (long long)b * H, (long long)(b + 1) * H});
      for (int hh = h0; hh < h0 + 2 && epi; ++hh) {
        if (kind == 0) {
          const long long base = b * QD + (long long)hh * D;
          t.writes.push_back({BUF_Q, base, base + D});
        } else {
          const long long base = kv_row(l, b, hh, bd.ctx[b]);
          t.writes.push_back({kind == 1 ? BUF_KC : BUF_VC, base, base + D});
        }
      }
    }
    return;
  }
  switch (op) {
    case OP_NORM:
    case OP_NORM2:
    case OP_NORMF: {
      // wide batch: row idx of the residual -> its normalised bf16 row
      const int b0 = idx, b1 = idx + 1;
      const int lx = op == OP_NORMF ? P.n_layers : l;
      if (mdec)  // (the MoE decoder's layers chain through the combine of the layer before)
        t.wait_ev = lx > 0 ? counter(EV_MCOMB, lx - 1) : counter(EV_IN, 0);
      else
        t.wait_ev = op == OP_NORM2 ? counter(EV_O, l) : counter(EV_IN, lx);
      t.notify_ev = op == OP_NORM ? counter(EV_N1, l) : op == OP_NORM2 ? counter(EV_N2, l) : counter(EV_NF, 0);
      for (int b = b0; b < b1; ++b) {
        t.reads.push_back({BUF_X, (long long)b * H, (long long)(b + 1) * H});
        if (op != OP_NORM2 && lx > 0 && !mdec)
          for (int kc = 0; kc < P.n_kc; ++kc) {
            const long long pb = ((long long)kc * P.max_batch + b) * H;
            t.reads.push_back({BUF_DPART, pb, pb + H});
          }
        if (op == OP_NORM && !mdec) t.writes.push_back({BUF_X, (long long)b * H, (long long)(b + 1) * H});
        t.writes.push_back({BUF_XN, (long long)b * H, (long long)(b + 1) * H});
      }
    } break;
    case OP_QKV: {
      QkvTile q = decode_qkv(P, idx);
      t.wait_ev = (mdec && l > 0) ? counter(EV_MCOMB, l - 1) : counter(EV_IN, l);
      t.notify_ev = counter(EV_QKV, l, q.group);
      int half = P.tile_qkv / 2;
      for (int b = 0; b < B; ++b) {
        t.reads.push_back({BUF_X, (long long)b * H, (long long)(b + 1) * H});
        if (l > 0 && !mdec)
          for (int kc = 0; kc < P.n_kc; ++kc) {
            long long pb = ((long long)kc * P.max_batch + b) * H;
            t.reads.push_back({BUF_DPART, pb, pb + H});
          }
        for (int part = 0; part < 2; ++part) {
          int j = q.j0 + part * (D / 2);
          if (q.kind == 0) {
            long long base = b * QD + (long long)q.head * D + j;
            t.writes.push_back({BUF_Q, base, base + half});
          } else {
            long long base = kv_row(l, b, q.group, bd.ctx[b]) + j;
            t.writes.push_back({q.kind == 1 ? BUF_KC : BUF_VC, base, base + half});
          }
        }
      }
    } break;
    case OP_ATTN: {
      // task c of (b, g): key chunks c * asplit .. of the sequence
      std::vector<int> nsp(B), pre(B + 1, 0);
      for (int b = 0; b < B; ++b) { nsp[b] = nsplit(b); pre[b + 1] = pre[b] + nsp[b]; }
      AttnTask a = decode_attn(idx, B, Hkv, nsp.data(), pre.data());
      t.wait_ev = counter(EV_QKV, l, wide ? 0 : a.g);
      t.notify_ev = counter(EV_ATTN, l);
      // A pair's last task to finish merges the pair's partials into the
      // output (a counter inside the task, not an event of the plan): the
      // model writes the output region from the pair's only task and the
      // partial slots from the others.
      const bool single = nsp[a.b] == 1;
      long long qb = a.b * QD + (long long)a.g * qpg * D;
      t.reads.push_back({BUF_Q, qb, qb + (long long)qpg * D});
      int p0 = a.c * asplit * P.chunk, p1 = std::min(p0 + asplit * P.chunk, bd.ctx[a.b] + 1);
      long long kb = kv_row(l, a.b, a.g, p0);
      t.reads.push_back({BUF_KC, kb, kb + (long long)(p1 - p0) * D});
      t.reads.push_back({BUF_VC, kb, kb + (long long)(p1 - p0) * D});
      if (single) {
        long long ob = a.b * QD + (long long)a.g * qpg * D;
        t.writes.push_back({BUF_ATTN, ob, ob + (long long)qpg * D});
      } else {
        long long pb = ((long long)a.b * Hkv + a.g) * P.max_chunks + a.c;
        t.writes.push_back({BUF_APART, pb, pb + 1});
      }
    } break;
    case OP_OPROJ: {
      t.wait_ev = counter(EV_ATTN, l);
      t.notify_ev = counter(EV_O, l);
      const int tile = idx / P.gseg_o;
      const bool epi = idx % P.gseg_o == 0;  // (the epilogue's task of the tile, as for QKV)
      for (int b = 0; b < B; ++b) {
        t.reads.push_back({BUF_ATTN, b * QD, (b + 1) * QD});
        if (!epi) continue;
        long long xb = (long long)b * H + (long long)tile * P.tile_o;
        t.reads.push_back({BUF_X, xb, xb + P.tile_o});
        if (l > 0 && !mdec && !wide)
          for (int kc = 0; kc < P.n_kc; ++kc) {
            long long pb = ((long long)kc * P.max_batch + b) * H + (long long)tile * P.tile_o;
            t.reads.push_back({BUF_DPART, pb, pb + P.tile_o});
          }
        t.writes.push_back({BUF_X, xb, xb + P.tile_o});
      }
    } break;
    case OP_GATEUP: {
      const int tile = idx / P.gseg_gu;
      const bool epi = idx % P.gseg_gu == 0;  // (the epilogue's task of the tile, as for QKV)
      t.wait_ev = wide ? counter(EV_N2, l) : counter(EV_O, l);
      t.notify_ev = counter(EV_GU, l, tile * P.tile_gu / P.kseg);
      for (int b = 0; b < B; ++b) {
        t.reads.push_back({wide ? BUF_XN : BUF_X, (long long)b * H, (long long)(b + 1) * H});
        if (!epi) continue;
        long long hb = (long long)b * F + (long long)tile * P.tile_gu;
        t.writes.push_back({BUF_H, hb, hb + P.tile_gu});
      }
    } break;
    case OP_DOWN: {
      int kc = idx / P.n_dtiles, n = idx % P.n_dtiles;
      t.wait_ev = counter(EV_GU, l, kc);
      t.notify_ev = counter(EV_IN, l + 1);
      for (int b = 0; b < B; ++b) {
        long long hb = (long long)b * F + (long long)kc * P.kseg;
        t.reads.push_back({BUF_H, hb, hb + P.kseg});
        long long pb = ((long long)kc * P.max_batch + b) * H + (long long)n * P.tile_down;
        t.writes.push_back({BUF_DPART, pb, pb + P.tile_down});
      }
    } break;
    case OP_LM: {
      t.wait_ev = wide ? counter(EV_NF, 0) : mdec ? counter(EV_MCOMB, P.n_layers - 1) : counter(EV_IN, P.n_layers);
      t.notify_ev = counter(EV_LM, 0);
      t.follow_fam = fam_index(OP_LMFIN, -1);
      t.follow_idx = 0;
      int r0 = idx * P.tile_lm, r1 = std::min(P.vocab, r0 + P.tile_lm);
      for (int b = 0; b < B; ++b) {
        t.reads.push_back({wide ? BUF_XN : BUF_X, (long long)b * H, (long long)(b + 1) * H});
        for (int kc = 0; kc < (mdec || wide ? 0 : P.n_kc); ++kc) {
          long long pb = ((long long)kc * P.max_batch + b) * H;
          t.reads.push_back({BUF_DPART, pb, pb + H});
        }
        t.writes.push_back({BUF_LOGITS, (long long)b * P.vocab + r0, (long long)b * P.vocab + r1});
      }
    } break;
    case OP_LMFIN: {
      for (int b = 0; b < B; ++b) t.writes.push_back({BUF_NEXT, b, b + 1});
    } break;
    // ---- MoE FFN (T = B tokens; per-layer scratch blocks)
    case OP_ROUTE: {
      t.wait_ev = mdec ? counter(EV_O, l) : -1;
      t.notify_ev = counter(EV_ROUTE, li);
      t.follow_fam = fam_index(OP_MINDPTR, l);
      t.follow_idx = 0;
      for (int tok = 8 * idx; tok < std::min(B, 8 * idx + 8); ++tok) {
        if (mdec) {
          t.reads.push_back({BUF_X, (long long)tok * H, (long long)(tok + 1) * H});
          t.writes.push_back({BUF_MXHAT, (li * maxT + tok) * H, (li * maxT + tok + 1) * H});
        }
        t.writes.push_back({BUF_MPAIR, (li * maxT + tok) * Kk, (li * maxT + tok + 1) * Kk});
        for (int j = 0; j < P.top_k; ++j) {  // the token's row copy in each selected expert's rows
          const size_t q = (size_t)tok * P.top_k + j;
          const long long row = ((long long)li * P.n_experts + rt->idx[q]) * P.moe_cap + rt->rank[q];
          t.writes.push_back({BUF_MXG, row * H, (row + 1) * H});
        }
      }
    } break;
    case OP_MINDPTR: {
      t.notify_ev = counter(EV_MIDX, li);
      t.reads.push_back({BUF_MPAIR, li * maxT * Kk, li * maxT * Kk + (long long)B * Kk});
      t.writes.push_back({BUF_MTAB, li, li + 1});
    } break;
    case OP_EGU: {
      const int tile = idx / P.nt_gu, n = idx % P.nt_gu;
      int r0, nr;
      tile_rows(tile, r0, nr);
      t.notify_ev = counter(EV_MH, li, tile);
      t.reads.push_back({BUF_MTAB, li, li + 1});
      {  // the tile's routed token rows
        const int e = rt->tile_e[tile];
        const long long row = ((long long)li * P.n_experts + e) * P.moe_cap +
                              (long long)rt->tile_m[tile] * moe_tile_rows(rt->hist[e], P.moe_tm, P.moe_big);
        t.reads.push_back({BUF_MXG, row * H, (row + nr) * H});
      }
      const long long c0 = (long long)n * P.moe_tn, c1 = std::min<long long>(P.eff, c0 + P.moe_tn);
      for (int r = r0; r < r0 + nr; ++r) {
        const long long rb = (li * maxT * Kk + r) * P.eff;
        t.writes.push_back({BUF_MH, rb + c0, rb + c1});
      }
    } break;
    case OP_EDOWN: {
      const int tile = idx / P.nt_d, n = idx % P.nt_d;
      int r0, nr;
      tile_rows(tile, r0, nr);
      t.wait_ev = counter(EV_MH, li, tile);
      t.notify_ev = counter(EV_MY, li);
      t.reads.push_back({BUF_MTAB, li, li + 1});
      t.reads.push_back({BUF_MH, (li * maxT * Kk + r0) * P.eff, (li * maxT * Kk + r0 + nr) * P.eff});
      for (int r = r0; r < r0 + nr; ++r) {
        const long long rb = (li * maxT * Kk + r) * H + (long long)n * P.moe_td;
        t.writes.push_back({BUF_MY, rb, rb + P.moe_td});
      }
    } break;
    case OP_COMBINE: {
      t.wait_ev = counter(EV_MY, li);
      t.notify_ev = counter(EV_MCOMB, li);
      if (!mdec) { t.follow_fam = fam_index(OP_MFIN, -1); t.follow_idx = 0; }
      t.reads.push_back({BUF_MTAB, li, li + 1});
      for (int tok = 8 * idx; tok < std::min(B, 8 * idx + 8); ++tok) {
        t.reads.push_back({BUF_MPAIR, (li * maxT + tok) * Kk, (li * maxT + tok + 1) * Kk});
        for (int j = 0; j < P.top_k; ++j) {  // the segment of the pair's expert (its row lies in it)
          const int e = rt->idx[(size_t)tok * P.top_k + j];
          t.reads.push_back({BUF_MY, (li * maxT * Kk + rt->indptr[e]) * H, (li * maxT * Kk + rt->indptr[e + 1]) * H});
        }
        if (mdec) {
          t.reads.push_back({BUF_X, (long long)tok * H, (long long)(tok + 1) * H});
          t.writes.push_back({BUF_X, (long long)tok * H, (long long)(tok + 1) * H});
        } else {
          t.writes.push_back({BUF_MOUT, (long long)tok * H, (long long)(tok + 1) * H});
        }
      }
    } break;
    default: break;  // MFIN: end of the layer call
  }
}

void Plan::successors(int ci, const Binding& bd, std::vector<int>& out) const {
  // find the tensor and coordinates of counter ci
  int ev = -1;
  for (int e = 0; e < EV_COUNT; ++e) {
    int n = dp.ev[e].dims[0] * (dp.ev[e].ndim > 1 ? dp.ev[e].dims[1] : 1) *
            (dp.ev[e].ndim > 2 ? dp.ev[e].dims[2] : 1);
    if (ci >= dp.ev[e].base && ci < dp.ev[e].base + n) { ev = e; break; }
  }
  if (ev < 0) return;
  int lin = ci - dp.ev[ev].base;
  int c[3] = {0, 0, 0};
  for (int d = dp.ev[ev].ndim - 1; d >= 0; --d) { c[d] = lin % dp.ev[ev].dims[d]; lin /= dp.ev[ev].dims[d]; }
  auto add = [&](int f, int lo, int n) { if (n > 0) { out.push_back(f); out.push_back(lo); out.push_back(n); } };
  const bool mdec = dp.kind == MK_MODEL_MOE_DECODER;
  const int ml = dp.kind == MK_MODEL_MOE_LAYER ? -1 : c[0];  // the MoE event's layer
  const bool wide = dp.wide != 0;
  const int n8 = ceil_div(bd.B, 8);
  switch (ev) {
    case EV_IN:
      if (mdec) break;  // (the MoE decoder's layers chain through EV_MCOMB)
      if (wide) {
        if (c[0] < dp.n_layers) add(fam_index(OP_NORM, c[0]), 0, bd.B);
        else add(fam_index(OP_NORMF, -1), 0, bd.B);
      } else if (c[0] < dp.n_layers) {
        add(fam_index(OP_QKV, c[0]), 0, dp.n_qkv_tiles);
      } else {
        add(fam_index(OP_LM, -1), 0, dp.n_lm_tiles);
      }
      break;
    case EV_N1: add(fam_index(OP_QKV, c[0]), 0, dp.n_qkv_tiles); break;
    case EV_N2: add(fam_index(OP_GATEUP, c[0]), 0, dp.n_gutiles); break;
    case EV_NF: add(fam_index(OP_LM, -1), 0, dp.n_lm_tiles); break;
    case EV_MIDX: add(fam_index(OP_EGU, ml), 0, bd.route[c[0]].tiles * dp.nt_gu); break;
    case EV_MH: add(fam_index(OP_EDOWN, ml), c[1] * dp.nt_d, dp.nt_d); break;
    case EV_MY: add(fam_index(OP_COMBINE, ml), 0, ceil_div(bd.B, 8)); break;
    case EV_MCOMB:
      if (!mdec) break;  // (the MoE layer's end is a follow-up)
      if (wide) {
        if (c[0] + 1 < dp.n_layers) add(fam_index(OP_NORM, c[0] + 1), 0, bd.B);
        else add(fam_index(OP_NORMF, -1), 0, bd.B);
      } else if (c[0] + 1 < dp.n_layers) {
        add(fam_index(OP_QKV, c[0] + 1), 0, dp.n_qkv_tiles);
      } else {
        add(fam_index(OP_LM, -1), 0, dp.n_lm_tiles);
      }
      break;
    case EV_QKV: {
      int pre = 0;
      const int asplit = step_attn_split(dp, bd.B, bd.ctx.data());
      for (int b = 0; b < bd.B; ++b) {
        const int ns = ceil_div(ceil_div(bd.ctx[b] + 1, dp.chunk), asplit);
        if (wide) add(fam_index(OP_ATTN, c[0]), dp.n_kv_heads * pre, dp.n_kv_heads * ns);  // every kv head
        else add(fam_index(OP_ATTN, c[0]), dp.n_kv_heads * pre + c[1] * ns, ns);
        pre += ns;
      }
    } break;
    case EV_ATTN: add(fam_index(OP_OPROJ, c[0]), 0, dp.n_otiles); break;
    case EV_O:
      if (mdec) add(fam_index(OP_ROUTE, c[0]), 0, n8);
      else if (wide) add(fam_index(OP_NORM2, c[0]), 0, bd.B);
      else add(fam_index(OP_GATEUP, c[0]), 0, dp.n_gutiles);
      break;
    case EV_GU: add(fam_index(OP_DOWN, c[0]), c[1] * dp.n_dtiles, dp.n_dtiles); break;
    default: break;  // EV_LM and EV_ROUTE trigger follow-ups
  }
}

// ---------------------------------------------------------------- build

// Shared-memory split of a CTA (see kSmemFixed): the staging buffer sized for
// `rows` batch rows and at least min_act bytes, the partial tiles (for the
// dense GEMV tasks; none for rows = 0), the rest to 16 KB ring slots.
static void smem_layout(DevPlan& P, int rows, int smem_bytes, int min_act) {
  P.gbatch = kMaxBatchRows;
  // (B <= 4 stages 2B rows: each row's bf16 value and its bf16 remainder)
  P.act_bytes = std::max(8192, (std::min(2 * rows, kMaxBatchRows) * kActPitch * 2 + 127) / 128 * 128);
  P.act_bytes = std::max(P.act_bytes, (min_act + 127) / 128 * 128);
  P.gred_bytes = rows > 0 ? 8 * P.gbatch * 64 * 4 : 0;
  P.smem_bytes = smem_bytes;
  P.ring_slots = std::min(16, (smem_bytes - kSmemFixed - P.act_bytes - P.gred_bytes - seq_table_bytes(P)) /
                                  P.slot_bytes);
}


// MoE FFN layer ("Event Tensor: A Unified Abstraction for Compiling Dynamic
// Megakernel", section "Core method", data-dependent dynamism).  The task
// graph: ROUTE (8 tokens each) -> follow-up MINDPTR (exp_indptr, tile table,
// row map; arms the count of EV_MY) -> EGU tiles, as many as exp_indptr
// implies -> per tile, EDOWN tasks -> COMBINE -> follow-up MFIN.  Task counts
// after ROUTE depend on the routing, so the layer runs on the dynamic queue.
static mk_status build_moe_plan(const mk_model_desc* m, const mk_plan_opts* o, int n_sm, int smem_bytes,
                                Plan& p, std::string& err) {
  const int H = m->hidden, E = m->n_experts, K = m->top_k, FF = m->expert_ffn, TM = m->max_tokens;
  if (H % 256 || H > 2048 || H < 256) { err = "hidden must be a multiple of 256 in [256, 2048]"; return MK_ERR_UNSUPPORTED; }
  if (E < 1 || E > 64) { err = "n_experts must be in [1, 64]"; return MK_ERR_UNSUPPORTED; }
  if (K < 1 || K > 8 || K > E) { err = "top_k must be in [1, min(8, n_experts)]"; return MK_ERR_UNSUPPORTED; }
  if (FF < 64 || FF % 64 || FF > 2048) { err = "expert_ffn must be a multiple of 64 in [64, 2048]"; return MK_ERR_UNSUPPORTED; }
  if (TM < 1 || TM > 4096) { err = "max_tokens must be in [1, 4096]"; return MK_ERR_UNSUPPORTED; }
  if (o->sched != MK_SCHED_DYNAMIC)
    { err = "an MoE layer's task counts depend on the routing: use MK_SCHED_DYNAMIC"; return MK_ERR_UNSUPPORTED; }
  if (n_sm < 1 || n_sm > 1024) { err = "n_sm out of range"; return MK_ERR_INVALID_ARG; }
  p.m = *m;
  p.m.layers = nullptr;
  p.o = *o;
  p.layer_w.clear();
  DevPlan& P = p.dp;
  P = DevPlan();
  P.kind = MK_MODEL_MOE_LAYER;
  P.sched = o->sched;
  P.n_sm = n_sm;
  P.hidden = H;
  P.debug_flags = o->debug_flags;
  P.spin_timeout_ns = o->spin_timeout_ns > 0 ? o->spin_timeout_ns : 2000000000LL;
  P.fault_ctr = -1;
  if (o->fault != 0) { err = "fault injection is available for decoder plans only"; return MK_ERR_INVALID_ARG; }
  if (o->debug_flags & MK_DEBUG_EMPTY_TASKS)
    { err = "empty tasks: an MoE layer's task graph depends on its routing"; return MK_ERR_INVALID_ARG; }
  P.n_experts = E; P.top_k = K; P.eff = FF; P.max_tokens = TM;
  P.moe_tm = kMoeTileRows;  // routed rows per GroupGEMM tile
  P.moe_tn = kMoeTaskRows;  // gate rows (and as many up rows) per EGU task
  P.moe_td = kMoeTaskRows;  // down rows per EDOWN task
  P.nt_gu = ceil_div(FF, P.moe_tn);
  P.nt_d = H / P.moe_td;
  P.moe_cap = TM;
  if (o->moe_tiles < 0 || o->moe_tiles > 2) { err = "moe_tiles must be 0, 1 or 2"; return MK_ERR_INVALID_ARG; }
  P.moe_big = o->moe_tiles != 2;
  // sum over experts of ceil(hist_e / tm) <= T*k/tm + (experts with a row)
  P.max_tiles = ceil_div(TM * K, P.moe_tm) + std::min(E, TM * K);
  P.slot_bytes = 16384;
  smem_layout(P, 0, smem_bytes, route_stage_bytes(H));
  if (P.ring_slots < 5) { err = "not enough shared memory for a 5-slot ring"; return MK_ERR_UNSUPPORTED; }

  p.code.clear();
  p.fams.clear();
  p.fam_names.clear();
  int debug_base = 0;
  auto add_family = [&](int op, int extent_expr, int max_extent, int followup) {
    FamilyDesc f{};
    f.op = op; f.layer = -1; f.extent_expr = extent_expr; f.max_extent = max_extent;
    f.debug_base = debug_base; f.followup = followup;
    debug_base += max_extent;
    P.fam_first_layer[op] = (int)p.fams.size();
    p.fams.push_back(f);
    p.fam_names.push_back(kOpNames[op]);
  };
  for (int op = 0; op < OP_COUNT; ++op) P.fam_first_layer[op] = -1;
  const int e_tok8 = Emit(p.code).op(X_B).push(8).op(X_CEILDIV).ret();  // ceil(T / 8); B stands for T
  add_family(OP_ROUTE, e_tok8, ceil_div(TM, 8), 0);
  add_family(OP_MINDPTR, emit_const(p.code, 1), 1, 1);
  // the extents below are set by the routing; the expressions give the maxima
  add_family(OP_EGU, emit_const(p.code, P.max_tiles * P.nt_gu), P.max_tiles * P.nt_gu, 0);
  add_family(OP_EDOWN, emit_const(p.code, P.max_tiles * P.nt_d), P.max_tiles * P.nt_d, 0);
  add_family(OP_COMBINE, e_tok8, ceil_div(TM, 8), 0);
  add_family(OP_MFIN, emit_const(p.code, 1), 1, 1);
  P.n_families = (int)p.fams.size();
  P.debug_slots = debug_base;
  P.fam_stride = 0;

  int base = 0;
  const int e_zero = emit_const(p.code, 0);
  for (int id = 0; id < EV_ROUTE; ++id) {  // the dense decoder's events are empty
    EventTensorDesc& e = P.ev[id];
    e.base = 0; e.ndim = 1; e.dims[0] = 0; e.dims[1] = e.dims[2] = 1; e.count_expr = e_zero;
  }
  auto add_event = [&](int id, int d0, int count_expr) {
    EventTensorDesc& e = P.ev[id];
    e.base = base; e.ndim = 1; e.dims[0] = d0; e.dims[1] = e.dims[2] = 1; e.count_expr = count_expr;
    base += d0;
  };
  add_event(EV_ROUTE, 1, e_tok8);
  add_event(EV_MIDX, 1, emit_const(p.code, 1));
  {
    EventTensorDesc& e = P.ev[EV_MH];
    e.base = base; e.ndim = 2; e.dims[0] = 1; e.dims[1] = P.max_tiles; e.dims[2] = 1;
    e.count_expr = emit_const(p.code, 0);  // armed at run time by MINDPTR for the tiles the routing made
    base += P.max_tiles;
  }
  add_event(EV_MY, 1, emit_const(p.code, 1 << 30));  // replaced at run time by MINDPTR
  add_event(EV_MCOMB, 1, e_tok8);
  P.n_counters = base;

  // no static instructions: one END per CTA
  P.n_instr_per_sm = 1;
  p.instr.assign((size_t)n_sm, Instr{-1, 0, 1, 0});
  // pushes per launch: ROUTE, EGU, one EDOWN range per tile, COMBINE, END
  P.queue_ranges = P.max_tiles + 8;
  p.layers.clear();
  p.rope.clear();
  P.w_router = m->moe.w_router;
  P.router_bias = m->moe.router_bias;
  P.w_egate = m->moe.w_gate;
  P.w_eup = m->moe.w_up;
  P.w_edown = m->moe.w_down;
  std::vector<unsigned char> image;
  lower_plan(p, image);
  return MK_OK;
}

mk_status build_plan(const mk_model_desc* m, const mk_plan_opts* o, int n_sm, int smem_bytes,
                     Plan& p, std::string& err) {
  if (!m || !o) { err = "null model or options"; return MK_ERR_INVALID_ARG; }
  if (m->kind == MK_MODEL_MOE_LAYER) return build_moe_plan(m, o, n_sm, smem_bytes, p, err);
  if (m->kind != MK_MODEL_DENSE && m->kind != MK_MODEL_MOE_DECODER) { err = "unknown model kind"; return MK_ERR_UNSUPPORTED; }
  // MoE decoder: the dense decoder's attention half, then per layer the MoE
  // FFN families of build_moe_plan on the B tokens (dynamic schedule only)
  const bool mdec = m->kind == MK_MODEL_MOE_DECODER;
  const int H = m->hidden, D = m->head_dim, Hq = m->n_q_heads, Hkv = m->n_kv_heads, F = mdec ? 0 : m->ffn;
  if (mdec && (o->debug_flags & MK_DEBUG_EMPTY_TASKS))
    { err = "empty tasks: an MoE layer's task graph depends on its routing"; return MK_ERR_INVALID_ARG; }
  if (mdec) {
    const int E = m->n_experts, K = m->top_k, FF = m->expert_ffn;
    if (E < 1 || E > 64) { err = "n_experts must be in [1, 64]"; return MK_ERR_UNSUPPORTED; }
    if (K < 1 || K > 8 || K > E) { err = "top_k must be in [1, min(8, n_experts)]"; return MK_ERR_UNSUPPORTED; }
    if (FF < 64 || FF % 64 || FF > 2048) { err = "expert_ffn must be a multiple of 64 in [64, 2048]"; return MK_ERR_UNSUPPORTED; }
    if (o->sched != MK_SCHED_DYNAMIC)
      { err = "an MoE layer's task counts depend on the routing: use MK_SCHED_DYNAMIC"; return MK_ERR_UNSUPPORTED; }
  }
  if (m->n_layers < 1 || m->vocab < 1 || Hkv < 1 || Hq < 1) { err = "non-positive dimension"; return MK_ERR_INVALID_ARG; }
  if (D != 64) { err = "head_dim must be 64"; return MK_ERR_UNSUPPORTED; }
  if (Hq % Hkv) { err = "n_q_heads must be a multiple of n_kv_heads"; return MK_ERR_INVALID_ARG; }
  if (Hq * D != H) { err = "n_q_heads * head_dim must equal hidden"; return MK_ERR_UNSUPPORTED; }
  if (H % 256 || H > 2048 || H < 256) { err = "hidden must be a multiple of 256 in [256, 2048]"; return MK_ERR_UNSUPPORTED; }
  if (!mdec && (F % 256 || F < 256)) { err = "ffn must be a positive multiple of 256"; return MK_ERR_UNSUPPORTED; }
  // above kMaxBatchRows the dense decoder runs the wide-batch path
  // (an MoE decoder above 8 rows runs the wide-batch attention half and LM
  // head; its FFN is the MoE layer either way)
  const bool wide = m->max_batch > kMaxBatchRows;
  const bool dwide = wide && !mdec;
  if (m->max_batch < 1 || m->max_batch > (mdec ? kMaxBatch : kMaxWideBatch))
    { err = mdec ? "max_batch must be in [1, 128] for an MoE decoder" : "max_batch must be in [1, 64]"; return MK_ERR_UNSUPPORTED; }
  if (m->max_ctx < 2 || m->n_slots < m->max_batch) { err = "max_ctx >= 2 and n_slots >= max_batch required"; return MK_ERR_INVALID_ARG; }
  if (o->sched != MK_SCHED_STATIC && o->sched != MK_SCHED_DYNAMIC) { err = "unknown schedule"; return MK_ERR_INVALID_ARG; }
  if (n_sm < 1 || n_sm > 1024) { err = "n_sm out of range"; return MK_ERR_INVALID_ARG; }

  p.m = *m;
  p.o = *o;
  p.layer_w.assign(m->layers ? m->layers : nullptr, m->layers ? m->layers + m->n_layers : nullptr);
  if (!m->layers) p.layer_w.assign(m->n_layers, mk_layer_weights{});
  p.m.layers = nullptr;
  DevPlan& P = p.dp;
  P = DevPlan();
  P.sched = o->sched;
  P.n_sm = n_sm;
  P.n_layers = m->n_layers; P.hidden = H; P.n_q_heads = Hq; P.n_kv_heads = Hkv; P.head_dim = D;
  P.ffn = F; P.vocab = m->vocab; P.max_batch = m->max_batch; P.max_ctx = m->max_ctx;
  P.n_slots = m->n_slots; P.eps = m->eps;
  P.debug_flags = o->debug_flags;
  P.spin_timeout_ns = o->spin_timeout_ns > 0 ? o->spin_timeout_ns : 2000000000LL;
  P.fault_ctr = -1;

  // K segment of the down projection (split-K), at most 2048 columns (wide
  // batch: 1024 by default, twice the down tasks for the phase)
  int kseg = mdec ? 2048 : (o->kseg ? o->kseg : std::min(F, wide ? 1024 : 2048));  // (no dense FFN in an MoE decoder)
  while (kseg > 256 && F % kseg) kseg -= 256;
  P.kseg = kseg;
  // GEMV tiles on tensor cores: 16, 32 or 64 rows per task in whole 16-row
  // blocks (QKV: 16 rotate-half pairs; gate/up: 16 + 16 or 32 + 32 rows), in
  // halves of at most 32 rows spread over 8 ring slots by column: slot j of a
  // half holds columns [j K/8, (j+1) K/8) of the half's rows.  Defaults: the
  // largest tiles (the per-task cost dominates the B=1 step)
  P.tile_qkv = o->tile_qkv ? o->tile_qkv : 32;
  P.tile_o = o->tile_o ? o->tile_o : 32;
  P.tile_gu = o->tile_gu ? o->tile_gu : 32;
  P.tile_down = o->tile_down ? o->tile_down : 64;
  P.tile_lm = o->tile_lm ? o->tile_lm : 64;
  P.chunk = o->attn_chunk ? o->attn_chunk : 64;
  P.slot_bytes = 16384;
  P.wide = wide ? 1 : 0;
  // key chunks per attention task: an option value is used as given; small
  // batches (below) follow each step, at most 32 chunks (2048 keys); wide
  // batches 24 (three per warp: a warp's next chunk loads while one is
  // computed; of 8, 16, 24 and 32, 16 was fastest at B = 16, 32 at B = 32 and
  // 24 at B = 64, 24 the best over the three)
  P.attn_split = o->attn_split ? o->attn_split : (wide ? 24 : 32);
  // with no split given, the split follows each step's B and contexts at
  // steps of up to 8 rows, in narrow and wide plans alike (step_attn_split:
  // 3 to 16 chunks on the 1B shape at B = 1..8)
  P.attn_auto = !o->attn_split ? 1 : 0;
  if (P.attn_split < 1 || P.attn_split > 64) { err = "attn_split must be in [1, 64]"; return MK_ERR_INVALID_ARG; }
  if (wide) {
    // tcgen05 GEMM tasks: kWideRows weight rows each (the MMA's M), every
    // weight matrix read in 64-column chunks, the batch as the MMA's N
    if (o->tile_qkv || o->tile_o || o->tile_gu || o->tile_down || o->tile_lm)
      { err = "the wide-batch path takes no GEMV tile options"; return MK_ERR_INVALID_ARG; }
    P.tile_qkv = P.tile_o = P.tile_gu = P.tile_down = P.tile_lm = kWideRows;
    if (H % kWideRows || F % kWideRows) { err = "wide batch: hidden and ffn must be multiples of 128"; return MK_ERR_UNSUPPORTED; }
    if (P.vocab < 1) { err = "non-positive vocabulary"; return MK_ERR_INVALID_ARG; }
    if (Hq / Hkv < 2 || (Hq / Hkv) % 2) { err = "wide batch: an even number of query heads per kv head"; return MK_ERR_UNSUPPORTED; }
  }
  P.act_rows = ceil_div(P.max_batch, 16) * 16;
  // wide batch: activations as value + remainder (near-fp32 products) while
  // both MMA operand rows fit (2 x 64 columns per accumulator)
  if (o->act_split < 0 || o->act_split > 2) { err = "act_split must be 0, 1 or 2"; return MK_ERR_INVALID_ARG; }
  P.act_split = wide && o->act_split != 2 && P.act_rows <= kMaxWideBatch;
  if (wide && o->act_split == 1 && !P.act_split)
    { err = "act_split: value + remainder rows need max_batch <= 64"; return MK_ERR_UNSUPPORTED; }
  if (!(P.kseg % 256 == 0 && F % P.kseg == 0 && P.kseg >= 1024 && P.kseg <= 2048))
    { err = "kseg must be a multiple of 256 in [1024, 2048] dividing ffn"; return MK_ERR_INVALID_ARG; }
  if (Hq / Hkv > 4) { err = "at most 4 query heads per kv head"; return MK_ERR_UNSUPPORTED; }
  if (!wide && P.tile_qkv != 32) { err = "tile_qkv must be 32 (16 rotate-half pairs)"; return MK_ERR_UNSUPPORTED; }
  if (!wide && !((P.tile_o == 16 || P.tile_o == 32) && H % P.tile_o == 0))
    { err = "tile_o must be 16 or 32 and divide hidden"; return MK_ERR_UNSUPPORTED; }
  if (!wide && !((P.tile_gu == 16 || P.tile_gu == 32) && P.kseg % P.tile_gu == 0))
    { err = "tile_gu must be 16 or 32 (gate + up rows each)"; return MK_ERR_UNSUPPORTED; }
  if (!wide && !((P.tile_down == 16 || P.tile_down == 32 || P.tile_down == 64) && H % P.tile_down == 0))
    { err = "tile_down must be 16, 32 or 64 and divide hidden"; return MK_ERR_UNSUPPORTED; }
  if (!wide && P.tile_lm != 32 && P.tile_lm != 64) { err = "tile_lm must be 32 or 64"; return MK_ERR_UNSUPPORTED; }
  if (P.chunk != 64) { err = "attn_chunk must be 64"; return MK_ERR_UNSUPPORTED; }
  // wide batch: K segments per GEMM tile (split K, see DevPlan::gseg_qkv):
  // 4 segments of at least 2 chunks of 64 columns (2 for gate/up, which
  // streams two weight parts), so that a phase has several tasks per SM
  P.gseg_qkv = P.gseg_o = P.gseg_gu = 1;
  if (wide) {
    P.gseg_qkv = std::min(4, H / 128);
    P.gseg_o = std::min(4, Hq * D / 128);
    P.gseg_gu = std::min(2, H / 128);
    if ((Hq + 2 * Hkv) * D / kWideRows > kGctrPerOp || H / kWideRows > kGctrPerOp ||
        (!mdec && F / kWideRows > kGctrPerOp))
      { err = "wide batch: at most 64 tiles of 128 rows per projection"; return MK_ERR_UNSUPPORTED; }
  }
  // task counts (wide batch: tiles x K segments; task i is segment i % gseg of tile i / gseg)
  P.n_qkv_tiles = (Hq + 2 * Hkv) * D / P.tile_qkv * P.gseg_qkv;
  P.n_otiles = H / P.tile_o * P.gseg_o;
  P.n_gutiles = F / P.tile_gu * P.gseg_gu;
  P.n_dtiles = H / P.tile_down;
  P.n_kc = F / P.kseg;
  if (wide && P.n_kc > 8) { err = "wide batch: at most 8 down-projection K segments (ffn / kseg)"; return MK_ERR_UNSUPPORTED; }
  P.n_lm_tiles = ceil_div(P.vocab, P.tile_lm);
  P.max_chunks = ceil_div(P.max_ctx, P.chunk);

  // shared memory: ring of 16 KB slots plus a fixed control area (wide
  // batch: the staging buffer holds the activation chunks of the GEMM tasks'
  // MMA issuer, kBStages x act_rows x 128 bytes, and afterwards the QKV
  // tiles' rotate-half exchange, 64 rows x act_rows fp32; no GEMV partial tiles)
  if (wide) {
    P.gbatch = 0;
    P.act_bytes = std::max(std::max(8192, 64 * P.act_rows * 4), kBStages * act_buf_rows(P.act_split, P.act_rows) * 128);
    if (mdec) P.act_bytes = std::max(P.act_bytes, (route_stage_bytes(H) + 127) / 128 * 128);  // (ROUTE tasks)
    P.gred_bytes = 0;
    P.smem_bytes = smem_bytes;
    P.ring_slots = std::min(16, (smem_bytes - kSmemFixed - P.act_bytes - seq_table_bytes(P)) / P.slot_bytes);
  } else {
    smem_layout(P, P.max_batch, smem_bytes, mdec ? route_stage_bytes(H) : 0);
  }
  if (P.ring_slots < 3) { err = "not enough shared memory for a 3-slot ring"; return MK_ERR_UNSUPPORTED; }

  // ---- expressions and families
  p.code.clear();
  p.fams.clear();
  p.fam_names.clear();
  int debug_base = 0;
  auto add_family = [&](int op, int layer, int extent_expr, int max_extent, int followup) {
    FamilyDesc f{};
    f.op = op; f.layer = layer; f.extent_expr = extent_expr; f.max_extent = max_extent;
    f.debug_base = debug_base; f.followup = followup;
    debug_base += max_extent;
    p.fams.push_back(f);
    p.fam_names.push_back(std::string(kOpNames[op]) + (layer >= 0 ? "." + std::to_string(layer) : ""));
  };
  // ATTN extent: Hkv * sum_b ceil(ceil((ctx_b + 1) / chunk) / asplit), asplit the step's split
  int e_attn;
  {
    Emit e(p.code);
    e.push(Hkv);
    p.code.push_back(X_SUM_B);
    size_t len_at = p.code.size();
    p.code.push_back(0);
    size_t body = p.code.size();
    p.code.push_back(X_VAR); p.code.push_back(X_CTX_AT);
    p.code.push_back(X_PUSH); p.code.push_back(1); p.code.push_back(X_ADD);
    p.code.push_back(X_PUSH); p.code.push_back(P.chunk); p.code.push_back(X_CEILDIV);
    p.code.push_back(X_ASPLIT); p.code.push_back(X_CEILDIV);
    p.code.push_back(X_RET);
    p.code[len_at] = (int)(p.code.size() - body);
    p.code.push_back(X_MUL);
    p.code.push_back(X_RET);
    e_attn = e.start;
  }
  // MoE decoder: the MoE FFN's geometry (as build_moe_plan) on at most max_batch tokens
  if (mdec) {
    P.kind = MK_MODEL_MOE_DECODER;
    P.n_experts = m->n_experts; P.top_k = m->top_k; P.eff = m->expert_ffn; P.max_tokens = P.max_batch;
    P.moe_tm = kMoeTileRows; P.moe_tn = kMoeTaskRows; P.moe_td = kMoeTaskRows;
    P.nt_gu = ceil_div(P.eff, P.moe_tn);
    P.nt_d = H / P.moe_td;
    P.moe_cap = P.max_tokens;
    if (o->moe_tiles < 0 || o->moe_tiles > 2) { err = "moe_tiles must be 0, 1 or 2"; return MK_ERR_INVALID_ARG; }
    P.moe_big = o->moe_tiles != 2;
    P.max_tiles = ceil_div(P.max_tokens * P.top_k, P.moe_tm) + std::min(P.n_experts, P.max_tokens * P.top_k);
    }
  const int e_tok8 = Emit(p.code).op(X_B).push(8).op(X_CEILDIV).ret();  // ceil(B / 8)
  const int e_tok1 = Emit(p.code).op(X_B).ret();                         // B (wide batch: one norm task per row)
  static const int kMoeDecOps[] = {OP_QKV, OP_ATTN, OP_OPROJ, OP_ROUTE, OP_MINDPTR, OP_EGU, OP_EDOWN, OP_COMBINE};
  static const int kWideOps[] = {OP_NORM, OP_QKV, OP_ATTN, OP_OPROJ, OP_NORM2, OP_GATEUP, OP_DOWN};
  static const int kMoeDecWideOps[] = {OP_NORM, OP_QKV, OP_ATTN, OP_OPROJ, OP_ROUTE, OP_MINDPTR, OP_EGU,
                                       OP_EDOWN, OP_COMBINE};
  const int fam_per_layer = mdec ? (wide ? 9 : 8) : wide ? 7 : kFamPerLayer;
  const int* layer_ops = mdec ? (wide ? kMoeDecWideOps : kMoeDecOps) : wide ? kWideOps : kLayerOps;
  const int min_split = P.attn_auto ? std::min(kAttnSplitMin, P.attn_split) : P.attn_split;
  const int max_tasks_attn = Hkv * P.max_batch * ceil_div(P.max_chunks, min_split);
  for (int l = 0; l < P.n_layers; ++l) {
    if (wide) add_family(OP_NORM, l, e_tok1, P.max_batch, 0);
    add_family(OP_QKV, l, emit_const(p.code, P.n_qkv_tiles), P.n_qkv_tiles, 0);
    add_family(OP_ATTN, l, e_attn, max_tasks_attn, 0);
    add_family(OP_OPROJ, l, emit_const(p.code, P.n_otiles), P.n_otiles, 0);
    if (dwide) add_family(OP_NORM2, l, e_tok1, P.max_batch, 0);
    if (mdec) {
      add_family(OP_ROUTE, l, e_tok8, ceil_div(P.max_tokens, 8), 0);
      add_family(OP_MINDPTR, l, emit_const(p.code, 1), 1, 1);
      add_family(OP_EGU, l, emit_const(p.code, P.max_tiles * P.nt_gu), P.max_tiles * P.nt_gu, 0);
      add_family(OP_EDOWN, l, emit_const(p.code, P.max_tiles * P.nt_d), P.max_tiles * P.nt_d, 0);
      add_family(OP_COMBINE, l, e_tok8, ceil_div(P.max_tokens, 8), 0);
    } else {
      add_family(OP_GATEUP, l, emit_const(p.code, P.n_gutiles), P.n_gutiles, 0);
      add_family(OP_DOWN, l, emit_const(p.code, P.n_dtiles * P.n_kc), P.n_dtiles * P.n_kc, 0);
    }
  }
  if (wide) add_family(OP_NORMF, -1, e_tok1, P.max_batch, 0);
  add_family(OP_LM, -1, emit_const(p.code, P.n_lm_tiles), P.n_lm_tiles, 0);
  add_family(OP_LMFIN, -1, emit_const(p.code, 1), 1, 1);
  P.n_families = (int)p.fams.size();
  if (P.n_families > kMaxFamilies || P.n_layers > 127) { err = "too many task families or layers"; return MK_ERR_UNSUPPORTED; }
  P.debug_slots = debug_base;
  P.fam_stride = fam_per_layer;
  for (int op = 0; op < OP_COUNT; ++op) P.fam_first_layer[op] = -1;
  for (int k = 0; k < fam_per_layer; ++k) P.fam_first_layer[layer_ops[k]] = k;
  {
    int g0 = P.n_layers * fam_per_layer;
    if (wide) P.fam_first_layer[OP_NORMF] = g0++;
    for (int k = 0; k < 2; ++k) P.fam_first_layer[kLmOps[k]] = g0 + k;
  }

  // ---- event tensors (shapes at the symbols' maxima, wait counts symbolic)
  int base = 0;
  auto add_event = [&](int id, int ndim, int d0, int d1, int d2, int count_expr) {
    EventTensorDesc& e = P.ev[id];
    e.base = base; e.ndim = ndim; e.dims[0] = d0; e.dims[1] = d1; e.dims[2] = d2;
    e.count_expr = count_expr;
    base += d0 * (ndim > 1 ? d1 : 1) * (ndim > 2 ? d2 : 1);
  };
  const int L = P.n_layers;
  const int qkv_per_group = (Hq / Hkv + 2) * (D / P.tile_qkv);
  add_event(EV_IN, 1, L + 1, 1, 1,
            Emit(p.code).push(0).coord(0).op(X_LT).push(P.n_dtiles * P.n_kc).op(X_MUL).ret());
  if (wide) add_event(EV_QKV, 2, L, 1, 1, emit_const(p.code, P.n_qkv_tiles));  // (a tile spans two kv heads)
  else add_event(EV_QKV, 2, L, Hkv, 1, emit_const(p.code, qkv_per_group));
  // (EV_CHUNK is unused: the attention tasks of a (sequence, kv head) merge
  // their partials in the last of them to finish, see task_attn)
  add_event(EV_CHUNK, 1, 1, 1, 1, emit_const(p.code, 0));
  // every attention task of the layer: Hkv * sum_b n_b
  add_event(EV_ATTN, 1, L, 1, 1, e_attn);
  add_event(EV_O, 1, L, 1, 1, emit_const(p.code, P.n_otiles));
  add_event(EV_GU, 2, L, P.n_kc, 1, emit_const(p.code, P.kseg / P.tile_gu * P.gseg_gu));
  add_event(EV_LM, 1, 1, 1, 1, emit_const(p.code, P.n_lm_tiles));
  if (mdec) {  // one element per layer (EV_MH: per layer and GroupGEMM tile)
    add_event(EV_ROUTE, 1, L, 1, 1, e_tok8);
    add_event(EV_MIDX, 1, L, 1, 1, emit_const(p.code, 1));
    add_event(EV_MH, 2, L, P.max_tiles, 1, emit_const(p.code, 0));  // armed at run time by MINDPTR
    add_event(EV_MY, 1, L, 1, 1, emit_const(p.code, 1 << 30));  // replaced at run time by MINDPTR
    add_event(EV_MCOMB, 1, L, 1, 1, e_tok8);
  } else {
    for (int id = EV_LM + 1; id <= EV_MCOMB; ++id) add_event(id, 1, 0, 1, 1, emit_const(p.code, 0));  // MoE: empty
  }
  if (wide) {
    add_event(EV_N1, 1, L, 1, 1, e_tok1);
    add_event(EV_N2, 1, dwide ? L : 0, 1, 1, e_tok1);
    add_event(EV_NF, 1, 1, 1, 1, e_tok1);
  } else {
    for (int id = EV_N1; id < EV_COUNT; ++id) add_event(id, 1, 0, 1, 1, emit_const(p.code, 0));  // wide only: empty
  }
  P.n_counters = base;

  // ---- static schedule: per-SM queues of block instructions in topological
  // (family) order; SM s takes block v = (s - rot_f) mod n_sm of family f, the
  // rotation rot_f spreading the blocks that get one task more.
  std::vector<int> regular;
  for (int f = 0; f < P.n_families; ++f)
    if (!p.fams[f].followup && !mdec) regular.push_back(f);
  P.n_instr_per_sm = (int)regular.size() + 1;
  p.instr.assign((size_t)n_sm * P.n_instr_per_sm, Instr{});
  Binding typical{1, {std::min(1024, P.max_ctx - 1)}};
  long long rot = 0;
  for (size_t k = 0; k < regular.size(); ++k) {
    int f = regular[k];
    for (int s = 0; s < n_sm; ++s) {
      Instr& in = p.instr[(size_t)s * P.n_instr_per_sm + k];
      in.family = f;
      in.v = (int)(((s - rot) % n_sm + n_sm) % n_sm);
      in.n = n_sm;
    }
    rot += p.family_extent(f, typical);
  }
  for (int s = 0; s < n_sm; ++s) {
    Instr& in = p.instr[(size_t)s * P.n_instr_per_sm + regular.size()];
    in.family = -1; in.v = 0; in.n = 1;
  }

  // ---- dynamic queue capacity: pushes per step at the symbols' maxima
  // per layer: QKV (1), ATTN (one per sequence and kv head), OPROJ (1),
  // GATEUP (1), DOWN (one per K segment) -- or for an MoE FFN: ROUTE, EGU,
  // COMBINE (1 each) and EDOWN (one per tile); then LM (1) and END (1)
  // wide batch: NORM, QKV, OPROJ, NORM2, GATEUP (1 each), ATTN (one per
  // sequence), DOWN (one per K segment); then NORMF, LM and END
  // (MoE decoder, wide: NORM, QKV, OPROJ, ROUTE, EGU, COMBINE, ATTN per
  // sequence, EDOWN per tile; then NORMF, LM, END)
  P.queue_ranges = mdec ? (wide ? L * (6 + P.max_batch + P.max_tiles) + 3 : L * (5 + Hkv * P.max_batch + P.max_tiles) + 2)
                   : wide ? L * (5 + P.max_batch + P.n_kc) + 3
                          : L * (3 + Hkv * P.max_batch + P.n_kc) + 2;

  // ---- layer pointers and the rotary table
  p.layers.resize(L);
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights& w = p.layer_w[l];
    p.layers[l] = LayerPtrs{w.attn_norm, w.wq, w.wk, w.wv, w.wo, w.ffn_norm, w.w_gate, w.w_up, w.w_down,
                            w.moe.w_router, w.moe.router_bias, w.moe.w_gate, w.moe.w_up, w.moe.w_down};
  }
  P.embed = m->embed;
  P.lm_head = m->lm_head ? m->lm_head : m->embed;
  P.final_norm = m->final_norm;
  P.k_cache = m->k_cache;
  P.v_cache = m->v_cache;
  p.rope.resize((size_t)P.max_ctx * (D / 2) * 2);
  for (int pos = 0; pos < P.max_ctx; ++pos)
    for (int i = 0; i < D / 2; ++i) {
      double ang = (double)pos * std::pow((double)m->rope_theta, -2.0 * i / D);
      p.rope[((size_t)pos * (D / 2) + i) * 2 + 0] = (float)std::cos(ang);
      p.rope[((size_t)pos * (D / 2) + i) * 2 + 1] = (float)std::sin(ang);
    }
  // ---- device fault injection: one event armed one above its notifies
  if (o->fault == MK_SIM_FAULT_COUNT_PLUS_ONE) {
    const int f = o->fault_family;
    const int op = (f >= 0 && f < P.n_families) ? p.fams[f].op : -1;
    if (op != OP_QKV && op != OP_OPROJ && op != OP_GATEUP && op != OP_DOWN && op != OP_LM)
      { err = "fault_family must be a qkv, oproj, gateup, down or lm family"; return MK_ERR_INVALID_ARG; }
    TaskRec t;
    p.task(f, 0, Binding{1, {0}}, t);  // these families notify the same counter at every binding
    P.fault_ctr = t.notify_ev;
  } else if (o->fault != 0) {
    err = "unknown fault kind";
    return MK_ERR_INVALID_ARG;
  }
  std::vector<unsigned char> image;
  lower_plan(p, image);
  return MK_OK;
}

// ---------------------------------------------------------------- lowering
void lower_plan(Plan& p, std::vector<unsigned char>& image) {
  DevPlan& P = p.dp;
  const int qpg = P.n_kv_heads > 0 ? P.n_q_heads / P.n_kv_heads : 0;  // 0 for an MoE layer
  long long off = 0;
  auto take = [&](long long bytes) { long long at = off; off += (bytes + 255) / 256 * 256; return at; };
  P.off_control = take(sizeof(Control));
  P.off_counters = take(4LL * P.n_counters);
  P.off_families = take((long long)sizeof(FamilyDesc) * P.n_families);
  P.off_expr = take(4LL * (long long)p.code.size());
  P.off_instr = take((long long)sizeof(Instr) * (long long)p.instr.size());
  P.off_layers = take((long long)sizeof(LayerPtrs) * P.n_layers);
  P.off_rope = take(4LL * (long long)p.rope.size());
  // tensor maps of the weights and activation buffers (encoded when the workspace is bound)
  P.off_tmap = take((long long)kTmapBytes * (std::max(P.n_layers, 1) * kTmapPerLayer + kTmapGlobal));
  P.off_queue = take((long long)sizeof(QRange) * P.queue_ranges);
  P.off_x = take(4LL * P.max_batch * P.hidden);
  P.off_q = take(4LL * P.max_batch * P.n_q_heads * P.head_dim);
  P.off_apart = take(4LL * P.max_batch * P.n_kv_heads * P.max_chunks * qpg * (P.head_dim + 2));
  P.off_attn = take(4LL * P.max_batch * P.n_q_heads * P.head_dim);
  P.off_h = take(4LL * P.max_batch * P.ffn);
  P.off_dpart = take(4LL * P.n_kc * P.max_batch * P.hidden);
  P.off_lmbest = take(8LL * P.max_batch);
  // wide batch: the bf16 activations the GEMM tasks load by TMA (act_rows rows
  // each, so that a box of act_rows rows stays inside the buffer)
  const long long ar = P.wide ? act_buf_rows(P.act_split, P.act_rows) : 0;
  P.off_xn = take(2LL * ar * P.hidden);
  P.off_attn_bf = take(2LL * ar * P.hidden);
  P.off_h_bf = take(2LL * ar * P.ffn);
  // wide batch, split K: the partial tiles of the largest phase (fp32
  // [task][parts][128 rows][act_rows]) and the tiles' counters
  long long gtasks = 0;
  if (P.wide) {
    if (P.gseg_qkv > 1) gtasks = std::max(gtasks, (long long)P.n_qkv_tiles);
    if (P.gseg_o > 1) gtasks = std::max(gtasks, (long long)P.n_otiles);
    if (P.gseg_gu > 1 && P.kind == MK_MODEL_DENSE) gtasks = std::max(gtasks, 2LL * P.n_gutiles);
  }
  P.off_gpart = take(gtasks * kWideRows * P.act_rows * 4);
  P.off_gctr = take(P.wide ? 4LL * 3 * kGctrPerOp : 0);
  P.off_actr = take(P.kind == MK_MODEL_MOE_LAYER ? 0 : 4LL * P.max_batch * P.n_kv_heads);
  if (P.kind != MK_MODEL_DENSE) {
    // one MoE scratch block per MoE layer (layer 0's offsets; the others follow at moe_stride)
    const long long pairs = (long long)P.max_tokens * P.top_k;
    const long long block0 = off;
    P.off_mhist = take(4LL * P.n_experts);
    P.off_mrank = take(4 * pairs);
    P.off_midx = take(4 * pairs);
    P.off_mw = take(4 * pairs);
    P.off_mindptr = take(4LL * (P.n_experts + 1));
    P.off_mtile = take(4LL * (P.n_experts + 1));
    P.off_mtile_e = take(4LL * P.max_tiles);
    P.off_mtile_m = take(4LL * P.max_tiles);
    P.off_mperm = take(4 * pairs);
    P.off_mrow = take(4 * pairs);
    P.off_mh = take(2 * pairs * P.eff);
    P.off_my = take(4 * pairs * P.hidden);
    P.off_mxhat = take(2LL * P.max_tokens * P.hidden);
    P.off_mxg = take(2LL * P.n_experts * P.moe_cap * P.hidden);
    P.moe_stride = off - block0;
    const int Lm = P.kind == MK_MODEL_MOE_DECODER ? P.n_layers : 1;
    off += P.moe_stride * (Lm - 1);
  }
  P.ws_bytes = off;
  // image = [off_families, off_queue): the read-only plan arrays
  image.assign((size_t)(P.off_queue - P.off_families), 0);
  auto put = [&](long long at, const void* src, size_t n) {
    if (n) std::memcpy(image.data() + (at - P.off_families), src, n);
  };
  put(P.off_families, p.fams.data(), sizeof(FamilyDesc) * p.fams.size());
  put(P.off_expr, p.code.data(), 4 * p.code.size());
  put(P.off_instr, p.instr.data(), sizeof(Instr) * p.instr.size());
  put(P.off_layers, p.layers.data(), sizeof(LayerPtrs) * p.layers.size());
  put(P.off_rope, p.rope.data(), 4 * p.rope.size());
}

// ---------------------------------------------------------------- bytes
double step_bytes(const Plan& p, const Binding& bd, bool with_logits) {
  const DevPlan& P = p.dp;
  if (P.kind != MK_MODEL_DENSE) return -1.0;  // MoE bytes depend on the routing
  double H = P.hidden, D = P.head_dim, Hq = P.n_q_heads, Hkv = P.n_kv_heads, F = P.ffn;
  double per_layer = ((Hq + 2 * Hkv) * D * H + H * Hq * D + 3 * F * H + 2 * H) * 2.0;
  double w = P.n_layers * per_layer + (double)P.vocab * H * 2.0 + H * 2.0;
  double kv_row = Hkv * D * 2.0 * 2.0 * P.n_layers;  // K and V, all layers
  double ctx_sum = 0;
  for (int b = 0; b < bd.B; ++b) ctx_sum += bd.ctx[b];
  double bytes = w + bd.B * H * 2.0 + kv_row * ctx_sum + kv_row * bd.B + bd.B * 4.0 * 2;
  if (with_logits) bytes += 4.0 * P.vocab * bd.B;
  return bytes;
}

// ---------------------------------------------------------------- validation
static bool check_binding(const Plan& p, const Binding& bd, std::string& err) {
  if (p.dp.kind == MK_MODEL_MOE_LAYER) {  // B is the token count; no contexts
    if (bd.B < 1 || bd.B > p.dp.max_tokens) { err = "token count out of range"; return false; }
    return true;
  }
  if (bd.B < 1 || bd.B > p.dp.max_batch) { err = "batch out of range"; return false; }
  if ((int)bd.ctx.size() < bd.B) { err = "ctx_lens shorter than batch"; return false; }
  for (int b = 0; b < bd.B; ++b)
    if (bd.ctx[b] < 0 || bd.ctx[b] >= p.dp.max_ctx) { err = "ctx_lens[b] out of [0, max_ctx)"; return false; }
  return true;
}

// Wait count of a counter for a binding: the armed expression, or for the
// MoE events armed at run time by the routing follow-up (EV_MY: one per down
// task; EV_MH: one per gate/up task of a tile the routing made) their value
// after that arming.
static int runtime_count(const Plan& p, int ev, int c0, int c1, int c2, const Binding& bd) {
  if (ev == EV_MY && c0 < (int)bd.route.size()) return bd.route[c0].tiles * p.dp.nt_d;
  if (ev == EV_MH && c0 < (int)bd.route.size()) return c1 < bd.route[c0].tiles ? p.dp.nt_gu : 0;
  return p.event_count(ev, c0, c1, c2, bd);
}

mk_status validate_plan(const Plan& p, const Binding& bd_in, std::string& err) {
  if (!check_binding(p, bd_in, err)) return MK_ERR_INVALID_ARG;
  Binding bd = bd_in;
  if (p.dp.kind != MK_MODEL_DENSE && bd.route.empty()) draw_routing(p, bd, 0, 0.0);
  const DevPlan& P = p.dp;
  std::vector<int> notifiers(P.n_counters, 0);
  std::vector<int> last_notifier_fam(P.n_counters, -1);
  std::vector<int> wait_fams;  // (counter, fam) pairs
  std::vector<std::pair<int, int>> waits;
  TaskRec t;
  std::vector<int> followups_seen(P.n_families, 0);
  for (int f = 0; f < P.n_families; ++f) {
    int n = p.actual_extent(f, bd);
    if (n < 0 || n > p.fams[f].max_extent) {
      err = "family " + p.fam_names[f] + " extent exceeds its reserved maximum";
      return MK_ERR_PLAN;
    }
    for (int i = 0; i < n; ++i) {
      p.task(f, i, bd, t);
      if (!t.exists) continue;
      if (t.notify_ev >= 0) {
        notifiers[t.notify_ev]++;
        last_notifier_fam[t.notify_ev] = std::max(last_notifier_fam[t.notify_ev], f);
      }
      if (t.wait_ev >= 0) waits.push_back({t.wait_ev, f});
      if (t.follow_fam >= 0 && t.follow_fam <= f) {
        err = "follow-up family precedes its trigger";
        return MK_ERR_PLAN;
      }
    }
  }
  // every armed count equals its number of notifiers
  for (int e = 0; e < EV_COUNT; ++e) {
    const EventTensorDesc& d = P.ev[e];
    int d1 = d.ndim > 1 ? d.dims[1] : 1, d2 = d.ndim > 2 ? d.dims[2] : 1;
    for (int a = 0; a < d.dims[0]; ++a)
      for (int b = 0; b < d1; ++b)
        for (int c = 0; c < d2; ++c) {
          int ci = p.counter(e, a, b, c);
          int cnt = runtime_count(p, e, a, b, c, bd);
          if (cnt != notifiers[ci]) {
            err = "event " + std::to_string(e) + " element (" + std::to_string(a) + "," + std::to_string(b) +
                  "," + std::to_string(c) + ") waits for " + std::to_string(cnt) + " but has " +
                  std::to_string(notifiers[ci]) + " notifiers";
            return MK_ERR_PLAN;
          }
        }
  }
  // waits only on events notified by earlier families (acyclic, topological)
  for (auto& w : waits)
    if (last_notifier_fam[w.first] >= w.second) {
      err = "family " + p.fam_names[w.second] + " waits on an event notified by a later family";
      return MK_ERR_PLAN;
    }
  // static queues are sorted in family order (deadlock freedom)
  for (int s = 0; s < P.n_sm; ++s) {
    int prev = -1;
    for (int k = 0; k < P.n_instr_per_sm; ++k) {
      const Instr& in = p.instr[(size_t)s * P.n_instr_per_sm + k];
      if (in.family < 0) break;
      if (in.family <= prev) { err = "static queue out of topological order"; return MK_ERR_PLAN; }
      prev = in.family;
    }
  }
  return MK_OK;
}

// ---------------------------------------------------------------- simulator
namespace {

struct VC {
  std::vector<unsigned> c;
  void join(const VC& o) { for (size_t i = 0; i < c.size(); ++i) c[i] = std::max(c[i], o.c[i]); }
};

struct Shadow {
  int w_worker = -1;
  unsigned w_clock = 0;
  std::vector<unsigned> reads;  // per worker
};

struct Sim {
  const Plan& p;
  const Binding& bd;
  int nw;
  std::vector<VC> wvc;
  std::vector<VC> evc;
  std::vector<int> counters;
  std::vector<std::unordered_map<long long, Shadow>> shadow;
  int races = 0;
  std::string first;
  Sim(const Plan& pl, const Binding& b, int n) : p(pl), bd(b), nw(n), shadow(BUF_COUNT) {}

  void access(int w, const Region& r, bool write) {
    // shadow units: 4 elements for row data, 1 for per-task records
    const long long G = (r.buf == BUF_APART || r.buf == BUF_NEXT) ? 1 : 4;
    for (long long u = r.lo / G; u <= (r.hi - 1) / G; ++u) {
      Shadow& s = shadow[r.buf][u];
      if (s.reads.empty()) s.reads.assign(nw, 0);
      const VC& me = wvc[w];
      bool ok = s.w_worker < 0 || s.w_worker == w || me.c[s.w_worker] >= s.w_clock;
      if (write)
        for (int r2 = 0; r2 < nw && ok; ++r2)
          if (r2 != w && s.reads[r2] > me.c[r2]) ok = false;
      if (!ok) {
        if (!races) first = "unordered access to buffer " + std::to_string(r.buf) + " unit " + std::to_string(u);
        races++;
      }
      if (write) { s.w_worker = w; s.w_clock = me.c[w]; std::fill(s.reads.begin(), s.reads.end(), 0); }
      else s.reads[w] = std::max(s.reads[w], me.c[w]);
    }
  }
};

struct Work {
  int fam, idx;
  std::vector<unsigned> vc;  // dynamic: clock snapshot carried by a pushed task
};

}  // namespace

static int run_order(const Plan& p, const Binding& bd, bool dynamic, std::mt19937& rng, int fault,
                     int fault_family, std::vector<int>& exec_count, mk_sim_report* rep) {
  const DevPlan& P = p.dp;
  int nw = std::max(1, std::min(P.n_sm, 64));
  Sim sim(p, bd, nw);
  sim.wvc.assign(nw, VC{std::vector<unsigned>(nw, 0)});
  sim.evc.assign(P.n_counters, VC{std::vector<unsigned>(nw, 0)});
  sim.counters.assign(P.n_counters, 0);
  bool fault_done = false;
  // clock of each event when its counter reached zero (armed at zero: none)
  std::vector<VC> fired(P.n_counters, VC{std::vector<unsigned>(nw, 0)});
  for (int e = 0; e < EV_COUNT; ++e) {
    const EventTensorDesc& d = P.ev[e];
    int d1 = d.ndim > 1 ? d.dims[1] : 1, d2 = d.ndim > 2 ? d.dims[2] : 1;
    for (int a = 0; a < d.dims[0]; ++a)
      for (int b = 0; b < d1; ++b)
        for (int c = 0; c < d2; ++c) sim.counters[p.counter(e, a, b, c)] = p.event_count(e, a, b, c, bd);
  }
  std::vector<int> ext(P.n_families);
  for (int f = 0; f < P.n_families; ++f) ext[f] = p.actual_extent(f, bd);
  // wrong wait counts: the event task 0 of the fault family notifies, armed
  // one above or one below its notifies (again after a run-time arming)
  int fault_ctr = -1, fault_delta = 0;
  if ((fault == MK_SIM_FAULT_COUNT_PLUS_ONE || fault == MK_SIM_FAULT_COUNT_MINUS_ONE) && fault_family >= 0 &&
      fault_family < P.n_families && ext[fault_family] > 0) {
    TaskRec t0;
    p.task(fault_family, 0, bd, t0);
    fault_ctr = t0.notify_ev;
    fault_delta = fault == MK_SIM_FAULT_COUNT_PLUS_ONE ? 1 : -1;
    if (fault_ctr >= 0) sim.counters[fault_ctr] += fault_delta;
  }

  // per-worker task sources
  std::vector<std::vector<Work>> local(nw);   // static: own queue; both: follow-ups
  std::vector<size_t> pos(nw, 0);
  std::vector<std::vector<Work>> follow(nw);
  std::vector<Work> shared;                   // dynamic queue (FIFO)
  size_t shared_head = 0;
  int ranges_pushed = 0;                      // queue entries the device would write
  if (!dynamic) {
    // simulated SM w plays the SMs congruent to w mod nw, in queue order
    for (int s = 0; s < P.n_sm; ++s) {
      int w = s % nw;
      for (int k = 0; k < P.n_instr_per_sm; ++k) {
        const Instr& in = p.instr[(size_t)s * P.n_instr_per_sm + k];
        if (in.family < 0) break;
        int lo, hi;
        instr_range(in, ext[in.family], lo, hi);
        for (int i = lo; i < hi; ++i) local[w].push_back({in.family, i, {}});
      }
    }
    for (int w = 0; w < nw; ++w)
      std::stable_sort(local[w].begin(), local[w].end(),
                       [](const Work& a, const Work& b) { return a.fam < b.fam; });
  } else {
    // the launch's first push, as on the device: the routing tasks of an MoE
    // layer call, or the QKV tiles of layer 0 of a decoder
    const int f0 = P.kind == MK_MODEL_MOE_LAYER ? p.fam_index(OP_ROUTE, -1)
                   : P.wide ? p.fam_index(OP_NORM, 0) : p.fam_index(OP_QKV, 0);
    ranges_pushed += 1;
    for (int i = 0; i < ext[f0]; ++i) shared.push_back({f0, i, std::vector<unsigned>(nw, 0)});
  }
  TaskRec t;
  int executed = 0;
  auto exec = [&](int w, const Work& wk) {
    VC& me = sim.wvc[w];
    me.c[w]++;
    p.task(wk.fam, wk.idx, bd, t);
    if (!wk.vc.empty()) { VC v{wk.vc}; me.join(v); }
    bool skip_wait = fault == MK_SIM_FAULT_NO_WAIT && wk.fam == fault_family;
    // the wait synchronises with the notifies that took the counter to zero
    // (a later, surplus notify is not ordered before the waiter)
    if (t.wait_ev >= 0 && !skip_wait) me.join(fired[t.wait_ev]);
    for (auto& r : t.reads) sim.access(w, r, false);
    for (auto& r : t.writes) sim.access(w, r, true);
    exec_count[p.fams[wk.fam].debug_base + wk.idx]++;
    executed++;
    if (p.fams[wk.fam].op == OP_MINDPTR) {
      // data-dependent event update: the routing follow-up arms the down
      // count and the gate/up count of every tile the routing made
      const int li = p.fams[wk.fam].layer < 0 ? 0 : p.fams[wk.fam].layer;
      const int cmy = p.counter(EV_MY, li);
      sim.counters[cmy] = bd.route[li].tiles * P.nt_d + (cmy == fault_ctr ? fault_delta : 0);
      for (int tl = 0; tl < bd.route[li].tiles; ++tl) {
        const int cmh = p.counter(EV_MH, li, tl);
        sim.counters[cmh] = P.nt_gu + (cmh == fault_ctr ? fault_delta : 0);
      }
    }
    if (t.notify_ev >= 0) {
      if (fault == MK_SIM_FAULT_DROP_NOTIFY && wk.fam == fault_family && !fault_done) { fault_done = true; return; }
      sim.evc[t.notify_ev].join(me);
      int old = sim.counters[t.notify_ev]--;
      auto push_succ = [&]() {
        std::vector<int> succ;
        p.successors(t.notify_ev, bd, succ);
        ranges_pushed += (int)succ.size() / 3;
        for (size_t k = 0; k < succ.size(); k += 3)
          for (int i = 0; i < succ[k + 2]; ++i) shared.push_back({succ[k], succ[k + 1] + i, me.c});
      };
      if (old == 1) {
        fired[t.notify_ev] = sim.evc[t.notify_ev];
        me.join(sim.evc[t.notify_ev]);  // the last notifier acquires every release
        if (t.follow_fam >= 0) follow[w].push_back({t.follow_fam, t.follow_idx, {}});
        if (dynamic) push_succ();
      }
    }
  };
  std::vector<Work> held(nw);
  std::vector<char> held_ok(nw, 0);
  auto ready = [&](int w) -> int {  // 1 follow-up, 2 regular, 0 blocked
    if (!follow[w].empty()) return 1;
    if (!dynamic) {
      if (pos[w] >= local[w].size()) return 0;
      TaskRec tr;
      p.task(local[w][pos[w]].fam, local[w][pos[w]].idx, bd, tr);
      bool skip_wait = fault == MK_SIM_FAULT_NO_WAIT && local[w][pos[w]].fam == fault_family;
      if (tr.wait_ev >= 0 && sim.counters[tr.wait_ev] != 0 && !skip_wait) return 0;
      return 2;
    }
    // dynamic: a worker pops the queue head into its held slot and runs it
    // once its event has fired (the device's controller waits on the counter
    // of a popped task as well)
    if (!held_ok[w]) {
      if (shared_head >= shared.size()) return 0;
      held[w] = shared[shared_head++];
      held_ok[w] = true;
    }
    TaskRec tr;
    p.task(held[w].fam, held[w].idx, bd, tr);
    bool skip_wait = fault == MK_SIM_FAULT_NO_WAIT && held[w].fam == fault_family;
    if (tr.wait_ev >= 0 && sim.counters[tr.wait_ev] > 0 && !skip_wait) return 0;
    return 2;
  };
  std::vector<int> cand;
  for (;;) {
    cand.clear();
    for (int w = 0; w < nw; ++w)
      if (ready(w)) cand.push_back(w);
    if (cand.empty()) break;
    int w = cand[rng() % cand.size()];
    int kind = ready(w);
    if (kind == 1) {
      // follow-ups run in LIFO order on the notifier, like the device
      Work wk = follow[w].back();
      follow[w].pop_back();
      exec(w, wk);
    } else if (!dynamic) {
      exec(w, local[w][pos[w]++]);
    } else {
      held_ok[w] = false;
      exec(w, held[w]);
    }
  }
  if (dynamic) {
    ranges_pushed += 1;  // the END range pushed after the last task
    if (ranges_pushed > P.queue_ranges) {
      rep->deadlocks++;
      if (!rep->first_error[0])
        std::snprintf(rep->first_error, sizeof(rep->first_error), "dynamic queue needs %d ranges, plan reserves %d",
                      ranges_pushed, P.queue_ranges);
    }
  }
  bool left = false;
  for (int w = 0; w < nw; ++w)
    if ((!dynamic && pos[w] < local[w].size()) || !follow[w].empty()) left = true;
  if (dynamic && shared_head < shared.size()) left = true;
  for (int w = 0; w < nw; ++w)
    if (held_ok[w]) left = true;
  // a plan that stops before the final task has deadlocked
  int fin = p.fam_index(P.kind == MK_MODEL_MOE_LAYER ? OP_MFIN : OP_LMFIN, -1);
  if (exec_count[p.fams[fin].debug_base] == 0) left = true;
  if (left) rep->deadlocks++;
  for (int ci = 0; ci < P.n_counters; ++ci)
    if (sim.counters[ci] != 0) { rep->nonzero_counters++; break; }
  rep->races += sim.races;
  if (sim.races && !rep->first_error[0])
    std::snprintf(rep->first_error, sizeof(rep->first_error), "%s", sim.first.c_str());
  if (left && !rep->first_error[0])
    std::snprintf(rep->first_error, sizeof(rep->first_error), "order stopped with tasks left (deadlock)");
  rep->tasks_per_order = executed;
  return executed;
}

mk_status simulate_plan(const Plan& p, const Binding& bd_in, int n_orders, unsigned seed, int fault,
                        int fault_family, mk_sim_report* rep) {
  std::string err;
  std::memset(rep, 0, sizeof(*rep));
  if (!check_binding(p, bd_in, err)) {
    std::snprintf(rep->first_error, sizeof(rep->first_error), "%s", err.c_str());
    return MK_ERR_INVALID_ARG;
  }
  // MoE plans: a routing drawn from the seed (odd seeds skewed), dynamic orders only
  Binding bd = bd_in;
  const bool moe = p.dp.kind != MK_MODEL_DENSE;
  if (moe) draw_routing(p, bd, seed, (seed & 1u) ? 1.2 : 0.0);
  std::mt19937 rng(seed);
  std::vector<int> want(p.dp.debug_slots, 0);
  for (int f = 0; f < p.dp.n_families; ++f)
    for (int i = 0; i < p.actual_extent(f, bd); ++i) {
      TaskRec t;
      p.task(f, i, bd, t);
      if (t.exists) want[p.fams[f].debug_base + i] = 1;
    }
  std::vector<int> first_set;
  for (int k = 0; k < n_orders; ++k) {
    bool dynamic = moe || (k % 2) == 1;
    std::vector<int> exec_count(p.dp.debug_slots, 0);
    run_order(p, bd, dynamic, rng, fault, fault_family, exec_count, rep);
    rep->orders_run++;
    if (exec_count != want) {
      rep->exactly_once_violations++;
      if (!rep->first_error[0]) std::snprintf(rep->first_error, sizeof(rep->first_error), "task set differs from the plan's");
    }
    std::vector<int> set(exec_count.size());
    for (size_t i = 0; i < set.size(); ++i) set[i] = exec_count[i] > 0;
    if (k == 0) first_set = set;
    else if (set != first_set) rep->static_dynamic_mismatch = 1;
  }
  bool bad = rep->races || rep->deadlocks || rep->exactly_once_violations || rep->nonzero_counters ||
             rep->static_dynamic_mismatch;
  return bad ? MK_ERR_PLAN : MK_OK;
}

}  // namespace mk
