// api.cpp — the extern "C" boundary of libmk.so (declared in include/mk.h).
// No exception crosses it; every failure returns an mk_status and leaves a
// message for mk_last_error().
#include <cuda_runtime.h>

#include <atomic>
#include <stdexcept>
#include <chrono>
#include <cstring>
#include <new>
#include <string>

#include "../../include/mk.h"
#include "launch.hpp"
#include "plan.hpp"

struct mk_plan {
  mk::Plan p;
};

namespace {
thread_local std::string g_err;

mk_status fail(mk_status s, const std::string& msg) {
  g_err = msg;
  return s;
}

bool binding_from(const mk_plan* hp, int batch, const int* ctx, mk::Binding& bd) {
  if (!hp || batch < 1) return false;
  bd.B = batch;
  if (hp->p.dp.kind == MK_MODEL_MOE_LAYER) {  // batch = tokens; no contexts
    if (batch > hp->p.dp.max_tokens) return false;
    bd.ctx.assign(batch, 0);
    return true;
  }
  if (batch > hp->p.dp.max_batch || !ctx) return false;
  bd.ctx.assign(ctx, ctx + batch);
  return true;
}
}  // namespace

extern "C" {

const char* mk_last_error(void) { return g_err.c_str(); }

mk_status mk_plan_build(const mk_model_desc* m, const mk_plan_opts* opts, mk_plan** out) {
  g_err.clear();
  const auto t_build0 = std::chrono::steady_clock::now();
  if (!m || !opts || !out) return fail(MK_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  try {
    int n_sm = opts->n_sm, smem = opts->smem_bytes, device = -1;
    std::string err;
    if (!opts->host_only) {
      int dev_sm = 0, optin = 0;
      mk_status s = mk::dev_query(&dev_sm, &optin, &device, err);
      if (s != MK_OK) return fail(s, err);
      if (n_sm <= 0) n_sm = dev_sm;
      if (n_sm > dev_sm) return fail(MK_ERR_INVALID_ARG, "n_sm exceeds the device's SM count");
      if (smem <= 0 || smem > optin) smem = optin;
    } else {
      if (n_sm <= 0) n_sm = 148;
      if (smem <= 0) smem = 232448;
    }
    mk_plan* hp = new mk_plan();
    mk_status s = mk::build_plan(m, opts, n_sm, smem, hp->p, err);
    if (s == MK_OK) {
      // the plan must validate on a small binding of the symbols before use
      // (MoE plans: on a routing drawn from a fixed seed)
      const bool layer = hp->p.dp.kind == MK_MODEL_MOE_LAYER;
      const int B = layer ? std::min(hp->p.dp.max_tokens, 16) : hp->p.dp.max_batch;
      std::vector<int> ctx(B, layer ? 0 : std::min(hp->p.dp.max_ctx - 1, 3 * hp->p.dp.chunk - 1));
      mk::Binding bd{B, ctx, {}};
      s = mk::validate_plan(hp->p, bd, err);
    }
    if (s != MK_OK) {
      delete hp;
      return fail(s, err);
    }
    static std::atomic<unsigned long long> next_uid{1};
    hp->p.device = device;
    hp->p.uid = next_uid++;
    hp->p.build_ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t_build0).count();
    *out = hp;
    return MK_OK;
  } catch (const std::bad_alloc&) {
    return fail(MK_ERR_INVALID_ARG, "out of host memory");
  } catch (const std::exception& e) {
    return fail(MK_ERR_PLAN, std::string("unexpected error while building the plan: ") + e.what());
  } catch (...) {
    return fail(MK_ERR_PLAN, "unexpected error while building the plan");
  }
}

size_t mk_plan_workspace_bytes(const mk_plan* p) { return p ? (size_t)p->p.dp.ws_bytes : 0; }

mk_status mk_plan_bind_workspace(mk_plan* hp, void* dev_ptr, size_t bytes, void* stream) {
  g_err.clear();
  if (!hp) return fail(MK_ERR_INVALID_ARG, "null plan");
  if (hp->p.device < 0) return fail(MK_ERR_UNSUPPORTED, "plan was built host_only");
  if (!dev_ptr || bytes < (size_t)hp->p.dp.ws_bytes)
    return fail(MK_ERR_WORKSPACE, "workspace missing or smaller than mk_plan_workspace_bytes()");
  if (((uintptr_t)dev_ptr) & 255) return fail(MK_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  try {
    std::vector<unsigned char> image;
    mk::lower_plan(hp->p, image);
    std::string err;
    mk_status s = mk::dev_bind(hp->p, dev_ptr, bytes, stream, image, err);
    if (s != MK_OK) return fail(s, err);
    hp->p.ws = dev_ptr;
    hp->p.ws_bound = bytes;
    return MK_OK;
  } catch (...) {
    return fail(MK_ERR_CUDA, "unexpected error while binding the workspace");
  }
}

mk_status mk_decode_step(mk_plan* hp, const mk_step_args* a, void* stream) {
  g_err.clear();
  if (!hp || !a) return fail(MK_ERR_INVALID_ARG, "null argument");
  if (hp->p.dp.kind == MK_MODEL_MOE_LAYER) return fail(MK_ERR_INVALID_ARG, "plan is an MoE layer (use mk_moe_layer)");
  if (!hp->p.ws) return fail(MK_ERR_WORKSPACE, "no workspace bound");
  if (a->batch < 1 || a->batch > hp->p.dp.max_batch) return fail(MK_ERR_INVALID_ARG, "batch out of [1, max_batch]");
  if (!a->token_ids || !a->slot_ids || !a->ctx_lens || !a->next_tokens)
    return fail(MK_ERR_INVALID_ARG, "token_ids, slot_ids, ctx_lens and next_tokens are required");
  std::string err;
  mk_status s = mk::dev_launch(hp->p, a, stream, err);
  return s == MK_OK ? MK_OK : fail(s, err);
}

mk_status mk_decode_step_static(mk_plan* hp, const mk_step_args* a, void* stream) {
  g_err.clear();
  if (!hp || !a) return fail(MK_ERR_INVALID_ARG, "null argument");
  if (hp->p.dp.kind != MK_MODEL_DENSE) return fail(MK_ERR_INVALID_ARG, "plan is not a dense decoder");
  if (hp->p.device < 0) return fail(MK_ERR_UNSUPPORTED, "plan was built host_only");
  if (a->batch < 1 || a->batch > hp->p.dp.max_batch) return fail(MK_ERR_INVALID_ARG, "batch out of [1, max_batch]");
  if (!a->token_ids || !a->slot_ids || !a->ctx_lens || !a->next_tokens)
    return fail(MK_ERR_INVALID_ARG, "token_ids, slot_ids, ctx_lens and next_tokens are required");
  if ((unsigned long long)hp->p.dp.ws_bytes > (unsigned long long)MK_STATIC_SCRATCH_BYTES)
    return fail(MK_ERR_WORKSPACE, "plan needs " + std::to_string(hp->p.dp.ws_bytes) +
                                      " bytes of scratch; the static scratch holds " +
                                      std::to_string((unsigned long long)MK_STATIC_SCRATCH_BYTES));
  try {
    std::string err;
    mk_status s = mk::dev_launch_static(hp->p, a, stream, err);
    return s == MK_OK ? MK_OK : fail(s, err);
  } catch (...) {
    return fail(MK_ERR_CUDA, "unexpected error in the static-scratch decode step");
  }
}

mk_status mk_moe_layer(mk_plan* hp, const mk_moe_args* a, void* stream) {
  g_err.clear();
  if (!hp || !a) return fail(MK_ERR_INVALID_ARG, "null argument");
  if (hp->p.dp.kind != MK_MODEL_MOE_LAYER) return fail(MK_ERR_INVALID_ARG, "plan is not an MoE layer");
  if (!hp->p.ws) return fail(MK_ERR_WORKSPACE, "no workspace bound");
  if (a->n_tokens < 1 || a->n_tokens > hp->p.dp.max_tokens)
    return fail(MK_ERR_INVALID_ARG, "n_tokens out of [1, max_tokens]");
  if (!a->x || !a->out) return fail(MK_ERR_INVALID_ARG, "x and out are required");
  std::string err;
  mk_status s = mk::dev_launch_moe(hp->p, a, stream, err);
  return s == MK_OK ? MK_OK : fail(s, err);
}

mk_status mk_get_stats(mk_plan* hp, mk_stats* st) {
  g_err.clear();
  if (!hp || !st) return fail(MK_ERR_INVALID_ARG, "null argument");
  const mk::DevPlan& P = hp->p.dp;
  st->launches = hp->p.launches;
  st->build_ms = hp->p.build_ms;
  st->n_families = P.n_families;
  st->n_counters = P.n_counters;
  st->ring_slots = P.ring_slots;
  st->n_sm = P.n_sm;
  st->workspace_bytes = P.ws_bytes;
  st->queue_ranges_cap = P.sched == MK_SCHED_DYNAMIC ? P.queue_ranges : 0;
  st->last_queue_ranges = -1;
  st->last_queue_tasks = -1;
  st->last_queue_pops = -1;
  if (hp->p.ws && hp->p.launches > 0 && P.sched == MK_SCHED_DYNAMIC) {
    mk::Control c;
    cudaError_t e = cudaMemcpy(&c, (unsigned char*)hp->p.ws + P.off_control, sizeof(c), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(MK_ERR_CUDA, std::string("control block read failed: ") + cudaGetErrorString(e));
    st->last_queue_ranges = (int)(c.q_tail >> 40);
    st->last_queue_tasks = (long long)(c.q_tail & ((1ull << 40) - 1));
    st->last_queue_pops = (long long)c.q_head;
  }
  return MK_OK;
}

mk_status mk_get_status(mk_plan* hp, mk_device_status* st) {
  g_err.clear();
  if (!hp || !st) return fail(MK_ERR_INVALID_ARG, "null argument");
  if (!hp->p.ws) return fail(MK_ERR_WORKSPACE, "no workspace bound");
  std::string err;
  mk_status s = mk::dev_status(hp->p, st, err);
  if (s == MK_ERR_CUDA) return fail(s, err);
  if (s != MK_OK) g_err = "device reported an error";
  return s;
}

mk_status mk_plan_reset(mk_plan* hp, void* stream) {
  g_err.clear();
  if (!hp) return fail(MK_ERR_INVALID_ARG, "null plan");
  if (!hp->p.ws) return fail(MK_ERR_WORKSPACE, "no workspace bound");
  std::string err;
  mk_status s = mk::dev_reset(hp->p, stream, err);
  return s == MK_OK ? MK_OK : fail(s, err);
}

int mk_plan_task_slots(const mk_plan* hp) { return hp ? hp->p.dp.debug_slots : 0; }
int mk_plan_num_families(const mk_plan* hp) { return hp ? hp->p.dp.n_families : 0; }

mk_status mk_plan_family_info(const mk_plan* hp, int f, mk_family_info* out) {
  g_err.clear();
  if (!hp || !out || f < 0 || f >= hp->p.dp.n_families) return fail(MK_ERR_INVALID_ARG, "bad family index");
  const mk::FamilyDesc& d = hp->p.fams[f];
  out->op = d.op;
  out->layer = d.layer;
  out->debug_base = d.debug_base;
  out->max_extent = d.max_extent;
  out->followup = d.followup;
  std::memset(out->name, 0, sizeof(out->name));
  std::strncpy(out->name, hp->p.fam_names[f].c_str(), sizeof(out->name) - 1);
  return MK_OK;
}

mk_status mk_plan_counter_region(const mk_plan* hp, long long* byte_offset, int* n_counters) {
  g_err.clear();
  if (!hp || !byte_offset || !n_counters) return fail(MK_ERR_INVALID_ARG, "null argument");
  *byte_offset = hp->p.dp.off_counters;
  *n_counters = hp->p.dp.n_counters;
  return MK_OK;
}

mk_status mk_plan_tiles(const mk_plan* hp, int* o) {
  g_err.clear();
  if (!hp || !o) return fail(MK_ERR_INVALID_ARG, "null argument");
  const mk::DevPlan& P = hp->p.dp;
  int v[16] = {P.tile_qkv, P.tile_o, P.tile_gu, P.tile_down, P.kseg, P.tile_lm, P.chunk, P.n_sm, P.ring_slots,
               P.attn_split, P.wide, P.act_split, P.gseg_qkv, P.gseg_o, P.gseg_gu, P.attn_auto};
  std::memcpy(o, v, sizeof(v));
  return MK_OK;
}

mk_status mk_plan_validate(const mk_plan* hp, int batch, const int* ctx) {
  g_err.clear();
  mk::Binding bd;
  if (!binding_from(hp, batch, ctx, bd)) return fail(MK_ERR_INVALID_ARG, "bad binding");
  try {
    std::string err;
    mk_status s = mk::validate_plan(hp->p, bd, err);
    return s == MK_OK ? MK_OK : fail(s, err);
  } catch (...) {
    return fail(MK_ERR_PLAN, "unexpected error during validation");
  }
}

mk_status mk_plan_simulate(const mk_plan* hp, int batch, const int* ctx, int n_orders, unsigned seed, int fault,
                           int fault_family, mk_sim_report* rep) {
  g_err.clear();
  mk::Binding bd;
  if (!rep || n_orders < 1) return fail(MK_ERR_INVALID_ARG, "bad arguments");
  if (!binding_from(hp, batch, ctx, bd)) return fail(MK_ERR_INVALID_ARG, "bad binding");
  try {
    mk_status s = mk::simulate_plan(hp->p, bd, n_orders, seed, fault, fault_family, rep);
    return s == MK_OK ? MK_OK : fail(s, rep->first_error);
  } catch (...) {
    return fail(MK_ERR_PLAN, "unexpected error during simulation");
  }
}

double mk_plan_step_bytes(const mk_plan* hp, int batch, const int* ctx, int with_logits) {
  mk::Binding bd;
  if (!binding_from(hp, batch, ctx, bd)) return -1.0;
  return mk::step_bytes(hp->p, bd, with_logits != 0);
}

void mk_plan_destroy(mk_plan* hp) { delete hp; }

}  // extern "C"
