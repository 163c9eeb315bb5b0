// megakernel.cu — one persistent sm_100a kernel that runs a whole decode step.
//
// Execution model ("Lecture 112: Production Megakernels for Real-World
// Inference", sections "Execution Model" and "Memory Pipelining"; "Event
// Tensor: A Unified Abstraction for Compiling Dynamic Megakernel", section
// "Core method"): one CTA per SM, each running an interpreter — a loop over a
// switch — over tasks taken from a queue in device memory (static: this SM's
// instruction list; dynamic: a shared queue that tasks are pushed onto when
// their event fires).  Tasks synchronise only through Event Tensor counters:
// notify() is an acquire-release atomic decrement, wait() spins until zero.
//
// Warp roles inside a CTA (320 threads):
//   warp 0  producer   walks the task stream ahead of execution and streams
//                      each task's weights (and cached KV rows) into a ring of
//                      16 KB shared-memory slots with bulk async copies; it
//                      never waits on events, so weight traffic runs ahead of
//                      synchronisation (weights do not depend on activations).
//   warp 1  controller waits on each task's event, hands the task to the
//                      compute warps, and notifies its events afterwards; the
//                      notifier whose decrement reaches zero runs the event's
//                      follow-up task (merge / reduction) and, in dynamic mode,
//                      pushes the event's consumer tasks.
//   warps 2-9 compute  RMSNorm-fused GEMV tiles, split-KV attention, merges.
// Every spin is bounded by the plan's timeout; on expiry the kernel records an
// error in the control block, raises an abort flag that every spin polls,
// drains its in-flight copies and exits.
#include <cuda_runtime.h>

#include "../../include/mk.h"
#include "device.cuh"
#include "plan_format.h"

namespace mk {

constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 64;
constexpr int kCtlThreads = kComputeThreads + 32;
constexpr int kFifo = 16;
constexpr int kMaxSlots = 16;
constexpr int kMaxFollow = 8;
constexpr int kMaxB = 4;        // batch rows a GEMV task keeps in registers
constexpr int kAccRows = 16;    // rows a compute thread accumulates per task
constexpr int BAR_GO = 1, BAR_DONE = 2, BAR_COMP = 3;
constexpr int kDynLookahead = 2;

struct StepParams {
  int B;
  const int* tokens;
  const int* slots;
  const int* ctx;
  float* logits;
  int* next_tokens;
  unsigned* task_counts;
  unsigned epoch;
};

struct TaskDesc {
  int32_t fam, op, layer, idx;
  int32_t ring_seq, nslots, pad0, pad1;
};

struct Smem {
  uint64_t full[kMaxSlots], empty[kMaxSlots];
  uint64_t fifo_full[kFifo], fifo_empty[kFifo];
  TaskDesc fifo[kFifo];
  TaskDesc cur;
  TaskDesc follow[kMaxFollow];
  int ctx[kMaxBatch], slot[kMaxBatch], tok[kMaxBatch], nch[kMaxBatch], pre[kMaxBatch + 1];
  int fam_ext[kMaxFamilies];
  float red[kComputeWarps][kAccRows * kMaxB];
  float fin[128 * kMaxB];
  float qs[256];
  float sc[4][64];
  float hm[4], hl[4];
  float newk[64], newv[64];
  volatile int released;  // regular tasks the controller has handed to compute
  int bad;
};
static_assert(sizeof(Smem) <= 14 * 1024, "fixed shared-memory area exceeds its reserve");

// ---------------------------------------------------------------- errors
__device__ void record_error(Control* ctl, int code, int fam, int idx, int ev) {
  if (atomicCAS(&ctl->status_code, 0, code) == 0) {
    ctl->status_family = fam;
    ctl->status_index = idx;
    ctl->status_event = ev;
    ctl->status_sm = blockIdx.x;
  }
  atomicExch(&ctl->abort, 1);
}

__device__ __forceinline__ bool aborted(Control* ctl) { return *(volatile int*)&ctl->abort != 0; }

// Bounded wait on an mbarrier phase; false if the kernel is aborting.
__device__ bool wait_mbar(uint64_t* bar, uint32_t parity, Control* ctl, long long timeout_ns, int fam, int idx) {
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

// ---------------------------------------------------------------- plan helpers
__device__ __forceinline__ int ev_ctr(const DevPlan& P, int ev, int c0, int c1 = 0, int c2 = 0) {
  const EventTensorDesc& e = P.ev[ev];
  int lin = c0;
  if (e.ndim > 1) lin = lin * e.dims[1] + c1;
  if (e.ndim > 2) lin = lin * e.dims[2] + c2;
  return e.base + lin;
}
__device__ __forceinline__ int fam_of(const DevPlan& P, int op, int layer) {
  return op >= OP_LM ? P.fam_first_layer[op] : P.fam_first_layer[op] + layer * P.fam_stride;
}
__device__ __forceinline__ bool is_followup(int op) {
  return op == OP_MERGE || op == OP_DRED || op == OP_LMGRP || op == OP_LMFIN;
}

// Counter a regular task waits on (-1: none).
__device__ int wait_counter(const DevPlan& P, const Smem& sm, const TaskDesc& t, int B) {
  switch (t.op) {
    case OP_QKV: return ev_ctr(P, EV_IN, t.layer);
    case OP_ATTN: {
      AttnTask a = decode_attn(t.idx, B, P.n_kv_heads, sm.nch, sm.pre);
      return ev_ctr(P, EV_QKV, t.layer, a.g);
    }
    case OP_OPROJ: return ev_ctr(P, EV_ATTN, t.layer);
    case OP_GATEUP: return ev_ctr(P, EV_O, t.layer);
    case OP_DOWN: return ev_ctr(P, EV_GU, t.layer, t.idx / P.n_dtiles);
    case OP_LM: return ev_ctr(P, EV_IN, P.n_layers);
    default: return -1;
  }
}

// ---------------------------------------------------------------- producer
struct Copy {
  const unsigned char* src;
  uint32_t dst_off;
  uint32_t bytes;
};

// Fills `cp` with the copies of slot j of a task; returns their count.
__device__ int slot_copies(const DevPlan& P, const Smem& sm, const LayerPtrs* layers, int op, int layer, int idx,
                           int j, int B, Copy* cp) {
  const int H = P.hidden, D = P.head_dim;
  const int rps = P.slot_bytes / (2 * H);
  switch (op) {
    case OP_QKV: {
      QkvTile q = decode_qkv(P, idx);
      const LayerPtrs& lp = layers[layer];
      const unsigned char* w =
          (const unsigned char*)(q.kind == 0 ? lp.wq : (q.kind == 1 ? lp.wk : lp.wv)) + (size_t)q.head * D * H * 2;
      int half_slots = (P.tile_qkv / 2) / rps;
      int part = j / half_slots, js = j % half_slots;
      int row = q.j0 + part * (D / 2) + js * rps;
      cp[0] = {w + (size_t)row * H * 2, 0, (uint32_t)(rps * H * 2)};
      return 1;
    }
    case OP_OPROJ: {
      const unsigned char* w = (const unsigned char*)layers[layer].wo;
      int row = idx * P.tile_o + j * rps;
      cp[0] = {w + (size_t)row * H * 2, 0, (uint32_t)(rps * H * 2)};
      return 1;
    }
    case OP_GATEUP: {
      int half_slots = P.tile_gu / rps;
      int part = j / half_slots, js = j % half_slots;
      const unsigned char* w = (const unsigned char*)(part == 0 ? layers[layer].w_gate : layers[layer].w_up);
      int row = idx * P.tile_gu + js * rps;
      cp[0] = {w + (size_t)row * H * 2, 0, (uint32_t)(rps * H * 2)};
      return 1;
    }
    case OP_DOWN: {
      int kc = idx / P.n_dtiles, n = idx % P.n_dtiles;
      int rpsk = P.slot_bytes / (2 * P.kseg);
      const unsigned char* w = (const unsigned char*)layers[layer].w_down;
      for (int r = 0; r < rpsk; ++r) {
        int row = n * P.tile_down + j * rpsk + r;
        cp[r] = {w + ((size_t)row * P.ffn + (size_t)kc * P.kseg) * 2, (uint32_t)(r * P.kseg * 2),
                 (uint32_t)(P.kseg * 2)};
      }
      return rpsk;
    }
    case OP_LM: {
      int r0 = idx * P.tile_lm + j * rps;
      int rows = min(rps, P.vocab - r0);
      if (rows <= 0) return 0;
      cp[0] = {(const unsigned char*)P.lm_head + (size_t)r0 * H * 2, 0, (uint32_t)(rows * H * 2)};
      return 1;
    }
    case OP_ATTN: {
      AttnTask a = decode_attn(idx, B, P.n_kv_heads, sm.nch, sm.pre);
      int p = sm.ctx[a.b];
      int n_old = min(P.chunk, p - a.c * P.chunk);
      if (n_old <= 0) return 0;
      size_t row0 = (((size_t)layer * P.n_slots + sm.slot[a.b]) * P.n_kv_heads + a.g) * P.max_ctx + (size_t)a.c * P.chunk;
      cp[0] = {(const unsigned char*)P.k_cache + row0 * D * 2, 0, (uint32_t)(n_old * D * 2)};
      cp[1] = {(const unsigned char*)P.v_cache + row0 * D * 2, (uint32_t)(P.chunk * D * 2), (uint32_t)(n_old * D * 2)};
      return 2;
    }
    default: return 0;
  }
}

__device__ int task_slots(const DevPlan& P, int op, int idx) {
  const int rps = P.slot_bytes / (2 * P.hidden);
  switch (op) {
    case OP_QKV: return P.tile_qkv / rps;
    case OP_OPROJ: return P.tile_o / rps;
    case OP_GATEUP: return 2 * P.tile_gu / rps;
    case OP_DOWN: return P.tile_down / (P.slot_bytes / (2 * P.kseg));
    case OP_LM: return ceil_div(min(P.tile_lm, P.vocab - idx * P.tile_lm), rps);
    case OP_ATTN: return 1;
    default: return 0;
  }
}

__device__ void producer(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring,
                         unsigned char* ws, Control* ctl) {
  const FamilyDesc* fams = reinterpret_cast<const FamilyDesc*>(ws + P.off_families);
  const LayerPtrs* layers = reinterpret_cast<const LayerPtrs*>(ws + P.off_layers);
  const long long tmo = P.spin_timeout_ns;
  uint32_t ring_seq = 0, fifo_seq = 0;
  int emitted = 0;
  int qr = 0;  // dynamic queue: range cursor of this CTA
  QRange* Q = reinterpret_cast<QRange*>(ws + P.off_queue);
  bool ok = true;

  auto emit = [&](int fam, int idx) -> bool {
    TaskDesc d;
    d.fam = fam;
    d.idx = idx;
    d.op = fam >= 0 ? fams[fam].op : OP_END;
    d.layer = fam >= 0 ? fams[fam].layer : -1;
    d.nslots = fam >= 0 ? task_slots(P, d.op, idx) : 0;
    d.ring_seq = (int)ring_seq;
    d.pad0 = d.pad1 = 0;
    int k = fifo_seq % kFifo;
    if (!wait_mbar(&sm.fifo_empty[k], ((fifo_seq / kFifo) & 1) ^ 1, ctl, tmo, fam, idx)) return false;
    sm.fifo[k] = d;
    mbar_arrive(&sm.fifo_full[k]);
    fifo_seq++;
    Copy cp[8];
    for (int j = 0; j < d.nslots; ++j) {
      int s = ring_seq % P.ring_slots;
      if (!wait_mbar(&sm.empty[s], ((ring_seq / P.ring_slots) & 1) ^ 1, ctl, tmo, fam, idx)) return false;
      int n = slot_copies(P, sm, layers, d.op, d.layer, idx, j, S.B, cp);
      uint32_t bytes = 0;
      for (int c = 0; c < n; ++c) bytes += cp[c].bytes;
      mbar_arrive_expect_tx(&sm.full[s], bytes);
      unsigned char* dst = ring + (size_t)s * P.slot_bytes;
      for (int c = 0; c < n; ++c) bulk_g2s(dst + cp[c].dst_off, cp[c].src, cp[c].bytes, &sm.full[s]);
      ring_seq++;
    }
    emitted++;
    return true;
  };

  if (P.sched == MK_SCHED_STATIC) {
    const Instr* ins = reinterpret_cast<const Instr*>(ws + P.off_instr) + (size_t)blockIdx.x * P.n_instr_per_sm;
    for (int k = 0; k < P.n_instr_per_sm && ok; ++k) {
      Instr in = ins[k];
      if (in.family < 0) break;
      int ext = sm.fam_ext[in.family];
      for (int i = in.start; i < ext && ok; i += in.stride) ok = emit(in.family, i);
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

// ---------------------------------------------------------------- controller
struct CtlState {
  int nf;
};

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

// notify() of a finished task: decrement its counter; the notifier whose
// decrement reaches zero queues the follow-up and (dynamic) pushes consumers.
// Runs on lane 0 of the controller warp; returns the number of follow-ups.
__device__ int notify_task(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws, Control* ctl,
                           int* counters, const TaskDesc& t, int nf) {
  const int B = S.B, Hkv = P.n_kv_heads;
  const bool dyn = P.sched == MK_SCHED_DYNAMIC;
  int ctr = -1, ffam = -1, fidx = 0;
  int ag = 0, akc = 0;
  switch (t.op) {
    case OP_QKV: ag = decode_qkv(P, t.idx).group; ctr = ev_ctr(P, EV_QKV, t.layer, ag); break;
    case OP_ATTN: {
      AttnTask a = decode_attn(t.idx, B, Hkv, sm.nch, sm.pre);
      ctr = ev_ctr(P, EV_CHUNK, t.layer, a.b, a.g);
      ffam = fam_of(P, OP_MERGE, t.layer);
      fidx = a.b * Hkv + a.g;
    } break;
    case OP_MERGE: ctr = ev_ctr(P, EV_ATTN, t.layer); break;
    case OP_OPROJ: ctr = ev_ctr(P, EV_O, t.layer); break;
    case OP_GATEUP: akc = t.idx * P.tile_gu / P.kseg; ctr = ev_ctr(P, EV_GU, t.layer, akc); break;
    case OP_DOWN: {
      int n = t.idx % P.n_dtiles;
      ctr = ev_ctr(P, EV_DSUM, t.layer, n);
      ffam = fam_of(P, OP_DRED, t.layer);
      fidx = n;
    } break;
    case OP_DRED: ctr = ev_ctr(P, EV_IN, t.layer + 1); break;
    case OP_LM: {
      int grp = t.idx / P.lm_group;
      ctr = ev_ctr(P, EV_LMG, grp);
      ffam = fam_of(P, OP_LMGRP, -1);
      fidx = grp;
    } break;
    case OP_LMGRP: ctr = ev_ctr(P, EV_LM, 0); ffam = fam_of(P, OP_LMFIN, -1); fidx = 0; break;
    case OP_LMFIN:
      if (dyn) push_range(P, S, ctl, ws, -1, 0, P.n_sm);  // one END per CTA
      return nf;
    default: return nf;
  }
  __threadfence();
  int old = atom_add_acq_rel(&counters[ctr], -1);
  if (old <= 0) { record_error(ctl, MK_ERR_DEVICE_BOUNDS, t.fam, t.idx, ctr); return nf; }
  if (old != 1) return nf;
  // the event fired
  if (ffam >= 0 && nf < kMaxFollow) {
    TaskDesc f;
    f.fam = ffam; f.op = (t.op == OP_ATTN) ? OP_MERGE : (t.op == OP_DOWN) ? OP_DRED : (t.op == OP_LM) ? OP_LMGRP : OP_LMFIN;
    f.layer = (f.op == OP_LMGRP || f.op == OP_LMFIN) ? -1 : t.layer;
    f.idx = fidx; f.ring_seq = 0; f.nslots = 0; f.pad0 = f.pad1 = 0;
    sm.follow[nf++] = f;
  }
  if (dyn) {
    switch (t.op) {
      case OP_QKV:
        for (int b = 0; b < B; ++b)
          push_range(P, S, ctl, ws, fam_of(P, OP_ATTN, t.layer), Hkv * sm.pre[b] + ag * sm.nch[b], sm.nch[b]);
        break;
      case OP_MERGE: push_range(P, S, ctl, ws, fam_of(P, OP_OPROJ, t.layer), 0, P.n_otiles); break;
      case OP_OPROJ: push_range(P, S, ctl, ws, fam_of(P, OP_GATEUP, t.layer), 0, P.n_gutiles); break;
      case OP_GATEUP: push_range(P, S, ctl, ws, fam_of(P, OP_DOWN, t.layer), akc * P.n_dtiles, P.n_dtiles); break;
      case OP_DRED:
        if (t.layer + 1 < P.n_layers) push_range(P, S, ctl, ws, fam_of(P, OP_QKV, t.layer + 1), 0, P.n_qkv_tiles);
        else push_range(P, S, ctl, ws, fam_of(P, OP_LM, -1), 0, P.n_lm_tiles);
        break;
      default: break;
    }
  }
  return nf;
}

__device__ void controller(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws, Control* ctl,
                           int* counters) {
  const int lane = threadIdx.x & 31;
  const long long tmo = P.spin_timeout_ns;
  const FamilyDesc* fams = reinterpret_cast<const FamilyDesc*>(ws + P.off_families);
  uint32_t fifo_seq = 0;
  TaskDesc p, held, t;
  bool have_p = false, have_held = false;
  int nf = 0;
  int known = -1;
  int released = 0;
  bool dead = false;

  auto finish_p = [&]() {
    bar_sync(BAR_DONE, kCtlThreads);
    int r = 0;
    if (lane == 0) r = notify_task(P, S, sm, ws, ctl, counters, p, nf);
    nf = __shfl_sync(0xffffffffu, r, 0);
    __syncwarp();
    have_p = false;
  };

  for (;;) {
    if (nf > 0) {
      t = sm.follow[nf - 1];
      nf--;
    } else if (have_held) {
      t = held;
      have_held = false;
    } else {
      int k = fifo_seq % kFifo;
      if (have_p) {
        // never block on the FIFO while holding an un-notified task: its
        // notify may be what the producer's next task (or pop) waits for
        int ready = 0;
        if (lane == 0) ready = mbar_test(&sm.fifo_full[k], (fifo_seq / kFifo) & 1);
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) {
          finish_p();
          if (nf > 0) continue;
        }
      }
      int okw = 1;
      if (lane == 0) okw = wait_mbar(&sm.fifo_full[k], (fifo_seq / kFifo) & 1, ctl, tmo, -1, -1);
      okw = __shfl_sync(0xffffffffu, okw, 0);
      __syncwarp();
      if (!okw) { dead = true; break; }
      t = sm.fifo[k];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.fifo_empty[k]);
      fifo_seq++;
    }
    if (t.op == OP_END) {
      if (have_p) {
        finish_p();
        if (nf > 0) { held = t; have_held = true; continue; }
      }
    } else if (!is_followup(t.op)) {
      int w = wait_counter(P, sm, t, S.B);
      if (w >= 0 && w != known) {
        int zero = 0;
        if (lane == 0) zero = ld_acquire(&counters[w]) == 0;
        zero = __shfl_sync(0xffffffffu, zero, 0);
        if (!zero && have_p) {
          // never spin while holding an un-notified task
          finish_p();
          if (nf > 0) { held = t; have_held = true; continue; }
        }
        if (!zero) {
          int okw = 1;
          if (lane == 0) {
            unsigned long long t0 = global_ns();
            for (int it = 0;; ++it) {
              if (ld_acquire(&counters[w]) == 0) break;
              if ((it & 15) == 15) {
                if (aborted(ctl)) { okw = 0; break; }
                if ((long long)(global_ns() - t0) > tmo) {
                  record_error(ctl, MK_ERR_DEVICE_TIMEOUT, t.fam, t.idx, w);
                  okw = 0;
                  break;
                }
              }
            }
          }
          okw = __shfl_sync(0xffffffffu, okw, 0);
          if (!okw) { dead = true; break; }
        }
        known = w;
      }
    }
    if (have_p) bar_sync(BAR_DONE, kCtlThreads);
    if (lane == 0) {
      sm.cur = t;
      if (t.op != OP_END && S.task_counts && (P.debug_flags & MK_DEBUG_TASK_COUNTS))
        atomicAdd(&S.task_counts[fams[t.fam].debug_base + t.idx], 1u);
      if (t.op != OP_END && !is_followup(t.op)) sm.released = ++released;
    }
    __syncwarp();
    bar_sync(BAR_GO, kCtlThreads);
    if (have_p) {
      int r = 0;
      if (lane == 0) r = notify_task(P, S, sm, ws, ctl, counters, p, nf);
      nf = __shfl_sync(0xffffffffu, r, 0);
      __syncwarp();
    }
    if (t.op == OP_END) break;
    p = t;
    have_p = true;
  }
  if (dead) {
    // shut the compute warps down: finish the task they hold, then send END
    if (have_p) bar_sync(BAR_DONE, kCtlThreads);
    if (lane == 0) {
      TaskDesc e;
      e.fam = -1; e.op = OP_END; e.layer = -1; e.idx = 0; e.ring_seq = 0; e.nslots = 0; e.pad0 = e.pad1 = 0;
      sm.cur = e;
      sm.released = 1 << 30;
    }
    __syncwarp();
    bar_sync(BAR_GO, kCtlThreads);
  }
}

// ---------------------------------------------------------------- compute
struct Act {
  int tag;
  float v[kMaxB][8];
};

// Loads the activation columns this thread owns (8 per row, block cb) for the
// B rows; kind 0: RMSNorm(x) * gamma, 1: attention output, 2: SwiGLU segment.
__device__ void load_act(const DevPlan& P, Smem& sm, unsigned char* ws, int B, int kind, const void* gamma,
                         int kc, int K, Act& a) {
  const int ct = threadIdx.x - 64, cw = ct >> 5, lane = ct & 31;
  const int kb = K / 8, cb = ct % kb;
  const float* src;
  size_t rstride;
  if (kind == 0) { src = reinterpret_cast<const float*>(ws + P.off_x); rstride = P.hidden; }
  else if (kind == 1) { src = reinterpret_cast<const float*>(ws + P.off_attn); rstride = (size_t)P.n_q_heads * P.head_dim; }
  else { src = reinterpret_cast<const float*>(ws + P.off_h) + (size_t)kc * P.kseg; rstride = P.ffn; }
#pragma unroll
  for (int b = 0; b < kMaxB; ++b) {
    if (b < B) {
      const float4* p4 = reinterpret_cast<const float4*>(src + b * rstride + cb * 8);
      float4 u = __ldcg(p4), w = __ldcg(p4 + 1);
      a.v[b][0] = u.x; a.v[b][1] = u.y; a.v[b][2] = u.z; a.v[b][3] = u.w;
      a.v[b][4] = w.x; a.v[b][5] = w.y; a.v[b][6] = w.z; a.v[b][7] = w.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) a.v[b][j] = 0.f;
    }
  }
  if (kind != 0) return;
  // RMSNorm: sum of squares over the K columns of each row
  const int wpg = kb / 32;  // warps per row group
#pragma unroll
  for (int b = 0; b < kMaxB; ++b) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(a.v[b][j], a.v[b][j], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) sm.red[cw][b] = ss;
  }
  bar_sync(BAR_COMP, kComputeThreads);
  const int g0 = (cw / wpg) * wpg;
  uint4 gw = __ldg(reinterpret_cast<const uint4*>(gamma) + cb);
  float gf[8];
  bf16x8_to_f32(gw, gf);
#pragma unroll
  for (int b = 0; b < kMaxB; ++b) {
    float ss = 0.f;
    for (int w = 0; w < wpg; ++w) ss += sm.red[g0 + w][b];
    float inv = 1.0f / sqrtf(ss / (float)K + P.eps);
#pragma unroll
    for (int j = 0; j < 8; ++j) a.v[b][j] = a.v[b][j] * inv * gf[j];
  }
  bar_sync(BAR_COMP, kComputeThreads);
}

// GEMV over a task's ring slots: rows of K bf16 weights, 4 rows per thread per
// slot; leaves sm.fin[row * kMaxB + b] = sum_k W[row][k] * act[b][k].
__device__ bool gemv_rows(const DevPlan& P, Smem& sm, unsigned char* ring, Control* ctl, const TaskDesc& d, int K,
                          int valid_rows, int B, const Act& a) {
  const int ct = threadIdx.x - 64, cw = ct >> 5, lane = ct & 31;
  const int kb = K / 8, G = kComputeThreads / kb, cb = ct % kb, rg = ct / kb;
  const int rps = 4 * G;  // rows per 16 KB slot
  float acc[kAccRows][kMaxB];
#pragma unroll
  for (int k = 0; k < kAccRows; ++k)
#pragma unroll
    for (int b = 0; b < kMaxB; ++b) acc[k][b] = 0.f;
  bool ok = true;
#pragma unroll
  for (int s = 0; s < kAccRows / 4; ++s) {
    if (s < d.nslots) {
      uint32_t seq = (uint32_t)d.ring_seq + s;
      int slot = seq % P.ring_slots;
      if (!wait_mbar(&sm.full[slot], (seq / P.ring_slots) & 1, ctl, P.spin_timeout_ns, d.fam, d.idx)) ok = false;
      const unsigned char* base = ring + (size_t)slot * P.slot_bytes;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        int rl = rg + rr * G;
        if (s * rps + rl < valid_rows) {
          uint4 w = *reinterpret_cast<const uint4*>(base + (size_t)rl * K * 2 + cb * 16);
          float wf[8];
          bf16x8_to_f32(w, wf);
#pragma unroll
          for (int b = 0; b < kMaxB; ++b) {
            float t = acc[s * 4 + rr][b];
#pragma unroll
            for (int j = 0; j < 8; ++j) t = fmaf(wf[j], a.v[b][j], t);
            acc[s * 4 + rr][b] = t;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
  }
  // reduce each (row, b) over the K/8 threads of the row group
#pragma unroll
  for (int k = 0; k < kAccRows; ++k) {
    if (k < 4 * d.nslots) {
#pragma unroll
      for (int b = 0; b < kMaxB; ++b) {
        if (b < B) {
          float v = acc[k][b];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) sm.red[cw][k * kMaxB + b] = v;
        }
      }
    }
  }
  bar_sync(BAR_COMP, kComputeThreads);
  const int wpg = kb / 32;
  const int rows = d.nslots * rps;
  for (int e = ct; e < rows * kMaxB; e += kComputeThreads) {
    int row = e / kMaxB, b = e % kMaxB;
    if (b >= B) continue;
    int s = row / rps, rl = row % rps;
    int g = rl % G, rr = rl / G;
    int k = s * 4 + rr;
    float v = 0.f;
    for (int w = 0; w < wpg; ++w) v += sm.red[g * wpg + w][k * kMaxB + b];
    sm.fin[row * kMaxB + b] = v;
  }
  bar_sync(BAR_COMP, kComputeThreads);
  return ok;
}

__device__ void task_attn(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring, unsigned char* ws,
                          Control* ctl, const TaskDesc& d) {
  const int ct = threadIdx.x - 64, cw = ct >> 5, lane = ct & 31;
  const int Hkv = P.n_kv_heads, qpg = P.n_q_heads / Hkv, D = P.head_dim, CH = P.chunk;
  AttnTask a = decode_attn(d.idx, S.B, Hkv, sm.nch, sm.pre);
  const int p = sm.ctx[a.b];
  const int n_old = max(0, min(CH, p - a.c * CH));
  const bool has_new = (p - a.c * CH) < CH;
  const int n_keys = n_old + (has_new ? 1 : 0);
  const float* q = reinterpret_cast<const float*>(ws + P.off_q) + (size_t)a.b * P.n_q_heads * D + (size_t)a.g * qpg * D;
  if (ct < qpg * D) sm.qs[ct] = __ldcg(q + ct) * 0.125f;  // 1/sqrt(64)
  if (has_new && ct < 2 * D) {
    size_t row = (((size_t)d.layer * P.n_slots + sm.slot[a.b]) * Hkv + a.g) * P.max_ctx + p;
    const unsigned short* src =
        reinterpret_cast<const unsigned short*>(ct < D ? P.k_cache : P.v_cache) + row * D + (ct % D);
    float v = bf16_bits_to_f32(__ldcg(src));
    if (ct < D) sm.newk[ct] = v; else sm.newv[ct - D] = v;
  }
  bar_sync(BAR_COMP, kComputeThreads);
  uint32_t seq = (uint32_t)d.ring_seq;
  int slot = seq % P.ring_slots;
  wait_mbar(&sm.full[slot], (seq / P.ring_slots) & 1, ctl, P.spin_timeout_ns, d.fam, d.idx);
  const unsigned char* kbase = ring + (size_t)slot * P.slot_bytes;
  const unsigned char* vbase = kbase + (size_t)CH * D * 2;
  // scores: thread -> (key kk, head h)
  {
    int kk = ct >> 2, h = ct & 3;
    if (h < qpg) {
      float s = -INFINITY;
      if (kk < n_old) {
        s = 0.f;
        const uint4* kr = reinterpret_cast<const uint4*>(kbase + (size_t)kk * D * 2);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          int ci = (i + kk) & 7;  // rotate the start so the warp's rows hit distinct banks
          float kf[8];
          bf16x8_to_f32(kr[ci], kf);
#pragma unroll
          for (int j = 0; j < 8; ++j) s = fmaf(kf[j], sm.qs[h * D + ci * 8 + j], s);
        }
      } else if (kk < n_keys) {
        s = 0.f;
        for (int j = 0; j < D; ++j) s = fmaf(sm.newk[j], sm.qs[h * D + j], s);
      }
      sm.sc[h][kk] = s;
    }
  }
  bar_sync(BAR_COMP, kComputeThreads);
  if (cw < qpg) {
    float v0 = sm.sc[cw][lane], v1 = sm.sc[cw][lane + 32];
    float m = fmaxf(v0, v1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float e0 = lane < n_keys ? expf(v0 - m) : 0.f;
    float e1 = lane + 32 < n_keys ? expf(v1 - m) : 0.f;
    float l = e0 + e1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    sm.sc[cw][lane] = e0;
    sm.sc[cw][lane + 32] = e1;
    if (lane == 0) { sm.hm[cw] = m; sm.hl[cw] = l; }
  }
  bar_sync(BAR_COMP, kComputeThreads);
  {
    int h = ct >> 6, dd = ct & 63;
    if (h < qpg) {
      float o = 0.f;
      for (int kk = 0; kk < n_old; ++kk) {
        unsigned short vb = *reinterpret_cast<const unsigned short*>(vbase + (size_t)kk * D * 2 + dd * 2);
        o = fmaf(sm.sc[h][kk], bf16_bits_to_f32(vb), o);
      }
      if (has_new) o = fmaf(sm.sc[h][n_old], sm.newv[dd], o);
      float* part = reinterpret_cast<float*>(ws + P.off_apart) +
                    (((size_t)a.b * Hkv + a.g) * P.max_chunks + a.c) * (size_t)(qpg * (D + 2));
      part[h * (D + 2) + dd] = o;
      if (dd == 0) { part[h * (D + 2) + D] = sm.hm[h]; part[h * (D + 2) + D + 1] = sm.hl[h]; }
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&sm.empty[slot]);
}

__device__ void task_merge(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ws, const TaskDesc& d) {
  const int ct = threadIdx.x - 64;
  const int Hkv = P.n_kv_heads, qpg = P.n_q_heads / Hkv, D = P.head_dim;
  const int b = d.idx / Hkv, g = d.idx % Hkv;
  const int nch = sm.nch[b];
  int h = ct >> 6, dd = ct & 63;
  if (h >= qpg) return;
  const float* part = reinterpret_cast<const float*>(ws + P.off_apart) +
                      ((size_t)b * Hkv + g) * P.max_chunks * (size_t)(qpg * (D + 2)) + h * (D + 2);
  const size_t cs = (size_t)qpg * (D + 2);
  float M = -INFINITY;
  for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(part + c * cs + D));
  float L = 0.f, O = 0.f;
  for (int c = 0; c < nch; ++c) {
    float w = expf(__ldcg(part + c * cs + D) - M);
    L = fmaf(__ldcg(part + c * cs + D + 1), w, L);
    O = fmaf(__ldcg(part + c * cs + dd), w, O);
  }
  float* out = reinterpret_cast<float*>(ws + P.off_attn) + (size_t)b * P.n_q_heads * D + (size_t)(g * qpg + h) * D;
  out[dd] = O / L;
}

__device__ void compute(const DevPlan& P, const StepParams& S, Smem& sm, unsigned char* ring, unsigned char* ws,
                        Control* ctl) {
  const int ct = threadIdx.x - 64, cw = ct >> 5, lane = ct & 31;
  const LayerPtrs* layers = reinterpret_cast<const LayerPtrs*>(ws + P.off_layers);
  const int B = S.B, H = P.hidden;
  float* x = reinterpret_cast<float*>(ws + P.off_x);
  Act a;
  a.tag = -1;
  for (;;) {
    bar_sync(BAR_GO, kCtlThreads);
    const TaskDesc d = sm.cur;
    if (d.op == OP_END) break;
    switch (d.op) {
      case OP_QKV: {
        int tag = d.layer * 64 + 0;
        if (a.tag != tag) { load_act(P, sm, ws, B, 0, layers[d.layer].attn_norm, 0, H, a); a.tag = tag; }
        gemv_rows(P, sm, ring, ctl, d, H, P.tile_qkv, B, a);
        QkvTile q = decode_qkv(P, d.idx);
        int half = P.tile_qkv / 2;
        for (int e = ct; e < half * kMaxB; e += kComputeThreads) {
          int jj = e / kMaxB, b = e % kMaxB;
          if (b >= B) continue;
          int j = q.j0 + jj;
          float x0 = sm.fin[jj * kMaxB + b], x1 = sm.fin[(half + jj) * kMaxB + b];
          int pos = sm.ctx[b];
          if (q.kind == 2) {
            size_t row = (((size_t)d.layer * P.n_slots + sm.slot[b]) * P.n_kv_heads + q.head) * P.max_ctx + pos;
            __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(P.v_cache) + row * P.head_dim;
            vc[j] = __float2bfloat16_rn(x0);
            vc[j + 32] = __float2bfloat16_rn(x1);
          } else {
            const float* rope = reinterpret_cast<const float*>(ws + P.off_rope) + ((size_t)pos * 32 + j) * 2;
            float c = __ldg(rope), s = __ldg(rope + 1);
            float y0 = x0 * c - x1 * s, y1 = x1 * c + x0 * s;
            if (q.kind == 0) {
              float* qb = reinterpret_cast<float*>(ws + P.off_q) + (size_t)b * P.n_q_heads * P.head_dim + q.head * P.head_dim;
              qb[j] = y0;
              qb[j + 32] = y1;
            } else {
              size_t row = (((size_t)d.layer * P.n_slots + sm.slot[b]) * P.n_kv_heads + q.head) * P.max_ctx + pos;
              __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(P.k_cache) + row * P.head_dim;
              kc[j] = __float2bfloat16_rn(y0);
              kc[j + 32] = __float2bfloat16_rn(y1);
            }
          }
        }
      } break;
      case OP_ATTN: task_attn(P, S, sm, ring, ws, ctl, d); break;
      case OP_MERGE: task_merge(P, S, sm, ws, d); break;
      case OP_OPROJ: {
        int tag = d.layer * 64 + 1;
        if (a.tag != tag) { load_act(P, sm, ws, B, 1, nullptr, 0, H, a); a.tag = tag; }
        gemv_rows(P, sm, ring, ctl, d, H, P.tile_o, B, a);
        for (int e = ct; e < P.tile_o * kMaxB; e += kComputeThreads) {
          int r = e / kMaxB, b = e % kMaxB;
          if (b >= B) continue;
          float* xp = x + (size_t)b * H + d.idx * P.tile_o + r;
          *xp = __ldcg(xp) + sm.fin[r * kMaxB + b];
        }
      } break;
      case OP_GATEUP: {
        int tag = d.layer * 64 + 2;
        if (a.tag != tag) { load_act(P, sm, ws, B, 0, layers[d.layer].ffn_norm, 0, H, a); a.tag = tag; }
        gemv_rows(P, sm, ring, ctl, d, H, 2 * P.tile_gu, B, a);
        float* h = reinterpret_cast<float*>(ws + P.off_h);
        for (int e = ct; e < P.tile_gu * kMaxB; e += kComputeThreads) {
          int r = e / kMaxB, b = e % kMaxB;
          if (b >= B) continue;
          float g = sm.fin[r * kMaxB + b], u = sm.fin[(P.tile_gu + r) * kMaxB + b];
          h[(size_t)b * P.ffn + d.idx * P.tile_gu + r] = g / (1.0f + expf(-g)) * u;
        }
      } break;
      case OP_DOWN: {
        int kc = d.idx / P.n_dtiles, n = d.idx % P.n_dtiles;
        int tag = d.layer * 64 + 8 + kc;
        if (a.tag != tag) { load_act(P, sm, ws, B, 2, nullptr, kc, P.kseg, a); a.tag = tag; }
        gemv_rows(P, sm, ring, ctl, d, P.kseg, P.tile_down, B, a);
        float* part = reinterpret_cast<float*>(ws + P.off_dpart);
        for (int e = ct; e < P.tile_down * kMaxB; e += kComputeThreads) {
          int r = e / kMaxB, b = e % kMaxB;
          if (b >= B) continue;
          part[((size_t)kc * P.max_batch + b) * H + n * P.tile_down + r] = sm.fin[r * kMaxB + b];
        }
      } break;
      case OP_DRED: {
        const float* part = reinterpret_cast<const float*>(ws + P.off_dpart);
        for (int e = ct; e < P.tile_down * kMaxB; e += kComputeThreads) {
          int r = e / kMaxB, b = e % kMaxB;
          if (b >= B) continue;
          size_t col = (size_t)d.idx * P.tile_down + r;
          float y = 0.f;
          for (int kc = 0; kc < P.n_kc; ++kc) y += __ldcg(part + ((size_t)kc * P.max_batch + b) * H + col);
          float* xp = x + (size_t)b * H + col;
          *xp = __ldcg(xp) + y;
        }
      } break;
      case OP_LM: {
        int tag = 60 * 64;
        if (a.tag != tag) { load_act(P, sm, ws, B, 0, P.final_norm, 0, H, a); a.tag = tag; }
        int r0 = d.idx * P.tile_lm;
        int vr = min(P.tile_lm, P.vocab - r0);
        gemv_rows(P, sm, ring, ctl, d, H, vr, B, a);
        if (S.logits)
          for (int e = ct; e < vr * kMaxB; e += kComputeThreads) {
            int r = e / kMaxB, b = e % kMaxB;
            if (b < B) S.logits[(size_t)b * P.vocab + r0 + r] = sm.fin[r * kMaxB + b];
          }
        if (cw < B) {
          unsigned long long best = 0;
          for (int r = lane; r < vr; r += 32) {
            unsigned long long k = argmax_key(sm.fin[r * kMaxB + cw], r0 + r);
            best = k > best ? k : best;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            unsigned long long v = __shfl_xor_sync(0xffffffffu, best, o);
            best = v > best ? v : best;
          }
          if (lane == 0)
            reinterpret_cast<unsigned long long*>(ws + P.off_lmpart)[(size_t)cw * P.n_lm_tiles + d.idx] = best;
        }
      } break;
      case OP_LMGRP:
      case OP_LMFIN: {
        if (cw < B) {
          const unsigned long long* src;
          int n;
          if (d.op == OP_LMGRP) {
            int t0 = d.idx * P.lm_group;
            n = min(P.lm_group, P.n_lm_tiles - t0);
            src = reinterpret_cast<const unsigned long long*>(ws + P.off_lmpart) + (size_t)cw * P.n_lm_tiles + t0;
          } else {
            n = P.n_lmgrp;
            src = reinterpret_cast<const unsigned long long*>(ws + P.off_lmgpart) + (size_t)cw * P.n_lmgrp;
          }
          unsigned long long best = 0;
          for (int i = lane; i < n; i += 32) {
            unsigned long long k = __ldcg(src + i);
            best = k > best ? k : best;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            unsigned long long v = __shfl_xor_sync(0xffffffffu, best, o);
            best = v > best ? v : best;
          }
          if (lane == 0) {
            if (d.op == OP_LMGRP)
              reinterpret_cast<unsigned long long*>(ws + P.off_lmgpart)[(size_t)cw * P.n_lmgrp + d.idx] = best;
            else
              S.next_tokens[cw] = argmax_key_index(best);
          }
        }
      } break;
      default: break;
    }
    bar_arrive(BAR_DONE, kCtlThreads);
  }
}

// ---------------------------------------------------------------- kernel
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
  if (tid == 0) { sm.bad = (B < 1 || B > P.max_batch || B > kMaxB) ? 1 : 0; sm.released = 0; }
  __syncthreads();
  if (!sm.bad && tid < B) {
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
    int run = 0;
    for (int b = 0; b < B; ++b) {
      sm.pre[b] = run;
      sm.nch[b] = ceil_div(sm.ctx[b] + 1, P.chunk);
      run += sm.nch[b];
    }
    sm.pre[B] = run;
  }
  __syncthreads();
  for (int f = tid; f < P.n_families; f += blockDim.x) {
    ExprEnv env{B, sm.ctx, {0, 0, 0}};
    sm.fam_ext[f] = expr_eval(code, fams[f].extent_expr, env);
  }
  const int gtid = blockIdx.x * blockDim.x + tid, gthreads = gridDim.x * blockDim.x;
  for (int i = gtid; i < P.n_counters; i += gthreads) {
    int e = 0;
    while (e + 1 < EV_COUNT && i >= P.ev[e + 1].base) ++e;
    int lin = i - P.ev[e].base;
    ExprEnv env{B, sm.ctx, {0, 0, 0}};
    for (int dd = P.ev[e].ndim - 1; dd >= 0; --dd) { env.coord[dd] = lin % P.ev[e].dims[dd]; lin /= P.ev[e].dims[dd]; }
    counters[i] = expr_eval(code, P.ev[e].count_expr, env);
  }
  {
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
  if (blockIdx.x == 0 && tid == 0 && P.sched == MK_SCHED_DYNAMIC) {
    ctl->q_head = 0;
    ctl->q_tail = 0;
    push_range(P, S, ctl, ws, fam_of(P, OP_QKV, 0), 0, P.n_qkv_tiles);  // EV_IN[0] is armed at zero
  }
  if (tid == 0) {
    for (int s = 0; s < P.ring_slots; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], kComputeWarps); }
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
    if ((tid & 31) == 0) producer(P, S, sm, ring, ws, ctl);
  } else if (warp == 1) {
    controller(P, S, sm, ws, ctl, counters);
  } else {
    compute(P, S, sm, ring, ws, ctl);
  }
}

}  // namespace mk

// ---------------------------------------------------------------- host glue
#include "launch.hpp"

namespace mk {

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

int smem_fixed_bytes() { return (int)((sizeof(Smem) + 1023) / 1024 * 1024); }

mk_status dev_bind(Plan& p, void* ws, size_t bytes, void* stream, const std::vector<unsigned char>& image,
                   std::string& err) {
  cudaStream_t s = (cudaStream_t)stream;
  size_t smem = (size_t)p.dp.ring_slots * p.dp.slot_bytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(megakernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, megakernel, kThreads, smem);
    if (e == cudaSuccess && nb < 1) { err = "megakernel does not fit on an SM"; return MK_ERR_UNSUPPORTED; }
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync((unsigned char*)ws + p.dp.off_families, image.data(), image.size(), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync((unsigned char*)ws + p.dp.off_control, 0, sizeof(Control), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) { err = std::string("bind failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.dp.smem_bytes = (int)smem;
  p.epoch = 0;
  return MK_OK;
}

mk_status dev_launch(Plan& p, const mk_step_args* a, void* stream, std::string& err) {
  StepParams sp;
  sp.B = a->batch;
  sp.tokens = a->token_ids;
  sp.slots = a->slot_ids;
  sp.ctx = a->ctx_lens;
  sp.logits = a->logits;
  sp.next_tokens = a->next_tokens;
  sp.task_counts = a->task_counts;
  sp.epoch = p.epoch + 1;
  unsigned char* ws = (unsigned char*)p.ws;
  DevPlan dp = p.dp;
  void* args[] = {(void*)&dp, (void*)&sp, (void*)&ws};
  cudaError_t e = cudaLaunchCooperativeKernel((const void*)megakernel, dim3(p.dp.n_sm), dim3(kThreads), args,
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
  if (e != cudaSuccess) { err = std::string("reset failed: ") + cudaGetErrorString(e); return MK_ERR_CUDA; }
  p.epoch = 0;
  return MK_OK;
}

}  // namespace mk
