"""B200 decode megakernel with Event-Tensor synchronisation — Python binding.

Thin ctypes binding of ``libmk.so`` (C ABI in ``include/mk.h``).  The
functions below carry the C names and only marshal arguments; the decode
step itself runs entirely in the library's CUDA kernel.  PyTorch is used for
device memory and streams only.  There is no CPU fallback: if the library is
missing, importing a function that needs it raises.
"""
from __future__ import annotations

import ctypes as C

from . import _abi
from ._abi import (MK_MODEL_MOE_LAYER, MK_MODEL_MOE_DECODER, mk_moe_weights, mk_moe_args, MK_OK, MK_ERR_INVALID_ARG,
                   MK_ERR_UNSUPPORTED, MK_ERR_WORKSPACE, MK_ERR_CUDA, MK_ERR_DEVICE_TIMEOUT, MK_ERR_DEVICE_BOUNDS,
                   MK_ERR_PLAN, MK_STATIC_SCRATCH_BYTES,
                   MK_SCHED_STATIC, MK_SCHED_DYNAMIC, MK_MODEL_DENSE, MK_DEBUG_TASK_COUNTS, MK_DEBUG_TRACE,
                   MK_DEBUG_EMPTY_TASKS,
                   MK_SIM_FAULT_NONE, MK_SIM_FAULT_DROP_NOTIFY, MK_SIM_FAULT_COUNT_PLUS_ONE,
                   MK_SIM_FAULT_NO_WAIT, MK_SIM_FAULT_COUNT_MINUS_ONE, OP_NAMES, mk_model_desc, mk_plan_opts, mk_step_args,
                   mk_layer_weights, mk_device_status, mk_family_info, mk_sim_report)

_lib = None


class MkError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"mk status {status}: {message}")
        self.status = status
        self.message = message


def lib():
    global _lib
    if _lib is None:
        _lib = _abi.load()
    return _lib


def _check(status: int):
    if status != MK_OK:
        raise MkError(status, lib().mk_last_error().decode(errors="replace"))


def _ints(vals):
    if vals is None:
        return None
    vals = [int(v) for v in vals]
    return (C.c_int * len(vals))(*vals)


# ---------------------------------------------------------------- C ABI, same names
def mk_last_error() -> str:
    return lib().mk_last_error().decode(errors="replace")


def mk_plan_build(desc: mk_model_desc, opts: mk_plan_opts) -> int:
    h = C.c_void_p()
    _check(lib().mk_plan_build(C.byref(desc), C.byref(opts), C.byref(h)))
    return h.value


def mk_plan_workspace_bytes(plan: int) -> int:
    return int(lib().mk_plan_workspace_bytes(plan))


def mk_plan_bind_workspace(plan: int, dev_ptr: int, nbytes: int, stream: int = 0):
    _check(lib().mk_plan_bind_workspace(plan, dev_ptr, nbytes, stream))


def mk_decode_step(plan: int, args: mk_step_args, stream: int = 0):
    _check(lib().mk_decode_step(plan, C.byref(args), stream))


def mk_decode_step_static(plan: int, args: mk_step_args, stream: int = 0):
    _check(lib().mk_decode_step_static(plan, C.byref(args), stream))


def mk_moe_layer(plan: int, args: mk_moe_args, stream: int = 0):
    _check(lib().mk_moe_layer(plan, C.byref(args), stream))


def mk_get_stats(plan: int) -> dict:
    """Plan and runtime counters (mk_get_stats) as a dict."""
    st = _abi.mk_stats()
    _check(lib().mk_get_stats(plan, C.byref(st)))
    return {name: getattr(st, name) for name, _ in st._fields_}


def mk_get_status(plan: int):
    st = mk_device_status()
    code = lib().mk_get_status(plan, C.byref(st))
    return code, st


def mk_plan_reset(plan: int, stream: int = 0):
    _check(lib().mk_plan_reset(plan, stream))


def mk_plan_task_slots(plan: int) -> int:
    return int(lib().mk_plan_task_slots(plan))


def mk_plan_num_families(plan: int) -> int:
    return int(lib().mk_plan_num_families(plan))


def mk_plan_family_info(plan: int, f: int) -> mk_family_info:
    info = mk_family_info()
    _check(lib().mk_plan_family_info(plan, f, C.byref(info)))
    return info


def mk_plan_tiles(plan: int) -> dict:
    out = (C.c_int * 16)()
    _check(lib().mk_plan_tiles(plan, out))
    keys = ("tile_qkv", "tile_o", "tile_gu", "tile_down", "kseg", "tile_lm", "chunk", "n_sm", "ring_slots",
            "attn_split", "wide", "act_split", "gseg_qkv", "gseg_o", "gseg_gu", "attn_auto")
    return dict(zip(keys, list(out)))


def mk_plan_counter_region(plan: int):
    """(byte offset in the workspace, number of int32 counters) of the Event Tensor counters."""
    off, n = C.c_longlong(), C.c_int()
    _check(lib().mk_plan_counter_region(plan, C.byref(off), C.byref(n)))
    return int(off.value), int(n.value)


def mk_plan_validate(plan: int, batch: int, ctx_lens) -> None:
    _check(lib().mk_plan_validate(plan, batch, _ints(ctx_lens)))


def mk_plan_simulate(plan: int, batch: int, ctx_lens, n_orders: int, seed: int = 0,
                     fault: int = MK_SIM_FAULT_NONE, fault_family: int = -1):
    rep = mk_sim_report()
    code = lib().mk_plan_simulate(plan, batch, _ints(ctx_lens), n_orders, seed, fault, fault_family,
                                  C.byref(rep))
    return code, rep


def mk_plan_step_bytes(plan: int, batch: int, ctx_lens, with_logits: bool = False) -> float:
    return float(lib().mk_plan_step_bytes(plan, batch, _ints(ctx_lens), int(with_logits)))


def mk_plan_destroy(plan: int):
    lib().mk_plan_destroy(plan)


# ---------------------------------------------------------------- convenience holder
def _ptr(t):
    return 0 if t is None else int(t.data_ptr())


class DenseDecoder:
    """A plan plus the tensors it points at (kept alive here).

    ``shape`` has the fields n_layers, hidden, n_q_heads, n_kv_heads,
    head_dim, ffn, vocab, eps, rope_theta, tied.  ``weights`` maps the names
    ``embed``, ``final_norm``, ``layers.{l}.{attn_norm,wq,wk,wv,wo,ffn_norm,
    w_gate,w_up,w_down}`` (and ``lm_head`` when untied) to bf16 tensors on the
    device.  ``k_cache``/``v_cache`` are bf16 ``[L][slots][Hkv][max_ctx][64]``.
    With ``host_only`` no GPU is touched (plan validation and simulation only).
    With ``workspace=False`` the plan gets no workspace and steps only through
    ``step(..., static_scratch=True)`` (mk_decode_step_static).
    """

    def __init__(self, shape, weights=None, k_cache=None, v_cache=None, max_batch=1, max_ctx=None,
                 n_slots=None, sched=MK_SCHED_STATIC, n_sm=0, host_only=False, debug=False,
                 spin_timeout_ns=0, trace=False, workspace=True, moe=None, empty_tasks=False, **tiles):
        import torch
        self.shape = shape
        w = weights or {}
        self._keep = [w, k_cache, v_cache]
        L = shape.n_layers
        self._layers = (mk_layer_weights * L)()
        for l in range(L):
            p = f"layers.{l}."
            for f in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down"):
                setattr(self._layers[l], f, _ptr(w.get(p + f)))
        if moe is not None:
            # MoE decoder: moe = (MoEShape, [per-layer dict router/w_gate/w_up/w_down], bias or None)
            mshape, mlayers, mbias = moe
            self._keep.append(moe)
            for l in range(L):
                mw = mlayers[l] if mlayers else {}
                self._layers[l].moe = mk_moe_weights(_ptr(mw.get("router")), _ptr(mbias), _ptr(mw.get("w_gate")),
                                                     _ptr(mw.get("w_up")), _ptr(mw.get("w_down")))
            sched = MK_SCHED_DYNAMIC
        if max_ctx is None:
            max_ctx = k_cache.shape[3]
        if n_slots is None:
            n_slots = k_cache.shape[1] if k_cache is not None else max_batch
        d = mk_model_desc()
        d.kind = MK_MODEL_DENSE if moe is None else MK_MODEL_MOE_DECODER
        if moe is not None:
            d.n_experts, d.top_k, d.expert_ffn = moe[0].n_experts, moe[0].top_k, moe[0].expert_ffn
        d.n_layers, d.hidden, d.n_q_heads, d.n_kv_heads = L, shape.hidden, shape.n_q_heads, shape.n_kv_heads
        d.head_dim, d.ffn, d.vocab = shape.head_dim, shape.ffn, shape.vocab
        d.eps, d.rope_theta = shape.eps, shape.rope_theta
        d.max_batch, d.max_ctx, d.n_slots = max_batch, max_ctx, n_slots
        d.embed = _ptr(w.get("embed"))
        d.lm_head = _ptr(w.get("lm_head")) if not getattr(shape, "tied", True) else 0
        d.final_norm = _ptr(w.get("final_norm"))
        d.layers = self._layers
        d.k_cache, d.v_cache = _ptr(k_cache), _ptr(v_cache)
        o = mk_plan_opts()
        o.sched, o.n_sm, o.host_only = sched, n_sm, int(host_only)
        o.spin_timeout_ns = spin_timeout_ns
        o.debug_flags = ((MK_DEBUG_TASK_COUNTS if debug else 0) | (MK_DEBUG_TRACE if trace else 0) |
                         (MK_DEBUG_EMPTY_TASKS if empty_tasks else 0))
        for k, v in tiles.items():
            setattr(o, k, int(v))
        self.desc, self.opts = d, o
        self.plan = mk_plan_build(d, o)
        self.ws = None
        if not host_only and workspace:
            nbytes = mk_plan_workspace_bytes(self.plan)
            self.ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=k_cache.device)
            base = (_ptr(self.ws) + 255) // 256 * 256
            mk_plan_bind_workspace(self.plan, base, nbytes, torch.cuda.current_stream().cuda_stream)

    def families(self):
        return [mk_plan_family_info(self.plan, f) for f in range(mk_plan_num_families(self.plan))]

    def tiles(self):
        return mk_plan_tiles(self.plan)

    def step(self, token_ids, slot_ids, ctx_lens, next_tokens, logits=None, task_counts=None, stream=None,
             trace=None, static_scratch=False, capture=None):
        """One decode step on ``stream`` (default: torch's current stream);
        through mk_decode_step_static when ``static_scratch``.  ``capture``
        maps ``resid``, ``moe_in``, ``topk``, ``hist``, ``indptr`` to device
        tensors that receive the step's debug captures (mk_step_args)."""
        import torch
        a = mk_step_args()
        if trace is not None:
            a.trace, a.trace_cap = _ptr(trace), int(trace.shape[1])
        if capture:
            a.capture_resid, a.capture_moe_in = _ptr(capture.get("resid")), _ptr(capture.get("moe_in"))
            a.capture_topk, a.capture_hist = _ptr(capture.get("topk")), _ptr(capture.get("hist"))
            a.capture_indptr = _ptr(capture.get("indptr"))
        a.batch = int(token_ids.numel())
        a.token_ids, a.slot_ids, a.ctx_lens = _ptr(token_ids), _ptr(slot_ids), _ptr(ctx_lens)
        a.logits, a.next_tokens, a.task_counts = _ptr(logits), _ptr(next_tokens), _ptr(task_counts)
        s = stream if stream is not None else torch.cuda.current_stream()
        (mk_decode_step_static if static_scratch else mk_decode_step)(self.plan, a, s.cuda_stream)

    def status(self):
        return mk_get_status(self.plan)

    def counters(self):
        """The Event Tensor counters in the bound workspace (int32 tensor on the device)."""
        import torch
        off, n = mk_plan_counter_region(self.plan)
        base = (_ptr(self.ws) + 255) // 256 * 256 - _ptr(self.ws)
        return self.ws[base + off: base + off + 4 * n].view(torch.int32)

    def stats(self):
        return mk_get_stats(self.plan)

    def reset(self):
        import torch
        mk_plan_reset(self.plan, torch.cuda.current_stream().cuda_stream)

    def close(self):
        if self.plan:
            mk_plan_destroy(self.plan)
            self.plan = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class MoELayer:
    """A plan for one mixture-of-experts FFN layer plus the tensors it points at.

    ``weights`` maps ``router`` ([E][H]), ``w_gate``/``w_up`` ([E][F][H]) and
    ``w_down`` ([E][H][F]) to bf16 device tensors; ``bias`` is an fp32 [E]
    device tensor added to the router logits, or None.  The plan runs on the
    dynamic schedule (its task counts follow the routing).
    """

    def __init__(self, shape, weights, bias=None, max_tokens=512, n_sm=0, debug=False, spin_timeout_ns=0,
                 host_only=False, moe_tiles=0):
        import torch
        self.shape = shape
        self._keep = [weights, bias]
        d = mk_model_desc()
        d.kind = MK_MODEL_MOE_LAYER
        d.hidden, d.n_experts, d.top_k, d.expert_ffn = shape.hidden, shape.n_experts, shape.top_k, shape.expert_ffn
        d.max_tokens = max_tokens
        w = weights or {}
        d.moe = mk_moe_weights(_ptr(w.get("router")), _ptr(bias), _ptr(w.get("w_gate")), _ptr(w.get("w_up")),
                               _ptr(w.get("w_down")))
        o = mk_plan_opts()
        o.sched, o.n_sm, o.host_only = MK_SCHED_DYNAMIC, n_sm, int(host_only)
        o.spin_timeout_ns = spin_timeout_ns
        o.debug_flags = MK_DEBUG_TASK_COUNTS if debug else 0
        o.moe_tiles = moe_tiles
        self.desc, self.opts = d, o
        self.plan = mk_plan_build(d, o)
        self.ws = None
        if not host_only:
            nbytes = mk_plan_workspace_bytes(self.plan)
            self.ws = torch.empty(nbytes + 256, dtype=torch.uint8, device="cuda")
            base = (_ptr(self.ws) + 255) // 256 * 256
            mk_plan_bind_workspace(self.plan, base, nbytes, torch.cuda.current_stream().cuda_stream)

    def families(self):
        return [mk_plan_family_info(self.plan, f) for f in range(mk_plan_num_families(self.plan))]

    def __call__(self, x, out, topk_idx=None, topk_w=None, hist=None, indptr=None, logits=None,
                 task_counts=None, stream=None):
        """out = MoE(x) for x, out bf16 [T][H] on the device (one launch)."""
        import torch
        a = mk_moe_args()
        a.n_tokens = int(x.shape[0])
        a.x, a.out = _ptr(x), _ptr(out)
        a.topk_idx, a.topk_w, a.hist, a.indptr = _ptr(topk_idx), _ptr(topk_w), _ptr(hist), _ptr(indptr)
        a.logits, a.task_counts = _ptr(logits), _ptr(task_counts)
        s = stream if stream is not None else torch.cuda.current_stream()
        mk_moe_layer(self.plan, a, s.cuda_stream)

    def status(self):
        return mk_get_status(self.plan)

    def counters(self):
        """The Event Tensor counters in the bound workspace (int32 tensor on the device)."""
        import torch
        off, n = mk_plan_counter_region(self.plan)
        base = (_ptr(self.ws) + 255) // 256 * 256 - _ptr(self.ws)
        return self.ws[base + off: base + off + 4 * n].view(torch.int32)

    def close(self):
        if self.plan:
            mk_plan_destroy(self.plan)
            self.plan = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
