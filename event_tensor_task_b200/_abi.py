"""ctypes mirror of include/mk.h: structs, constants and prototypes.

Argument marshalling only; every step of the decode path runs in libmk.so.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmk.so")

MK_OK = 0
MK_ERR_INVALID_ARG = -1
MK_ERR_UNSUPPORTED = -2
MK_ERR_WORKSPACE = -3
MK_ERR_CUDA = -4
MK_ERR_DEVICE_TIMEOUT = -5
MK_ERR_DEVICE_BOUNDS = -6
MK_ERR_PLAN = -7

MK_SCHED_STATIC = 0
MK_SCHED_DYNAMIC = 1
MK_MODEL_DENSE = 0
MK_DEBUG_TASK_COUNTS = 1
MK_DEBUG_TRACE = 2
MK_DEBUG_EMPTY_TASKS = 4
MK_STATIC_SCRATCH_BYTES = 8 * 1024 * 1024

MK_SIM_FAULT_NONE = 0
MK_SIM_FAULT_DROP_NOTIFY = 1
MK_SIM_FAULT_COUNT_PLUS_ONE = 2
MK_SIM_FAULT_NO_WAIT = 3
MK_SIM_FAULT_COUNT_MINUS_ONE = 4

MK_MODEL_MOE_LAYER = 1
MK_MODEL_MOE_DECODER = 2

OP_NAMES = {1: "qkv", 2: "attn", 3: "merge", 4: "oproj", 5: "gateup", 6: "down", 7: "norm",
            8: "lm", 9: "norm2", 10: "lmfin", 11: "route", 12: "mindptr", 13: "egu", 14: "edown", 15: "combine",
            16: "mfin", 17: "normf"}


class mk_moe_weights(C.Structure):
    _fields_ = [("w_router", C.c_void_p), ("router_bias", C.c_void_p), ("w_gate", C.c_void_p),
                ("w_up", C.c_void_p), ("w_down", C.c_void_p)]


class mk_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")] + [
                    ("moe", mk_moe_weights)]


class mk_model_desc(C.Structure):
    _fields_ = [
        ("kind", C.c_int), ("n_layers", C.c_int), ("hidden", C.c_int), ("n_q_heads", C.c_int),
        ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int), ("vocab", C.c_int),
        ("eps", C.c_float), ("rope_theta", C.c_float), ("max_batch", C.c_int), ("max_ctx", C.c_int),
        ("n_slots", C.c_int), ("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
        ("layers", C.POINTER(mk_layer_weights)), ("k_cache", C.c_void_p), ("v_cache", C.c_void_p),
        ("n_experts", C.c_int), ("top_k", C.c_int), ("expert_ffn", C.c_int), ("max_tokens", C.c_int),
        ("moe", mk_moe_weights),
    ]


class mk_moe_args(C.Structure):
    _fields_ = [
        ("n_tokens", C.c_int), ("x", C.c_void_p), ("out", C.c_void_p), ("topk_idx", C.c_void_p),
        ("topk_w", C.c_void_p), ("hist", C.c_void_p), ("indptr", C.c_void_p), ("logits", C.c_void_p),
        ("task_counts", C.c_void_p),
    ]


class mk_plan_opts(C.Structure):
    _fields_ = [
        ("sched", C.c_int), ("n_sm", C.c_int), ("host_only", C.c_int), ("smem_bytes", C.c_int),
        ("tile_qkv", C.c_int), ("tile_o", C.c_int), ("tile_gu", C.c_int), ("tile_down", C.c_int),
        ("kseg", C.c_int), ("tile_lm", C.c_int), ("attn_chunk", C.c_int),
        ("spin_timeout_ns", C.c_longlong), ("debug_flags", C.c_uint), ("fault", C.c_int),
        ("fault_family", C.c_int), ("attn_split", C.c_int), ("moe_tiles", C.c_int), ("act_split", C.c_int),
    ]


class mk_step_args(C.Structure):
    _fields_ = [
        ("batch", C.c_int), ("token_ids", C.c_void_p), ("slot_ids", C.c_void_p), ("ctx_lens", C.c_void_p),
        ("logits", C.c_void_p), ("next_tokens", C.c_void_p), ("task_counts", C.c_void_p),
        ("trace", C.c_void_p), ("trace_cap", C.c_int),
        ("capture_resid", C.c_void_p), ("capture_moe_in", C.c_void_p), ("capture_topk", C.c_void_p),
        ("capture_hist", C.c_void_p), ("capture_indptr", C.c_void_p),
    ]


class mk_device_status(C.Structure):
    _fields_ = [("code", C.c_int), ("family", C.c_int), ("index", C.c_int), ("event", C.c_int), ("sm", C.c_int)]


class mk_stats(C.Structure):
    _fields_ = [("launches", C.c_longlong), ("build_ms", C.c_double), ("n_families", C.c_int),
                ("n_counters", C.c_int), ("ring_slots", C.c_int), ("n_sm", C.c_int),
                ("workspace_bytes", C.c_longlong), ("queue_ranges_cap", C.c_int), ("last_queue_ranges", C.c_int),
                ("last_queue_tasks", C.c_longlong), ("last_queue_pops", C.c_longlong)]


class mk_family_info(C.Structure):
    _fields_ = [("op", C.c_int), ("layer", C.c_int), ("debug_base", C.c_int), ("max_extent", C.c_int),
                ("followup", C.c_int), ("name", C.c_char * 16)]


class mk_sim_report(C.Structure):
    _fields_ = [("orders_run", C.c_int), ("tasks_per_order", C.c_int), ("races", C.c_int),
                ("deadlocks", C.c_int), ("exactly_once_violations", C.c_int), ("nonzero_counters", C.c_int),
                ("static_dynamic_mismatch", C.c_int), ("first_error", C.c_char * 160)]


# name -> (restype, argtypes); every symbol include/mk.h declares
PROTOTYPES = {
    "mk_last_error": (C.c_char_p, []),
    "mk_plan_build": (C.c_int, [C.POINTER(mk_model_desc), C.POINTER(mk_plan_opts), C.POINTER(C.c_void_p)]),
    "mk_plan_workspace_bytes": (C.c_size_t, [C.c_void_p]),
    "mk_plan_bind_workspace": (C.c_int, [C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "mk_decode_step": (C.c_int, [C.c_void_p, C.POINTER(mk_step_args), C.c_void_p]),
    "mk_decode_step_static": (C.c_int, [C.c_void_p, C.POINTER(mk_step_args), C.c_void_p]),
    "mk_moe_layer": (C.c_int, [C.c_void_p, C.POINTER(mk_moe_args), C.c_void_p]),
    "mk_get_status": (C.c_int, [C.c_void_p, C.POINTER(mk_device_status)]),
    "mk_get_stats": (C.c_int, [C.c_void_p, C.POINTER(mk_stats)]),
    "mk_plan_reset": (C.c_int, [C.c_void_p, C.c_void_p]),
    "mk_plan_task_slots": (C.c_int, [C.c_void_p]),
    "mk_plan_num_families": (C.c_int, [C.c_void_p]),
    "mk_plan_family_info": (C.c_int, [C.c_void_p, C.c_int, C.POINTER(mk_family_info)]),
    "mk_plan_tiles": (C.c_int, [C.c_void_p, C.POINTER(C.c_int)]),
    "mk_plan_counter_region": (C.c_int, [C.c_void_p, C.POINTER(C.c_longlong), C.POINTER(C.c_int)]),
    "mk_plan_validate": (C.c_int, [C.c_void_p, C.c_int, C.POINTER(C.c_int)]),
    "mk_plan_simulate": (C.c_int, [C.c_void_p, C.c_int, C.POINTER(C.c_int), C.c_int, C.c_uint, C.c_int,
                                   C.c_int, C.POINTER(mk_sim_report)]),
    "mk_plan_step_bytes": (C.c_double, [C.c_void_p, C.c_int, C.POINTER(C.c_int), C.c_int]),
    "mk_plan_destroy": (None, [C.c_void_p]),
}


def load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise RuntimeError(
            f"libmk.so not found at {path}: build it with `python -m event_tensor_task_b200.build` "
            "(there is no CPU fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
