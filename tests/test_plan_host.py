"""Host-only tests of the C ABI and the task-graph compiler (no GPU needed).

The plan simulator is the race detector: it runs the lowered plan in seeded
random interleavings with vector clocks over the regions each task reads and
writes, and checks exactly-once execution, counters at zero, and that static
and dynamic scheduling run the same task set.
"""
import os
import re

import pytest

import event_tensor_task_b200 as mk
import workloads as wl
from oracle import tasks as ot

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_symbol():
    hdr = open(os.path.join(ROOT, "include", "mk.h")).read()
    declared = set(re.findall(r"\b(mk_[a-z_]+)\s*\(", hdr))
    assert declared, "no declarations found"
    lib = mk.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(mk._abi.PROTOTYPES), declared ^ set(mk._abi.PROTOTYPES)


def _host(shape, max_batch=4, max_ctx=320, sched=mk.MK_SCHED_STATIC, n_sm=16, **tiles):
    return mk.DenseDecoder(shape, max_batch=max_batch, max_ctx=max_ctx, n_slots=max_batch, sched=sched,
                           n_sm=n_sm, host_only=True, **tiles)


def test_plan_build_and_tiles():
    d = _host(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_sm=148)
    t = d.tiles()
    assert t["tile_qkv"] == 32 and t["tile_o"] == 32 and t["tile_gu"] == 32 and t["tile_down"] == 64
    assert t["kseg"] == 2048 and t["tile_lm"] == 64 and t["chunk"] == 64 and t["n_sm"] == 148
    fams = d.families()
    assert len(fams) == 16 * 5 + 2
    assert [f.name.decode() for f in fams[:5]] == ["qkv.0", "attn.0", "oproj.0", "gateup.0", "down.0"]
    assert sum(f.followup for f in fams) == 1  # (LMFIN; a pair's last attention task merges the pair)


def test_plan_rejects_oversized_tiles():
    # a GEMV task is at most 64 rows (two halves of up to 32 rows, each over
    # 8 column slices); tiles that are not whole 16-row blocks are refused
    for bad in (dict(tile_gu=64), dict(tile_lm=128), dict(tile_o=64), dict(tile_down=128), dict(tile_o=8),
                dict(tile_down=24), dict(tile_qkv=16), dict(tile_lm=16), dict(tile_gu=8)):
        with pytest.raises(mk.MkError):
            _host(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_sm=148, **bad)
    for ok in (dict(tile_o=16), dict(tile_down=16), dict(tile_down=32), dict(tile_gu=16), dict(tile_lm=32)):
        _host(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_sm=148, **ok).close()


def test_plan_rejects_bad_shapes():
    bad = wl.DenseShape(n_layers=1, hidden=320, n_q_heads=5, n_kv_heads=1, head_dim=64, ffn=1024, vocab=64)
    with pytest.raises(mk.MkError) as e:
        _host(bad)
    assert e.value.status in (mk._abi.MK_ERR_UNSUPPORTED, mk._abi.MK_ERR_INVALID_ARG)
    with pytest.raises(mk.MkError):
        _host(wl.TINY, tile_qkv=24)
    with pytest.raises(mk.MkError):
        _host(wl.TINY, max_batch=65)
    with pytest.raises(mk.MkError):  # the wide-batch path takes no GEMV tile options
        _host(wl.TINY, max_batch=16, tile_o=16)


def test_step_bytes_matches_hand_count():
    d = _host(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_sm=148)
    s = wl.LLAMA_1B
    H, F, D = s.hidden, s.ffn, s.head_dim
    per_layer = ((s.n_q_heads + 2 * s.n_kv_heads) * D * H + H * H + 3 * F * H + 2 * H) * 2
    weights = s.n_layers * per_layer + s.vocab * H * 2 + H * 2
    kv = 1024 * 16 * 8 * 64 * 2 * 2
    want = weights + H * 2 + kv + 16 * 8 * 64 * 2 * 2 + 8
    assert mk.mk_plan_step_bytes(d.plan, 1, [1024]) == pytest.approx(want, rel=1e-12)
    assert abs(want / 1e9 - 2.505) < 0.01  # 2.505 GB per step at B=1, ctx 1024


@pytest.mark.parametrize("B,ctx", [(1, [64]), (2, [0, 130]), (4, [5, 63, 64, 255])])
def test_validate_bindings(B, ctx):
    d = _host(wl.TINY)
    mk.mk_plan_validate(d.plan, B, ctx)


@pytest.mark.parametrize("sched", [mk.MK_SCHED_STATIC, mk.MK_SCHED_DYNAMIC])
@pytest.mark.parametrize("B,ctx", [(1, [64]), (3, [0, 70, 190])])
def test_simulator_clean(sched, B, ctx):
    d = _host(wl.TINY, sched=sched, n_sm=8)
    code, rep = mk.mk_plan_simulate(d.plan, B, ctx, n_orders=60, seed=7)
    assert code == 0, rep.first_error
    assert rep.races == 0 and rep.deadlocks == 0 and rep.exactly_once_violations == 0
    assert rep.nonzero_counters == 0 and rep.static_dynamic_mismatch == 0
    t = d.tiles()
    tiles = {k: t[k] for k in ("tile_qkv", "chunk", "tile_o", "tile_gu", "tile_down", "kseg", "tile_lm")}
    assert tiles == dict(tile_qkv=32, chunk=64, tile_o=32, tile_gu=32, tile_down=64, kseg=1024, tile_lm=64)
    assert t["attn_split"] == 32 and t["attn_auto"] == 1  # the split follows the step, at most 2048 keys
    want = ot.expected_dense_tasks(wl.TINY, B, ctx, dict(tiles, split=32, split_auto=True, n_sm=t["n_sm"]))
    assert rep.tasks_per_order == len(want)


@pytest.mark.parametrize("B,ctx,split", [(1, [1024], 3), (2, [300, 250], 3), (3, [600, 900, 200], 10),
                                         (4, [696, 2450, 2106, 216], 29), (8, [4095] * 8, 32)])
def test_simulator_adaptive_attention_split(B, ctx, split):
    # the lowered plan's tasks for a step (the per-step split evaluated in the
    # plan's expressions and task model) against the oracle's task set, over
    # splits from the floor of 3 to the cap of 32, with multi-task pairs: the
    # 1B shape on 148 SMs at B=1 (T = 99), the tiny shape on 8 SMs (T = 6)
    shape, n_sm = (wl.LLAMA_1B, 148) if B == 1 else (wl.TINY, 8)
    d = _host(shape, max_batch=8, max_ctx=4160, n_sm=n_sm)
    mk.mk_plan_validate(d.plan, B, ctx)
    code, rep = mk.mk_plan_simulate(d.plan, B, ctx, n_orders=1, seed=3)
    assert code == 0 and rep.races == 0 and rep.nonzero_counters == 0, rep.first_error
    t = d.tiles()
    tiles = {k: t[k] for k in ("tile_qkv", "chunk", "tile_o", "tile_gu", "tile_down", "kseg", "tile_lm", "n_sm")}
    assert ot.step_split(shape, B, ctx, dict(tiles, split=t["attn_split"], split_auto=True)) == split
    want = ot.expected_dense_tasks(shape, B, ctx, dict(tiles, split=t["attn_split"], split_auto=True))
    assert rep.tasks_per_order == len(want)
    d.close()


@pytest.mark.parametrize("B,ctx,split", [(4, [600, 900, 200, 50], 10), (9, [600, 900, 200, 50, 0, 1, 2, 3, 4], 24)])
def test_simulator_wide_plan_attention_split(B, ctx, split):
    # a wide-batch plan (max_batch 16) takes the per-step split up to 8 rows
    # and its fixed 24 above: the tiny shape on 8 SMs (T = 6)
    d = _host(wl.TINY, max_batch=16, max_ctx=1024, n_sm=8)
    t = d.tiles()
    assert t["wide"] == 1 and t["attn_auto"] == 1 and t["attn_split"] == 24
    mk.mk_plan_validate(d.plan, B, ctx)
    code, rep = mk.mk_plan_simulate(d.plan, B, ctx, n_orders=1, seed=5)
    assert code == 0 and rep.races == 0 and rep.nonzero_counters == 0, rep.first_error
    tiles = {k: t[k] for k in ("tile_qkv", "chunk", "tile_o", "tile_gu", "tile_down", "kseg", "tile_lm", "n_sm")}
    tiles.update(split=24, split_auto=True, wide=True, gseg=(t["gseg_qkv"], t["gseg_o"], t["gseg_gu"]))
    assert ot.step_split(wl.TINY, B, ctx, tiles) == split
    assert rep.tasks_per_order == len(ot.expected_dense_tasks(wl.TINY, B, ctx, tiles))
    d.close()


def test_simulator_many_orders():
    d = _host(wl.TINY, n_sm=5)
    code, rep = mk.mk_plan_simulate(d.plan, 2, [3, 128], n_orders=1000, seed=11)
    assert code == 0 and rep.orders_run == 1000, rep.first_error


def _family(d, name):
    return [f.name.decode() for f in d.families()].index(name)


def test_fault_dropped_notify_is_detected():
    d = _host(wl.TINY, n_sm=4)
    code, rep = mk.mk_plan_simulate(d.plan, 1, [64], 4, 1, mk.MK_SIM_FAULT_DROP_NOTIFY, _family(d, "gateup.1"))
    assert code != 0 and rep.deadlocks == rep.orders_run


def test_fault_wrong_wait_count_is_detected():
    d = _host(wl.TINY, n_sm=4)
    code, rep = mk.mk_plan_simulate(d.plan, 1, [64], 4, 1, mk.MK_SIM_FAULT_COUNT_PLUS_ONE, _family(d, "qkv.0"))
    assert code != 0 and rep.deadlocks == rep.orders_run and rep.nonzero_counters == rep.orders_run


@pytest.mark.parametrize("fam", ["oproj.0", "down.1", "attn.0", "lm"])
def test_fault_missing_wait_is_a_race(fam):
    d = _host(wl.TINY, n_sm=8)
    code, rep = mk.mk_plan_simulate(d.plan, 2, [10, 100], 20, 3, mk.MK_SIM_FAULT_NO_WAIT, _family(d, fam))
    assert code != 0 and rep.races > 0, rep.first_error


def test_dynamic_queue_capacity_deep_model():
    # 16 layers: the per-layer queue pushes add up; the simulator checks the
    # plan's reserved range count against the pushes of a full step
    deep = wl.DenseShape(n_layers=16, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024,
                         vocab=1024)
    d = _host(deep, max_batch=2, sched=mk.MK_SCHED_DYNAMIC, n_sm=8)
    for B, ctx in [(1, [64]), (2, [300, 5])]:
        code, rep = mk.mk_plan_simulate(d.plan, B, ctx, n_orders=4, seed=5)
        assert code == 0, rep.first_error


def test_moe_plan_build_families_and_limits():
    lay = mk.MoELayer(wl.MOE_64x8, None, max_tokens=512, n_sm=148, host_only=True)
    names = [f.name.decode() for f in lay.families()]
    assert names == ["route", "mindptr", "egu", "edown", "combine", "mfin"]
    fu = {f.name.decode(): f.followup for f in lay.families()}
    assert fu["mindptr"] == 1 and fu["mfin"] == 1 and fu["egu"] == 0
    ext = {f.name.decode(): f.max_extent for f in lay.families()}
    # max tiles = ceil(512 * 8 / 64) + min(64, 4096) = 128; per tile ceil(F/128) = 11 gate/up tasks
    # and H/128 = 16 down tasks (128 weight rows each, the tcgen05 MMA's M)
    assert ext["egu"] == 128 * 11 and ext["edown"] == 128 * 16 and ext["route"] == 64
    assert mk.mk_plan_workspace_bytes(lay.plan) > 512 * 8 * (1408 * 2 + 2048 * 4)
    lay.close()
    for bad in (dict(n_experts=65), dict(top_k=9), dict(expert_ffn=1400), dict(expert_ffn=1376), dict(hidden=2304)):
        shp = wl.MoEShape(**{**dict(hidden=2048, n_experts=64, top_k=8, expert_ffn=1408), **bad})
        with pytest.raises(mk.MkError):
            mk.MoELayer(shp, None, max_tokens=64, n_sm=148, host_only=True)


def test_plan_option_ranges():
    # the option fields accept their documented values and refuse the rest
    for v in (0, 1, 2):
        mk.MoELayer(wl.MOE_64x8, None, max_tokens=8, n_sm=148, host_only=True, moe_tiles=v).close()
    for bad in (dict(moe_tiles=3), dict(moe_tiles=-1)):
        with pytest.raises(mk.MkError):
            mk.MoELayer(wl.MOE_64x8, None, max_tokens=8, n_sm=148, host_only=True, **bad)
    for split in (1, 8, 64):
        d = _host(wl.LLAMA_1B, max_batch=4, max_ctx=4160, n_sm=148, attn_split=split)
        assert d.tiles()["attn_split"] == split
        d.close()
    for bad in (dict(attn_split=65), dict(attn_split=-1), dict(act_split=3)):
        with pytest.raises(mk.MkError):
            _host(wl.LLAMA_1B, max_batch=16, max_ctx=1088, n_sm=148, **bad)
    # a given split is fixed; no split up to 8 rows: adaptive, at most 32
    assert _host(wl.LLAMA_1B, max_batch=4, max_ctx=4160, n_sm=148, attn_split=8).tiles()["attn_auto"] == 0
    t = _host(wl.LLAMA_1B, max_batch=8, max_ctx=4160, n_sm=148).tiles()
    assert (t["attn_split"], t["attn_auto"]) == (32, 1)
    # wide-batch defaults: 24 chunks per attention task above 8 rows (adaptive
    # up to 8), split K 4 / 4 / 2
    t = _host(wl.LLAMA_1B, max_batch=64, max_ctx=1088, n_sm=148).tiles()
    assert (t["attn_split"], t["attn_auto"], t["gseg_qkv"], t["gseg_o"], t["gseg_gu"], t["kseg"]) == \
        (24, 1, 4, 4, 2, 1024)


def test_moe_plan_requires_dynamic_schedule_and_rejects_dense_calls():
    d = mk.mk_model_desc()
    d.kind = mk.MK_MODEL_MOE_LAYER
    d.hidden, d.n_experts, d.top_k, d.expert_ffn, d.max_tokens = 2048, 64, 8, 1408, 64
    o = mk.mk_plan_opts()
    o.sched, o.host_only, o.n_sm = mk.MK_SCHED_STATIC, 1, 148
    with pytest.raises(mk.MkError) as e:
        mk.mk_plan_build(d, o)
    assert e.value.status == mk.MK_ERR_UNSUPPORTED
    o.sched = mk.MK_SCHED_DYNAMIC
    plan = mk.mk_plan_build(d, o)
    a = mk.mk_step_args()
    a.batch = 1
    with pytest.raises(mk.MkError):
        mk.mk_decode_step(plan, a, 0)
    mk.mk_plan_destroy(plan)


def test_stats_without_a_device():
    # mk_get_stats on a host-only plan: the plan's figures, no launch yet
    d = _host(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_sm=148)
    st = d.stats()
    assert st["launches"] == 0 and st["build_ms"] > 0.0
    assert st["n_families"] == len(d.families()) and st["n_sm"] == 148
    assert st["ring_slots"] == d.tiles()["ring_slots"]
    assert st["workspace_bytes"] == mk.mk_plan_workspace_bytes(d.plan)
    assert st["queue_ranges_cap"] == 0  # static schedule
    assert st["last_queue_tasks"] == -1 and st["last_queue_pops"] == -1
    d.close()


def test_shared_memory_split_per_max_batch():
    # the staging buffer holds 2 x max_batch bf16 rows (value and remainder)
    # up to 8 rows, the rest of 227 KB goes to 16 KB ring slots after the 9 KB
    # fixed area and the 16 KB of GEMV partial tiles
    rows = {1: 2, 2: 4, 4: 8, 8: 8}
    for mb, want in ((1, 12), (2, 11), (4, 10), (8, 10)):
        act = max(8192, (rows[mb] * (2048 + 8) * 2 + 127) // 128 * 128)
        assert (232448 - 9 * 1024 - act - 16384) // 16384 == want
        d = _host(wl.LLAMA_1B, max_batch=mb, max_ctx=1088, n_sm=148)
        assert d.tiles()["ring_slots"] == want
        d.close()
    # above 8 rows the wide-batch path: no partial tiles; the staging buffer
    # holds the MMA issuer's activation chunks (3 stages x rows x 128 B, rows
    # = max_batch rounded up to 16, twice that with the value + remainder
    # split) or the QKV exchange (64 x rows fp32)
    for mb, split, act in ((9, 0, 3 * 32 * 128), (64, 0, 3 * 128 * 128), (64, 2, 3 * 64 * 128)):
        d = _host(wl.LLAMA_1B, max_batch=mb, max_ctx=1088, n_sm=148, act_split=split)
        t = d.tiles()
        assert t["tile_qkv"] == t["tile_o"] == t["tile_gu"] == t["tile_down"] == t["tile_lm"] == 128
        assert t["act_split"] == (split != 2)
        assert t["ring_slots"] == (232448 - 9 * 1024 - act) // 16384
        d.close()
    with pytest.raises(mk.MkError):  # value + remainder rows only up to 64 batch rows
        _host(wl.LLAMA_1B, max_batch=128, max_ctx=1088, n_sm=148, act_split=1,
              moe=(wl.MOE_64x8, None, None))
    with pytest.raises(mk.MkError):
        _host(wl.LLAMA_1B, max_batch=65, max_ctx=1088, n_sm=148)


# ---------------------------------------------------------------- MoE graphs in the simulator
TINY_MOE = wl.MoEShape(hidden=256, n_experts=8, top_k=2, expert_ffn=64)


def _moe_layer_host(n_sm=16, max_tokens=512):
    return mk.MoELayer(wl.MOE_64x8, None, max_tokens=max_tokens, n_sm=n_sm, host_only=True)


def _moe_decoder_host(n_sm=8, max_batch=4):
    return mk.DenseDecoder(wl.TINY, max_batch=max_batch, max_ctx=320, n_slots=max_batch, n_sm=n_sm,
                           host_only=True, moe=(TINY_MOE, None, None))


@pytest.mark.parametrize("T", [1, 8, 64, 200])
@pytest.mark.parametrize("seed", [2, 3])  # uniform and Zipf-skewed routing
def test_moe_layer_simulator_clean(T, seed):
    # data-dependent arming and triggering: the routing follow-up arms the
    # down count and one gate/up count per tile, and pushes as many GroupGEMM
    # tasks as exp_indptr implies; every order must be race-free, run each
    # task once and leave every counter at zero
    lay = _moe_layer_host()
    code, rep = mk.mk_plan_simulate(lay.plan, T, None, n_orders=6, seed=seed)
    assert code == 0, rep.first_error
    assert rep.races == 0 and rep.deadlocks == 0 and rep.exactly_once_violations == 0 and rep.nonzero_counters == 0
    # route + combine (ceil(T/8) each), mindptr, mfin, and per tile ceil(F/128) gate/up + H/128 down tasks
    fixed = 2 * ((T + 7) // 8) + 2
    assert (rep.tasks_per_order - fixed) % (11 + 16) == 0 and rep.tasks_per_order > fixed
    mk.mk_plan_validate(lay.plan, T, None)


def test_moe_layer_simulator_one_token_touches_eight_tiles():
    # T = 1 with top-8 routing: 8 experts with one row each -> 8 tiles
    lay = _moe_layer_host()
    code, rep = mk.mk_plan_simulate(lay.plan, 1, None, n_orders=2, seed=4)
    assert code == 0 and rep.tasks_per_order == 2 + 2 + 8 * (11 + 16), rep.first_error


@pytest.mark.parametrize("B,ctx", [(1, [64]), (3, [5, 70, 130]), (4, [0, 1, 63, 64])])
def test_moe_decoder_simulator_clean(B, ctx):
    d = _moe_decoder_host()
    for seed in (1, 2):
        code, rep = mk.mk_plan_simulate(d.plan, B, ctx, n_orders=20, seed=seed)
        assert code == 0, rep.first_error
        assert rep.races == 0 and rep.deadlocks == 0 and rep.nonzero_counters == 0
    mk.mk_plan_validate(d.plan, B, ctx)


@pytest.mark.parametrize("fam,fault,want", [
    ("egu", mk.MK_SIM_FAULT_DROP_NOTIFY, "deadlock"),
    ("route", mk.MK_SIM_FAULT_COUNT_PLUS_ONE, "deadlock"),
    ("edown", mk.MK_SIM_FAULT_DROP_NOTIFY, "deadlock"),
    # a tile armed with one gate/up task too few: its down tasks read a
    # SwiGLU row block that is still being written
    ("egu", mk.MK_SIM_FAULT_COUNT_MINUS_ONE, "race"),
    # the down count armed one too low: the combine reads unfinished rows
    ("edown", mk.MK_SIM_FAULT_COUNT_MINUS_ONE, "race"),
    # the routing event one too low: exp_indptr built before every pair is counted
    ("route", mk.MK_SIM_FAULT_COUNT_MINUS_ONE, "race"),
])
def test_moe_layer_simulator_detects_faults(fam, fault, want):
    # (MoE plans run the dynamic schedule only: a task is pushed when its
    # event fires, so the data-dependent counts the routing arms are what
    # orders the GroupGEMM tiles)
    lay = _moe_layer_host()
    f = [x.name.decode() for x in lay.families()].index(fam)
    code, rep = mk.mk_plan_simulate(lay.plan, 24, None, 6, 5, fault, f)
    assert code != 0
    if want == "deadlock":
        assert rep.deadlocks == rep.orders_run
    elif want == "race":
        assert rep.races > 0, rep.first_error


@pytest.mark.parametrize("fam,want", [("oproj.1", "race"), ("edown.0", "race"), ("egu.1", "deadlock"),
                                      ("combine.0", "deadlock")])
def test_moe_decoder_count_minus_one(fam, want):
    # ROUTE reads the residual the O projection wrote, COMBINE the rows of
    # every down task: one notify too few releases them early.  With B = 3
    # the layer has one COMBINE task, and with F = 64 a tile has one gate/up
    # task, so those events armed at zero never fire (their consumers are
    # pushed by the notify that reaches zero)
    d = _moe_decoder_host()
    f = [x.name.decode() for x in d.families()].index(fam)
    code, rep = mk.mk_plan_simulate(d.plan, 3, [5, 70, 130], 20, 3, mk.MK_SIM_FAULT_COUNT_MINUS_ONE, f)
    assert code != 0
    if want == "race":
        assert rep.races > 0, rep.first_error
    else:
        assert rep.deadlocks == rep.orders_run
