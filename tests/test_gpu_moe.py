"""GPU parity of the MoE FFN layer (mk_moe_layer) against the CPU oracle.

Every check goes through the C ABI on cuda:0.  Exact: the router logits
(fixed fp32 summation order on both sides), the top-k expert ids, the
expert histogram, exp_indptr and the set of tasks the launch ran.  Within
tolerance: the softmax weights (fp32 vs fp64, 1e-5) and the layer output
(max |gpu - oracle| <= 2e-2 * max |oracle|; the GPU stores the SwiGLU rows
and the output in bf16).
"""
import pytest
import torch

import event_tensor_task_b200 as mk
import oracle
import workloads as wl
from oracle import tasks as ot
from gpu_common import rel_err, counters_at_zero, TOL

pytestmark = pytest.mark.gpu

# the plan's GroupGEMM tiles: routed rows per tile (128 for experts with more
# than 64 rows: routing-aware), weight rows per task
TILES = {"tm": 64, "big": 128, "tn": 128, "td": 128}
TINY_MOE = wl.MoEShape(hidden=256, n_experts=8, top_k=2, expert_ffn=64)


def _weights(shape):
    w_cpu = wl.moe_weights(shape, seed=0)
    return w_cpu, {k: v.to("cuda:0") for k, v in w_cpu.items()}


def _task_set(layer, counts):
    got = set()
    for f in layer.families():
        seg = counts[f.debug_base:f.debug_base + f.max_extent]
        assert int(seg.max()) <= 1, f"{f.name.decode()}: a task ran more than once"
        for i in torch.nonzero(seg).flatten().tolist():
            got.add((f.name.decode(), -1, i))
    return got


def _check(shape, layer, w_cpu, bias_cpu, T, seed=0):
    dev = "cuda:0"
    H, E, K = shape.hidden, shape.n_experts, shape.top_k
    x = wl.moe_tokens(T, H, seed=seed)
    ref = oracle.moe_layer(x, w_cpu, K, bias_cpu)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    idx = torch.full((T, K), -1, dtype=torch.int32, device=dev)
    wts = torch.empty(T, K, dtype=torch.float32, device=dev)
    hist = torch.empty(E, dtype=torch.int32, device=dev)
    indptr = torch.empty(E + 1, dtype=torch.int32, device=dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    counts = torch.zeros(mk.mk_plan_task_slots(layer.plan), dtype=torch.int32, device=dev)
    layer(x.to(dev), out, topk_idx=idx, topk_w=wts, hist=hist, indptr=indptr, logits=logits, task_counts=counts)
    torch.cuda.synchronize()
    code, st = layer.status()
    assert code == 0, f"device status {code} family {st.family} index {st.index} event {st.event}"
    counters_at_zero(layer)
    assert torch.equal(logits.cpu(), ref["logits"]), "router logits differ (the summation order is fixed)"
    assert torch.equal(idx.cpu(), ref["idx"])
    assert torch.equal(hist.cpu(), ref["hist"])
    assert torch.equal(indptr.cpu(), ref["indptr"])
    assert float((wts.cpu().double() - ref["weights"]).abs().max()) <= 1e-5
    assert rel_err(out.float(), ref["out"]) <= TOL
    assert _task_set(layer, counts.cpu()) == ot.expected_moe_tasks(T, ref["hist"], H, shape.expert_ffn, TILES)
    return ref


@pytest.fixture(scope="module")
def tiny():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    w_cpu, w = _weights(TINY_MOE)
    bias_cpu = wl.zipf_bias(TINY_MOE.n_experts)
    layer = mk.MoELayer(TINY_MOE, w, bias_cpu.to("cuda:0"), max_tokens=200, debug=True)
    yield w_cpu, bias_cpu, layer
    layer.close()


@pytest.mark.parametrize("T", [1, 5, 13, 64, 200])
def test_tiny_moe_parity(tiny, T):
    # ragged token counts (not multiples of 8), one plan for every T
    w_cpu, bias_cpu, layer = tiny
    _check(TINY_MOE, layer, w_cpu, bias_cpu, T, seed=T)


def test_tiny_moe_repeated_calls(tiny):
    # the histogram and the data-dependent counts are re-armed every launch
    w_cpu, bias_cpu, layer = tiny
    for T in (13, 200, 1, 13):
        _check(TINY_MOE, layer, w_cpu, bias_cpu, T, seed=7)


@pytest.fixture(scope="module")
def moe64():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    w_cpu, w = _weights(wl.MOE_64x8)
    bias_cpu = wl.zipf_bias(wl.MOE_64x8.n_experts)
    uniform = mk.MoELayer(wl.MOE_64x8, w, None, max_tokens=512, debug=True)
    skewed = mk.MoELayer(wl.MOE_64x8, w, bias_cpu.to("cuda:0"), max_tokens=512, debug=True)
    yield w_cpu, bias_cpu, uniform, skewed
    uniform.close()
    skewed.close()


@pytest.mark.parametrize("T", [1, 8, 64, 512])
@pytest.mark.parametrize("regime", ["uniform", "zipf"])
def test_moe_64x8_parity(moe64, T, regime):
    w_cpu, bias_cpu, uniform, skewed = moe64
    if regime == "uniform":
        ref = _check(wl.MOE_64x8, uniform, w_cpu, None, T)
    else:
        ref = _check(wl.MOE_64x8, skewed, w_cpu, bias_cpu, T)
    assert int(ref["hist"].sum()) == 8 * T
