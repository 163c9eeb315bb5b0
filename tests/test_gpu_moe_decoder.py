"""GPU parity of the MoE decoder (MK_MODEL_MOE_DECODER: each layer's FFN is
an MoE layer) against the CPU oracle, through mk_decode_step on cuda:0.

Continuous batching: one plan, the batch size and the contexts change every
step; skewed (Zipf) routing; dynamic schedule.  The oracle's decode step
takes the MoE FFN on the bf16-rounded normalised residual rows (the MoE
layer's input is a stored bf16 tensor).  Checked per step:
  - logits and the residual after every layer within max |gpu - oracle| <=
    2e-2 * max |oracle|, greedy tokens (up to near ties);
  - the expert set of every token equal to the oracle's own routing, or a
    near tie (the experts that differ lie within 2e-2 * max |logit| of the
    top-k boundary); a row routed across a near tie leaves the comparison
    from that layer on (its later values follow another, equally valid
    routing), at most one row in eight;
  - layer-local routing, exact: each layer's top-k ids, expert histogram and
    exp_indptr equal the oracle's MoE layer run on the bf16 router input the
    GPU captured for that layer (floating-point drift across layers cannot
    flip a comparison there);
  - every event counter at zero after the step.
"""
import pytest
import torch

import event_tensor_task_b200 as mk
import oracle
import workloads as wl
from conftest import record_margin
from gpu_common import rel_err, check_argmax, counters_at_zero, TOL

ROUTE_TIE = 2e-2  # near-tie routing margin, relative to max |router logit| of the row

pytestmark = pytest.mark.gpu


class MoeCase:
    def __init__(self, shape, mshape, max_batch, max_ctx, ctx_fill):
        dev = "cuda:0"
        self.shape, self.mshape = shape, mshape
        self.w_cpu = wl.dense_weights(shape, seed=0)
        self.m_cpu = [wl.moe_weights(mshape, seed=0, prefix=f"layers.{l}.moe.") for l in range(shape.n_layers)]
        self.bias = wl.zipf_bias(mshape.n_experts)
        self.K_cpu, self.V_cpu = wl.kv_cache(shape, max_batch, max_ctx, ctx_fill, seed=0)
        self.w = {k: v.to(dev) for k, v in self.w_cpu.items()}
        self.m = [{k: v.to(dev) for k, v in d.items()} for d in self.m_cpu]
        self.K, self.V = self.K_cpu.to(dev), self.V_cpu.to(dev)
        self.dec = mk.DenseDecoder(shape, self.w, self.K, self.V, max_batch=max_batch, max_ctx=max_ctx,
                                   n_slots=max_batch, moe=(mshape, self.m, self.bias.to(dev)))
        self.orc = oracle.DenseOracle(shape, self.w_cpu)

    def oracle_moe(self, l, u):
        r = oracle.moe_layer(u.to(torch.bfloat16), self.m_cpu[l], self.mshape.top_k, self.bias)
        self.routes[l] = r
        return r["out"]

    def step(self, K, V, tokens, slots, ctx):
        dev = "cuda:0"
        self.routes = {}
        ref = self.orc.step(K, V, tokens, slots, ctx, moe=self.oracle_moe, capture=True)
        B = len(tokens)
        L, H, E, k = self.shape.n_layers, self.shape.hidden, self.mshape.n_experts, self.mshape.top_k
        nxt = torch.full((B,), -1, dtype=torch.int32, device=dev)
        logits = torch.empty(B, self.shape.vocab, dtype=torch.float32, device=dev)
        cap = {"resid": torch.full((L, B, H), float("nan"), device=dev),
               "moe_in": torch.zeros(L, B, H, dtype=torch.bfloat16, device=dev),
               "topk": torch.full((L, B, k), -1, dtype=torch.int32, device=dev),
               "hist": torch.full((L, E), -1, dtype=torch.int32, device=dev),
               "indptr": torch.full((L, E + 1), -1, dtype=torch.int32, device=dev)}
        self.dec.step(torch.tensor(tokens, dtype=torch.int32, device=dev),
                      torch.tensor(slots, dtype=torch.int32, device=dev),
                      torch.tensor(ctx, dtype=torch.int32, device=dev), nxt, logits=logits, capture=cap)
        torch.cuda.synchronize()
        code, st = self.dec.status()
        assert code == 0, f"device status {code} family {st.family} index {st.index} event {st.event}"
        counters_at_zero(self.dec)
        cap = {n: t.cpu() for n, t in cap.items()}
        diverged = set()  # rows whose routing took the other side of a near tie
        for l in range(L):  # (layer by layer first: a failure names the layer)
            # layer-local routing on the GPU's own bf16 router input
            r = oracle.moe_layer(cap["moe_in"][l], self.m_cpu[l], k, self.bias)
            assert torch.equal(cap["topk"][l], r["idx"]), f"layer {l}: top-k ids"
            assert torch.equal(cap["hist"][l], r["hist"]), f"layer {l}: expert histogram"
            assert torch.equal(cap["indptr"][l], r["indptr"]), f"layer {l}: exp_indptr"
            # against the oracle's own routing: the same expert sets, or a near tie
            for b in range(B):
                if b not in diverged and not same_experts(cap["topk"][l][b], self.routes[l], b, k):
                    diverged.add(b)
            assert len(diverged) <= max(1, B // 8), f"layer {l}: {len(diverged)} of {B} rows routed differently"
            for b in range(B):
                if b not in diverged:
                    assert rel_err(cap["resid"][l, b], ref["residual"][l][b]) <= TOL, f"layer {l} row {b}"
        for b in range(B):
            if b not in diverged:
                assert rel_err(logits[b].cpu(), ref["logits"][b]) <= TOL, f"logits row {b}"
                check_argmax(nxt[b].cpu(), ref["logits"][b])
        return ref


def same_experts(gpu_idx, route, b, k):
    """Whether row b's GPU expert set equals the oracle's.  A differing set is
    accepted as a near tie when every expert in the symmetric difference has
    an oracle router logit within ROUTE_TIE * max |logit| of the boundary
    between the k-th and (k+1)-th largest (the router input of the two sides
    differs by the bf16 rounding of the normalised residual, which can move a
    logit across that boundary); anything else fails."""
    mine, theirs = set(gpu_idx.tolist()), set(route["idx"][b].tolist())
    if mine == theirs:
        return True
    lg = route["logits"][b].double()
    s = torch.sort(lg, descending=True).values
    boundary = 0.5 * float(s[k - 1] + s[k]) if k < lg.numel() else float(s[-1])
    margin = ROUTE_TIE * float(lg.abs().max())
    far = [e for e in mine ^ theirs if abs(float(lg[e]) - boundary) > margin]
    assert not far, f"row {b}: experts {sorted(mine)} vs oracle {sorted(theirs)}, {far} not near the top-{k} boundary"
    record_margin(route_tie=True)
    return False


def _walk(case, steps):
    K, V = case.K_cpu.clone(), case.V_cpu.clone()
    for tokens, slots, ctx in steps:
        case.step(K, V, tokens, slots, ctx)


def test_tiny_moe_decoder_continuous_batching():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mshape = wl.MoEShape(hidden=256, n_experts=8, top_k=2, expert_ffn=64)
    case = MoeCase(wl.TINY, mshape, max_batch=4, max_ctx=320, ctx_fill=[64, 10, 130, 200])
    _walk(case, [([17], [0], [64]),
                 ([3, 900, 511], [1, 2, 3], [10, 130, 200]),
                 ([5, 6, 7, 8], [0, 1, 2, 3], [65, 11, 131, 201]),
                 ([9, 10], [2, 0], [132, 66])])


def test_tiny_moe_decoder_batch_of_eight():
    # B up to 8: the MoE FFN on 8 tokens (ROUTE in one task, ragged per-expert
    # rows) after attention over eight ragged contexts
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mshape = wl.MoEShape(hidden=256, n_experts=8, top_k=2, expert_ffn=64)
    fill = [64, 10, 130, 200, 0, 77, 250, 5]
    case = MoeCase(wl.TINY, mshape, max_batch=8, max_ctx=320, ctx_fill=fill)
    _walk(case, [(list(range(11, 19)), list(range(8)), fill),
                 ([19, 20, 21, 22, 23], [7, 0, 4, 2, 5], [6, 65, 1, 131, 78])])


def test_moe_decoder_1b_attention_64_experts():
    # two layers of the 1B attention shape, each FFN the 64-expert top-8 layer
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    shape = wl.DenseShape(n_layers=2, hidden=2048, n_q_heads=32, n_kv_heads=8, head_dim=64, ffn=8192,
                          vocab=128256)
    case = MoeCase(shape, wl.MOE_64x8, max_batch=4, max_ctx=1100, ctx_fill=[256, 1000, 512, 300])
    tok = wl.token_ids(4, shape.vocab).tolist()
    _walk(case, [([tok[0]], [0], [256]),
                 (tok[:3], [0, 1, 2], [257, 1000, 512]),
                 (tok, [0, 1, 2, 3], [258, 1001, 513, 300])])


def test_tiny_moe_decoder_wide_batch():
    # above 8 rows the decoder's attention half and LM head run the wide-batch
    # path (tcgen05 GEMM tasks on materialised bf16 activations); its FFN is
    # the MoE layer on the B tokens: one plan for B = 16, 9 and 12
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mshape = wl.MoEShape(hidden=256, n_experts=8, top_k=2, expert_ffn=64)
    fill = [64, 10, 130, 200, 0, 77, 250, 5, 1, 2, 3, 100, 64, 65, 129, 33]
    case = MoeCase(wl.TINY, mshape, max_batch=16, max_ctx=320, ctx_fill=fill)
    assert case.dec.tiles()["wide"] == 1
    tok = wl.token_ids(16, wl.TINY.vocab).tolist()
    _walk(case, [(tok, list(range(16)), fill),
                 (tok[:9], [15, 0, 4, 2, 5, 7, 9, 11, 13], [34, 65, 1, 131, 78, 6, 3, 101, 65]),
                 (tok[:12], list(range(12)), [65, 11, 131, 201, 1, 79, 251, 7, 2, 4, 4, 102])])


def test_tiny_moe_decoder_batch_128():
    # the widest plan (max_batch 128: activation boxes and MMA N of 128 rows)
    # on the tiny shape, B = 128 and 70
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mshape = wl.MoEShape(hidden=256, n_experts=8, top_k=2, expert_ffn=64)
    fill = [int(c) for c in wl.context_lengths(128, 0, 300, stream="tiny-128")]
    case = MoeCase(wl.TINY, mshape, max_batch=128, max_ctx=320, ctx_fill=fill)
    tok = wl.token_ids(128, wl.TINY.vocab).tolist()
    _walk(case, [(tok, list(range(128)), fill),
                 (tok[:70], list(range(70)), [c + 1 for c in fill[:70]])])


def test_moe_decoder_1b_attention_batch_128():
    # the MoE decoder workload's width: two layers of the 1B attention shape,
    # 64 experts top-8 per layer, B = 128 with contexts uniform in [256, 4096]
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    shape = wl.DenseShape(n_layers=2, hidden=2048, n_q_heads=32, n_kv_heads=8, head_dim=64, ffn=8192,
                          vocab=128256)
    ctx = [int(c) for c in wl.context_lengths(128, 256, 4096, stream="moe-decoder-ctx")]
    case = MoeCase(shape, wl.MOE_64x8, max_batch=128, max_ctx=4104, ctx_fill=ctx)
    tok = wl.token_ids(128, shape.vocab).tolist()
    _walk(case, [(tok, list(range(128)), ctx)])
