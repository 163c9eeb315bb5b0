"""GPU parity of the dense decode megakernel against the CPU oracle.

Every check goes through the C ABI (libmk.so) on cuda:0.  Tolerance: max
|gpu - oracle| <= 2e-2 * max |oracle| per tensor; integer results (task set,
argmax up to near ties) exact.
"""
import pytest
import torch

import event_tensor_task_b200 as mk
import workloads as wl
from gpu_common import DenseCase, rel_err, check_argmax, TOL
from oracle import tasks as ot

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    return DenseCase(wl.TINY, max_batch=4, max_ctx=320, n_slots=4, ctx_fill=[64, 0, 70, 190])


def _oracle_step(case, tokens, slots, ctx, capture=False):
    K, V = case.K_cpu.clone(), case.V_cpu.clone()
    return case.oracle.step(K, V, tokens, slots, ctx, capture=capture), K, V


def test_tiny_single_step_parity(tiny):
    tokens, slots, ctx = [17], [0], [64]
    ref, K, V = _oracle_step(tiny, tokens, slots, ctx)
    got = tiny.gpu_step(tokens, slots, ctx)
    assert rel_err(got["logits"], ref["logits"]) <= TOL
    check_argmax(got["next_tokens"][0], ref["logits"][0])
    tiny.check_task_set(got["task_counts"], 1, ctx)
    # the appended cache rows (rotated key, value) match the oracle's
    for l in range(wl.TINY.n_layers):
        assert rel_err(tiny.K[l, 0, :, 64].cpu(), K[l, 0, :, 64]) <= TOL
        assert rel_err(tiny.V[l, 0, :, 64].cpu(), V[l, 0, :, 64]) <= TOL


def test_tiny_ragged_batch_parity(tiny):
    # sequences at context 0 (empty cache), 70 and 190 in slots 1..3; the
    # residual after every layer is compared too
    tokens, slots, ctx = [3, 900, 511], [1, 2, 3], [0, 70, 190]
    ref, _, _ = _oracle_step(tiny, tokens, slots, ctx, capture=True)
    got = tiny.gpu_step(tokens, slots, ctx, capture=True)
    tiny.check_hidden(got, ref)
    for b in range(3):
        assert rel_err(got["logits"][b], ref["logits"][b]) <= TOL
        check_argmax(got["next_tokens"][b], ref["logits"][b])
    tiny.check_task_set(got["task_counts"], 3, ctx)


def test_tiny_symbolic_shapes_one_plan(tiny):
    # one plan, one kernel: B and the contexts change every step
    for tokens, slots, ctx in [([5], [0], [64]), ([6, 7, 8, 9], [0, 1, 2, 3], [64, 0, 70, 190]),
                               ([10, 11], [3, 1], [190, 0])]:
        ref, _, _ = _oracle_step(tiny, tokens, slots, ctx)
        got = tiny.gpu_step(tokens, slots, ctx)
        assert rel_err(got["logits"], ref["logits"]) <= TOL
        tiny.check_task_set(got["task_counts"], len(tokens), ctx)


def test_tiny_static_equals_dynamic_bitwise(tiny):
    dyn = DenseCase(wl.TINY, max_batch=4, max_ctx=320, n_slots=4, ctx_fill=[64, 0, 70, 190],
                    sched=mk.MK_SCHED_DYNAMIC)
    tokens, slots, ctx = [3, 900, 511], [1, 2, 3], [0, 70, 190]
    a = tiny.gpu_step(tokens, slots, ctx)
    b = dyn.gpu_step(tokens, slots, ctx)
    assert torch.equal(a["logits"], b["logits"])
    assert torch.equal(a["next_tokens"], b["next_tokens"])
    dyn.check_task_set(b["task_counts"], 3, ctx)
    # the dynamic queue of that launch: every task except the follow-ups
    # (MERGE, LMFIN run where their event fired) was pushed once, plus one
    # END per CTA, and every push was popped
    want = ot.expected_dense_tasks(wl.TINY, 3, ctx, dyn.tiles_for_oracle())
    st = dyn.dec.stats()
    pushed = sum(1 for f, _, _ in want if f != "lmfin") + st["n_sm"]
    assert st["last_queue_tasks"] == pushed and st["last_queue_pops"] == pushed
    assert 0 < st["last_queue_ranges"] <= st["queue_ranges_cap"] and st["launches"] == 1


def test_tiny_dynamic_steps_after_reset(tiny):
    # a reset restarts the launch epochs; queue entries tagged by the epochs
    # before it must not be taken for entries of the steps after it
    dyn = DenseCase(wl.TINY, max_batch=4, max_ctx=320, n_slots=4, ctx_fill=[64, 0, 70, 190],
                    sched=mk.MK_SCHED_DYNAMIC)
    tokens, slots, ctx = [3, 900, 511], [1, 2, 3], [0, 70, 190]
    ref, _, _ = _oracle_step(dyn, tokens, slots, ctx)
    for rnd in range(2):
        for i in range(4):
            got = dyn.gpu_step(tokens, slots, ctx)
            assert rel_err(got["logits"], ref["logits"]) <= TOL
            dyn.check_task_set(got["task_counts"], 3, ctx)
        dyn.dec.reset()


def test_tiny_greedy_walk(tiny):
    # greedy decode; both sides continue from the oracle's token
    tok, pos = 42, 64
    K, V = tiny.K_cpu.clone(), tiny.V_cpu.clone()
    torch.cuda.synchronize()
    tiny.K.copy_(tiny.K_cpu.to("cuda:0"))
    tiny.V.copy_(tiny.V_cpu.to("cuda:0"))
    for step in range(8):
        ref = tiny.oracle.step(K, V, [tok], [0], [pos])
        got = tiny.gpu_step([tok], [0], [pos], counts=False)
        assert rel_err(got["logits"], ref["logits"]) <= TOL
        check_argmax(got["next_tokens"][0], ref["logits"][0])
        tok = int(ref["next_tokens"][0])
        pos += 1


@pytest.fixture(scope="module")
def llama():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    return DenseCase(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_slots=1, ctx_fill=[1024])


def test_llama1b_greedy_32_steps_parity(llama):
    # the 32-step greedy window from context 1024 against the oracle, both
    # sides continuing from the oracle's token; task set at the first step,
    # the residual after every layer at the first and the last step
    tokens = wl.token_ids(1, wl.LLAMA_1B.vocab).tolist()
    llama.K.copy_(llama.K_cpu.to("cuda:0"))
    llama.V.copy_(llama.V_cpu.to("cuda:0"))
    K, V = llama.K_cpu.clone(), llama.V_cpu.clone()
    tok, pos = tokens[0], 1024
    for step in range(32):
        edge = step in (0, 31)
        ref = llama.oracle.step(K, V, [tok], [0], [pos], capture=edge)
        got = llama.gpu_step([tok], [0], [pos], counts=(step == 0), capture=edge)
        assert rel_err(got["logits"], ref["logits"]) <= TOL
        check_argmax(got["next_tokens"][0], ref["logits"][0])
        if edge:
            llama.check_hidden(got, ref)
        if step == 0:
            llama.check_task_set(got["task_counts"], 1, [pos])
        tok = int(ref["next_tokens"][0])
        pos += 1


def test_llama1b_greedy_32_static_vs_dynamic(llama):
    dev = "cuda:0"
    dyn = mk.DenseDecoder(wl.LLAMA_1B, llama.w, llama.K, llama.V, max_batch=1, max_ctx=1088, n_slots=1,
                          sched=mk.MK_SCHED_DYNAMIC)
    tok0 = int(wl.token_ids(1, wl.LLAMA_1B.vocab)[0])
    seqs = []
    for dec in (llama.dec, dyn):
        llama.K.copy_(llama.K_cpu.to(dev))
        llama.V.copy_(llama.V_cpu.to(dev))
        cur = torch.tensor([tok0], dtype=torch.int32, device=dev)
        slot = torch.zeros(1, dtype=torch.int32, device=dev)
        out = []
        logits = torch.empty(1, wl.LLAMA_1B.vocab, device=dev)
        last = None
        for i in range(32):
            ctx = torch.tensor([1024 + i], dtype=torch.int32, device=dev)
            nxt = torch.empty(1, dtype=torch.int32, device=dev)
            dec.step(cur, slot, ctx, nxt, logits=logits)
            cur = nxt
            out.append(nxt)
        torch.cuda.synchronize()
        assert dec.status()[0] == 0
        seqs.append((torch.cat(out).cpu(), logits.cpu().clone()))
    assert torch.equal(seqs[0][0], seqs[1][0])
    assert torch.equal(seqs[0][1], seqs[1][1])  # bit-identical final logits


def test_llama1b_long_ragged_contexts():
    # the symbolic-batch workload's context range: three sequences at 128,
    # 2100 and 4095 cached tokens in one step (3 to 65 key chunks each)
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    ctx = [128, 2100, 4095]
    case = DenseCase(wl.LLAMA_1B, max_batch=4, max_ctx=4104, n_slots=4, ctx_fill=ctx + [0])
    tokens = wl.token_ids(3, wl.LLAMA_1B.vocab).tolist()
    ref, _, _ = _oracle_step(case, tokens, [0, 1, 2], ctx)
    got = case.gpu_step(tokens, [0, 1, 2], ctx)
    for b in range(3):
        assert rel_err(got["logits"][b], ref["logits"][b]) <= TOL
        check_argmax(got["next_tokens"][b], ref["logits"][b])
    case.check_task_set(got["task_counts"], 3, ctx)


@pytest.mark.parametrize("sched", [mk.MK_SCHED_STATIC, mk.MK_SCHED_DYNAMIC])
def test_tiny_batch_of_eight(sched):
    # B up to 8: every column of the GEMV's MMA n = 8 carries a batch row;
    # one plan steps B = 8, 5 and 1 with ragged contexts
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    fill = [64, 0, 70, 190, 5, 127, 128, 300]
    case = DenseCase(wl.TINY, max_batch=8, max_ctx=320, n_slots=8, ctx_fill=fill, sched=sched)
    K, V = case.K_cpu.clone(), case.V_cpu.clone()
    tok = wl.token_ids(8, wl.TINY.vocab).tolist()
    for tokens, slots, ctx in [(tok, list(range(8)), fill),
                               (tok[:5], [7, 1, 3, 0, 5], [301, 1, 191, 65, 128]),
                               (tok[:1], [6], [129])]:
        ref = case.oracle.step(K, V, tokens, slots, ctx)
        got = case.gpu_step(tokens, slots, ctx)
        for b in range(len(tokens)):
            assert rel_err(got["logits"][b], ref["logits"][b]) <= TOL
            check_argmax(got["next_tokens"][b], ref["logits"][b])
        case.check_task_set(got["task_counts"], len(tokens), ctx)


def test_llama1b_batch_of_eight():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    ctx = [128, 700, 1500, 2100, 64, 0, 999, 4095]
    case = DenseCase(wl.LLAMA_1B, max_batch=8, max_ctx=4104, n_slots=8, ctx_fill=ctx)
    tokens = wl.token_ids(8, wl.LLAMA_1B.vocab).tolist()
    ref, _, _ = _oracle_step(case, tokens, list(range(8)), ctx, capture=True)
    got = case.gpu_step(tokens, list(range(8)), ctx, capture=True)
    case.check_hidden(got, ref)
    for b in range(8):
        assert rel_err(got["logits"][b], ref["logits"][b]) <= TOL
        check_argmax(got["next_tokens"][b], ref["logits"][b])
    case.check_task_set(got["task_counts"], 8, ctx)


@pytest.mark.parametrize("sched", [mk.MK_SCHED_STATIC, mk.MK_SCHED_DYNAMIC])
def test_llama1b_many_steps_ring_reuse(llama, sched):
    # 64-row tasks take 16 ring slots, so a task reuses ring positions of its
    # own first slots: many steps in a row must neither stall nor change the
    # result (the last step is compared with a fresh single step)
    case = llama if sched == mk.MK_SCHED_STATIC else DenseCase(wl.LLAMA_1B, max_batch=1, max_ctx=1088, n_slots=1,
                                                              ctx_fill=[1024], sched=sched)
    assert case.dec.tiles()["ring_slots"] < 16 and case.dec.tiles()["tile_lm"] == 64
    tokens, slots, ctx = [77], [0], [1024]
    first = case.gpu_step(tokens, slots, ctx)
    for _ in range(150):
        last = case.gpu_step(tokens, slots, ctx, counts=False)
    assert torch.equal(first["logits"], last["logits"])
