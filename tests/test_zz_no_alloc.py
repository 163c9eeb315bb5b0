"""mk_decode_step_static (scratch in a module-scope device array, no device
allocation) against mk_decode_step (caller workspace), through the C ABI.

The file name sorts last, so in a full run these tests come after every other
GPU test; they must also pass alone.  Both entry points run the same kernel
on the same plan shape, so results are compared bit for bit: logits, next
tokens and the KV-cache rows each step appends.
"""
import pytest
import torch

import event_tensor_task_b200 as mk
import workloads as wl


def _case(shape, max_batch, max_ctx, ctx_fill, sched, workspace):
    w = {k: v.to("cuda:0") for k, v in wl.dense_weights(shape, seed=0).items()}
    K, V = wl.kv_cache(shape, max_batch, max_ctx, ctx_fill, seed=0)
    K, V = K.to("cuda:0"), V.to("cuda:0")
    dec = mk.DenseDecoder(shape, w, K, V, max_batch=max_batch, max_ctx=max_ctx, n_slots=max_batch, sched=sched,
                          workspace=workspace)
    return dec, K, V


def _two_calls(dec, calls, static_scratch):
    """Run the calls in a row; each call after the first feeds back the
    previous call's next tokens.  Returns per call (logits, next tokens)."""
    dev = "cuda:0"
    out, prev = [], None
    for tokens, slots, ctx in calls:
        tok = torch.tensor(tokens, dtype=torch.int32, device=dev)
        if prev is not None:
            n = min(len(tokens), prev.numel())
            tok[:n] = prev[:n]
        sl = torch.tensor(slots, dtype=torch.int32, device=dev)
        cx = torch.tensor(ctx, dtype=torch.int32, device=dev)
        nxt = torch.full((len(slots),), -1, dtype=torch.int32, device=dev)
        logits = torch.empty(len(slots), dec.shape.vocab, dtype=torch.float32, device=dev)
        dec.step(tok, sl, cx, nxt, logits=logits, static_scratch=static_scratch)
        out.append((logits, nxt))
        prev = nxt
    torch.cuda.synchronize()
    return [(l.cpu(), n.cpu()) for l, n in out]


def _compare(shape, max_batch, max_ctx, ctx_fill, calls, sched):
    ref, K_r, V_r = _case(shape, max_batch, max_ctx, ctx_fill, sched, workspace=True)
    sta, K_s, V_s = _case(shape, max_batch, max_ctx, ctx_fill, sched, workspace=False)
    assert mk.mk_plan_workspace_bytes(sta.plan) <= mk.MK_STATIC_SCRATCH_BYTES
    a = _two_calls(ref, calls, static_scratch=False)
    assert ref.status()[0] == 0
    b = _two_calls(sta, calls, static_scratch=True)
    for (la, na), (lb, nb) in zip(a, b):
        assert (nb >= 0).all(), "a static-scratch step left next tokens unwritten"
        assert torch.equal(na, nb)
        assert torch.equal(la, lb)
    assert torch.equal(K_r, K_s) and torch.equal(V_r, V_s)


@pytest.fixture(scope="module")
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


@pytest.mark.gpu
@pytest.mark.parametrize("sched", [mk.MK_SCHED_STATIC, mk.MK_SCHED_DYNAMIC])
def test_static_scratch_matches_workspace_tiny(gpu, sched):
    # two calls in a row, the second with another batch size and contexts
    calls = [([17, 3], [0, 1], [64, 70]), ([0, 0, 511], [0, 1, 3], [65, 71, 190])]
    _compare(wl.TINY, 4, 320, [64, 70, 0, 190], calls, sched)


@pytest.mark.gpu
def test_static_scratch_matches_workspace_llama1b(gpu):
    tok = int(wl.token_ids(1, wl.LLAMA_1B.vocab)[0])
    calls = [([tok], [0], [1024]), ([tok], [0], [1025])]
    _compare(wl.LLAMA_1B, 1, 1088, [1024], calls, mk.MK_SCHED_STATIC)


@pytest.mark.gpu
def test_static_scratch_switches_back_to_an_earlier_plan(gpu):
    # plan A, then plan B, then plan A again: the scratch re-uploads A's arrays
    calls = [([5], [0], [64]), ([6], [0], [65])]
    ref, _, _ = _case(wl.TINY, 1, 256, [64], mk.MK_SCHED_STATIC, workspace=True)
    a, _, _ = _case(wl.TINY, 1, 256, [64], mk.MK_SCHED_STATIC, workspace=False)
    b, _, _ = _case(wl.TINY, 2, 320, [64, 10], mk.MK_SCHED_DYNAMIC, workspace=False)
    want = _two_calls(ref, calls, static_scratch=False)
    got_a1 = _two_calls(a, calls, static_scratch=True)
    _two_calls(b, [([7, 8], [0, 1], [64, 10])], static_scratch=True)
    # plan A's cache now holds rows from its first run; the rows it writes again are identical
    got_a2 = _two_calls(a, calls, static_scratch=True)
    for (lw, nw), (l1, n1), (l2, n2) in zip(want, got_a1, got_a2):
        assert torch.equal(nw, n1) and torch.equal(nw, n2)
        assert torch.equal(lw, l1) and torch.equal(lw, l2)


@pytest.mark.gpu
def test_static_scratch_dynamic_plans_back_to_back(gpu):
    # two dynamic plans of different max_batch (so different queue and
    # control offsets in the shared array): the larger one first, then the
    # smaller, each bitwise equal to its workspace twin
    dyn = mk.MK_SCHED_DYNAMIC
    calls_b = [([9, 10, 11], [0, 1, 2], [64, 10, 130]), ([1, 2, 3], [0, 1, 2], [65, 11, 131])]
    calls_a = [([5, 6], [0, 1], [64, 10]), ([7, 8], [0, 1], [65, 11])]
    ref_b, _, _ = _case(wl.TINY, 4, 320, [64, 10, 130, 200], dyn, workspace=True)
    ref_a, _, _ = _case(wl.TINY, 2, 256, [64, 10], dyn, workspace=True)
    sta_b, _, _ = _case(wl.TINY, 4, 320, [64, 10, 130, 200], dyn, workspace=False)
    sta_a, _, _ = _case(wl.TINY, 2, 256, [64, 10], dyn, workspace=False)
    want = _two_calls(ref_b, calls_b, static_scratch=False) + _two_calls(ref_a, calls_a, static_scratch=False)
    got = _two_calls(sta_b, calls_b, static_scratch=True) + _two_calls(sta_a, calls_a, static_scratch=True)
    for (lw, nw), (lg, ng) in zip(want, got):
        assert torch.equal(nw, ng) and torch.equal(lw, lg)
    # every entry point counts its launches
    assert sta_b.stats()["launches"] == 2 and sta_a.stats()["launches"] == 2


@pytest.mark.gpu
def test_static_scratch_rejects_a_plan_above_its_size(gpu):
    # a 32768-long context makes the rope table alone 8 MiB
    shape = wl.TINY
    K = torch.zeros(shape.n_layers, 1, shape.n_kv_heads, 32768, shape.head_dim, dtype=torch.bfloat16, device="cuda:0")
    w = {k: v.to("cuda:0") for k, v in wl.dense_weights(shape, seed=0).items()}
    dec = mk.DenseDecoder(shape, w, K, K.clone(), max_batch=1, max_ctx=32768, n_slots=1, workspace=False)
    need = mk.mk_plan_workspace_bytes(dec.plan)
    assert need > mk.MK_STATIC_SCRATCH_BYTES
    dev = "cuda:0"
    one = torch.zeros(1, dtype=torch.int32, device=dev)
    with pytest.raises(mk.MkError) as e:
        dec.step(one, one, one, one.clone(), static_scratch=True)
    assert e.value.status == mk.MK_ERR_WORKSPACE
    assert str(need) in e.value.message


def test_static_scratch_rejects_a_host_only_plan():
    # argument checks come before any CUDA call, so this runs without a GPU
    dec = mk.DenseDecoder(wl.TINY, max_batch=1, max_ctx=256, n_slots=1, host_only=True)
    a = mk.mk_step_args()
    a.batch = 1
    with pytest.raises(mk.MkError) as e:
        mk.mk_decode_step_static(dec.plan, a, 0)
    assert e.value.status == mk.MK_ERR_UNSUPPORTED
