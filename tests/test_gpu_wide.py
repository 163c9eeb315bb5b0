"""GPU parity of the wide-batch path (max_batch > 8) against the CPU oracle.

Above 8 batch rows one plan runs the wide-batch layout: NORM tasks
materialise the residual and the normalised bf16 activations, every
projection is a tcgen05 GEMM task (128 weight rows x the batch, fp32
accumulators in tensor memory), and an attention task streams up to
attn_split key chunks with an online softmax.  One plan and one kernel serve
every B from 1 to max_batch (symbolic batch and contexts).  Up to 64 rows
the activations are stored as bf16 value + bf16 remainder rows, multiplied
in one MMA and added in the epilogue.  Checked through
the C ABI on cuda:0: logits and the residual after every layer within max
|gpu - oracle| <= 2e-2 * max |oracle|, greedy tokens (up to near ties), the
task set exactly, every event counter at zero.
"""
import pytest
import torch

import event_tensor_task_b200 as mk
import workloads as wl
from gpu_common import DenseCase, rel_err, check_argmax, TOL

pytestmark = pytest.mark.gpu


def _check(case, tokens, slots, ctx, K, V, hidden=True):
    ref = case.oracle.step(K, V, tokens, slots, ctx, capture=hidden)
    got = case.gpu_step(tokens, slots, ctx, capture=hidden)
    for b in range(len(tokens)):
        assert rel_err(got["logits"][b], ref["logits"][b]) <= TOL, f"row {b}"
        check_argmax(got["next_tokens"][b], ref["logits"][b])
    if hidden:
        case.check_hidden(got, ref)
    case.check_task_set(got["task_counts"], len(tokens), ctx)
    return ref


@pytest.mark.parametrize("sched,split", [(mk.MK_SCHED_STATIC, 0), (mk.MK_SCHED_DYNAMIC, 0),
                                         (mk.MK_SCHED_STATIC, 2)])
def test_tiny_wide_batch_symbolic_shapes(sched, split):
    # one plan (max_batch 16): B = 16, 9, 1, 12 and 4 with ragged contexts, the
    # oracle's cache following the appends; activations as value + remainder
    # rows (default) and as plain bf16 rows.  The steps of at most 8 rows take
    # the per-step attention split (B = 4 at these contexts: 3 chunks per task,
    # so three of its (sequence, kv head) pairs have 2 tasks and a merge)
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    fill = [64, 0, 70, 190, 5, 127, 128, 300, 1, 2, 255, 33, 64, 65, 129, 200]
    case = DenseCase(wl.TINY, max_batch=16, max_ctx=320, n_slots=16, ctx_fill=fill, sched=sched, act_split=split)
    assert case.dec.tiles()["wide"] == 1 and case.dec.tiles()["act_split"] == (split != 2)
    K, V = case.K_cpu.clone(), case.V_cpu.clone()
    tok = wl.token_ids(16, wl.TINY.vocab).tolist()
    steps = [(tok, list(range(16)), fill),
             (tok[:9], [15, 1, 3, 0, 5, 7, 2, 9, 11], [201, 1, 191, 65, 128, 301, 71, 3, 34]),
             (tok[:1], [6], [128]),
             (tok[:12], list(range(12)), [65, 2, 72, 192, 6, 129, 129, 302, 3, 4, 256, 35]),
             (tok[:4], [0, 7, 10, 15], [66, 303, 257, 202])]
    for tokens, slots, ctx in steps:
        _check(case, tokens, slots, ctx, K, V)


def test_llama1b_wide_batch_16_32_64():
    # the symbolic-batch workload: one plan (max_batch 64) and one kernel for
    # B = 16, 32 and 64, contexts drawn uniform in [128, 4096]
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    ctx = [int(c) for c in wl.context_lengths(64, 128, 4096)]
    case = DenseCase(wl.LLAMA_1B, max_batch=64, max_ctx=4160, n_slots=64, ctx_fill=ctx)
    K, V = case.K_cpu.clone(), case.V_cpu.clone()
    tok = wl.token_ids(64, wl.LLAMA_1B.vocab).tolist()
    for B in (16, 32, 64):
        # sequence b continues at its own position (earlier steps appended rows)
        step_ctx = [ctx[b] + (B > 16) * (b < 16) + (B > 32) * (b < 32) for b in range(B)]
        _check(case, tok[:B], list(range(B)), step_ctx, K, V, hidden=(B == 64))
