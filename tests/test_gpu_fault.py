"""Failure detection on the GPU without a GPU fault (bounded device waits).

A host-built plan arms one event with a wait count one above the number of
notifies it will get (the plan simulator's COUNT_PLUS_ONE fault, lowered to
the device plan through mk_plan_opts.fault).  The tasks that wait on it spin
until the plan's spin-wait limit (5 ms here): the kernel records
MK_ERR_DEVICE_TIMEOUT in its status word, raises the abort flag that every
spin polls, drains its in-flight copies and exits, so the launch ends and
the CUDA context stays usable.  No trap, no endless loop, no bad address.
"""
import pytest
import torch

import event_tensor_task_b200 as mk
import workloads as wl
from gpu_common import DenseCase, rel_err, TOL

def _family(shape, name):
    probe = mk.DenseDecoder(shape, max_batch=1, max_ctx=320, n_slots=1, host_only=True)
    names = [f.name.decode() for f in probe.families()]
    probe.close()
    return names.index(name), names


@pytest.mark.gpu
@pytest.mark.parametrize("sched", [mk.MK_SCHED_STATIC, mk.MK_SCHED_DYNAMIC])
def test_unmet_event_times_out_and_context_survives(sched):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    fam, names = _family(wl.TINY, "gateup.0")
    bad = DenseCase(wl.TINY, max_batch=1, max_ctx=320, n_slots=1, ctx_fill=[64], sched=sched, debug=False,
                    spin_timeout_ns=5_000_000, fault=mk.MK_SIM_FAULT_COUNT_PLUS_ONE, fault_family=fam)
    dev = "cuda:0"
    one = lambda v: torch.tensor([v], dtype=torch.int32, device=dev)
    for attempt in range(2):
        nxt = torch.full((1,), -1, dtype=torch.int32, device=dev)
        bad.dec.step(one(17), one(0), one(64), nxt)
        torch.cuda.synchronize()  # the launch ends: every wait is bounded
        code, st = bad.dec.status()
        assert code == mk.MK_ERR_DEVICE_TIMEOUT, (attempt, code)
        assert 0 <= st.sm < 148
        # the task that gave up waits downstream of the unmet event (or is the
        # queue / a barrier of the same stalled step)
        assert st.family == -1 or names[st.family].split(".")[0] in ("down", "qkv", "lm", "oproj", "gateup",
                                                                      "attn"), names[st.family]
        assert int(nxt.cpu()[0]) == -1, "a step stopped by a timeout must not publish a token"
        bad.dec.reset()
        assert bad.dec.status()[0] == mk.MK_OK
    # the context is usable: a clean plan on the same device steps correctly
    good = DenseCase(wl.TINY, max_batch=1, max_ctx=320, n_slots=1, ctx_fill=[64], sched=sched)
    K, V = good.K_cpu.clone(), good.V_cpu.clone()
    ref = good.oracle.step(K, V, [17], [0], [64])
    got = good.gpu_step([17], [0], [64])
    assert rel_err(got["logits"], ref["logits"]) <= TOL


def test_fault_option_is_checked_on_the_host():
    # a family whose notified event depends on the step's symbols is refused
    fam, _ = _family(wl.TINY, "attn.0")
    with pytest.raises(mk.MkError) as e:
        mk.DenseDecoder(wl.TINY, max_batch=1, max_ctx=320, n_slots=1, host_only=True,
                        fault=mk.MK_SIM_FAULT_COUNT_PLUS_ONE, fault_family=fam)
    assert e.value.status == mk.MK_ERR_INVALID_ARG
