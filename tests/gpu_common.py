"""Shared helpers of the GPU parity tests: build a decoder on cuda:0 from the
seeded workloads, run steps through the C ABI, compare with the oracle."""
import torch

import event_tensor_task_b200 as mk
import workloads as wl
from oracle import tasks as ot

TOL = 2e-2  # max |gpu - ref| <= TOL * max |ref| per compared tensor


def rel_err(got, ref):
    """max |got - ref| / max |ref| (recorded for the session's margin report)."""
    from conftest import record_margin
    got = got.double().cpu()
    ref = ref.double().cpu()
    e = float((got - ref).abs().max() / ref.abs().max().clamp_min(1e-30))
    record_margin(e)
    return e


def counters_at_zero(dec):
    """Every Event Tensor counter of the plan reads zero after a finished step."""
    ctr = dec.counters().cpu()
    nz = torch.nonzero(ctr).flatten().tolist()
    assert not nz, f"{len(nz)} event counters not at zero after the step (first {nz[:5]}: {ctr[nz[:5]].tolist()})"


def to_dev(w, dev="cuda:0"):
    return {k: v.to(dev) for k, v in w.items()}


class DenseCase:
    """Weights, cache and a plan for one dense shape, plus its oracle."""

    def __init__(self, shape, max_batch, max_ctx, n_slots, ctx_fill, sched=mk.MK_SCHED_STATIC,
                 debug=True, seed=0, **tiles):
        import oracle
        self.shape = shape
        self.w_cpu = wl.dense_weights(shape, seed=seed)
        self.K_cpu, self.V_cpu = wl.kv_cache(shape, n_slots, max_ctx, ctx_fill, seed=seed)
        self.w = to_dev(self.w_cpu)
        self.K = self.K_cpu.to("cuda:0")
        self.V = self.V_cpu.to("cuda:0")
        self.dec = mk.DenseDecoder(shape, self.w, self.K, self.V, max_batch=max_batch, max_ctx=max_ctx,
                                   n_slots=n_slots, sched=sched, debug=debug, **tiles)
        self.oracle = oracle.DenseOracle(shape, self.w_cpu)

    def tiles_for_oracle(self):
        t = self.dec.tiles()
        return dict(tile_qkv=t["tile_qkv"], chunk=t["chunk"], tile_o=t["tile_o"], tile_gu=t["tile_gu"],
                    tile_down=t["tile_down"], kseg=t["kseg"], tile_lm=t["tile_lm"], split=t["attn_split"],
                    split_auto=bool(t["attn_auto"]), n_sm=t["n_sm"], wide=bool(t["wide"]),
                    gseg=(t["gseg_qkv"], t["gseg_o"], t["gseg_gu"]))

    def gpu_step(self, tokens, slots, ctx, with_logits=True, counts=True, capture=False):
        """One step through mk_decode_step; with ``capture`` also the residual
        after every layer.  Checks the device status and that every event
        counter ended at zero."""
        dev = "cuda:0"
        B = len(tokens)
        cap = None
        if capture:
            cap = {"resid": torch.full((self.shape.n_layers, B, self.shape.hidden), float("nan"), device=dev)}
        tok = torch.tensor(tokens, dtype=torch.int32, device=dev)
        sl = torch.tensor(slots, dtype=torch.int32, device=dev)
        cx = torch.tensor(ctx, dtype=torch.int32, device=dev)
        nxt = torch.full((B,), -1, dtype=torch.int32, device=dev)
        logits = torch.empty(B, self.shape.vocab, dtype=torch.float32, device=dev) if with_logits else None
        tc = torch.zeros(mk.mk_plan_task_slots(self.dec.plan), dtype=torch.int32, device=dev) if counts else None
        self.dec.step(tok, sl, cx, nxt, logits=logits, task_counts=tc, capture=cap)
        torch.cuda.synchronize()
        code, st = self.dec.status()
        assert code == 0, f"device status {code} family {st.family} index {st.index} event {st.event}"
        counters_at_zero(self.dec)
        return {"next_tokens": nxt.cpu(), "logits": None if logits is None else logits.cpu(),
                "task_counts": None if tc is None else tc.cpu(),
                "resid": None if cap is None else cap["resid"].cpu()}

    def check_hidden(self, got, ref):
        """The residual after every layer against the oracle's captures."""
        for l in range(self.shape.n_layers):
            for b in range(got["resid"].shape[1]):
                assert rel_err(got["resid"][l, b], ref["residual"][l][b]) <= TOL, f"layer {l} row {b}"

    def check_task_set(self, counts, B, ctx):
        """Every task of the step ran exactly once; nothing else ran."""
        want = ot.expected_dense_tasks(self.shape, B, ctx, self.tiles_for_oracle())
        got = set()
        for f in self.dec.families():
            name = f.name.decode()
            fam, _, layer = name.partition(".")
            layer = int(layer) if layer else -1
            seg = counts[f.debug_base:f.debug_base + f.max_extent]
            assert int(seg.max()) <= 1, f"{name}: a task ran more than once"
            for i in torch.nonzero(seg).flatten().tolist():
                got.add((fam, layer, i))
        assert got == want, (len(got), len(want), sorted(want - got)[:5], sorted(got - want)[:5])


def check_argmax(gpu_tok, ref_logits, tol=TOL):
    """The GPU token is the oracle's argmax, or within the near-tie margin of it."""
    ref = ref_logits.double()
    best = int(torch.argmax(ref))
    if int(gpu_tok) == best:
        return True
    margin = float(ref[best] - ref[int(gpu_tok)])
    assert margin <= tol * float(ref.abs().max()), f"token {int(gpu_tok)} vs {best}, margin {margin}"
    from conftest import record_margin
    record_margin(near_tie=True)
    return False
