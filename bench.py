"""Decode-step benchmark of the B200 megakernel (one JSON line on rank 0).

Workload: the Llama-1B-shaped dense decoder (16 layers, hidden 2048, 32/8
heads x 64, FFN 8192, vocab 128256, tied embeddings), bf16 N(0, 0.02)
random weights, batch 1, KV cache bf16 N(0, 1) at context 1024; each timed
step is one greedy decode step, the steps cycling through the 32-step decode
window (positions 1024..1055) with the argmax token fed back on the device.
The weights (2.47 GB) stream from HBM every step, far above the 126 MB L2,
so no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--sched static|dynamic]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

N > 1 (under torchrun) runs N independent replicas, one per GPU (the decode
step has no data-path exchange); the value is all ranks' tokens over the
slowest rank's device time.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("decode step µs & tokens/s (1B dense, B=1..64; MoE); achieved HBM GB/s vs 8 TB/s")
CTX0 = 1024
WINDOW = 32


def kernel_source_sha():
    """sha256 over the kernel sources, as recorded in the ncu summaries."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "event_tensor_task_b200", "csrc")
    files = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")) +
                   glob.glob(os.path.join(csrc, "*.h")))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def ncu_traffic(summary="megakernel_llama1b_b1_ncu.md"):
    """DRAM bytes per launch (read + write) from the committed ncu summary,
    or None when the kernel sources changed since that capture."""
    try:
        with open(os.path.join(ROOT, "profiles", summary)) as f:
            text = f.read()
    except OSError:
        return None
    import re
    sha = re.search(r"Kernel source sha256[^`]*`([0-9a-f]{64})`", text)
    tr = re.search(r"traffic: (\d+) bytes", text)
    if not sha or not tr or sha.group(1) != kernel_source_sha():
        return None
    return int(tr.group(1))


def bf16_peak():
    """Measured dense bf16 TFLOP/s (burst) of this machine's B200s, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # start timing only once the sampler is producing samples
            t0 = time.time()
            while len(self.lines) < 2 and time.time() - t0 < 10:
                time.sleep(0.05)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def setup_model(dev, seed=0):
    import torch
    import workloads as wl
    s = wl.LLAMA_1B
    w_cpu = wl.dense_weights(s, seed=seed)
    max_ctx = CTX0 + WINDOW + 32
    K_cpu, V_cpu = wl.kv_cache(s, 1, max_ctx, [CTX0], seed=seed)
    w = {k: v.to(dev, non_blocking=False) for k, v in w_cpu.items()}
    K, V = K_cpu.to(dev), V_cpu.to(dev)
    torch.cuda.synchronize()
    return s, w_cpu, w, K_cpu, V_cpu, K, V, max_ctx


class TorchPerOpDecoder:
    """Same-box comparison point: the same decode step as ordinary per-op
    PyTorch on the same bf16 weights (cuBLAS bf16 GEMV/GEMM with the q/k/v
    and gate/up weights concatenated, fp32 RMSNorm/RoPE, bf16 scaled-dot-
    product attention with a length mask over the cache padded to the
    window's last position), run eagerly or replayed as one CUDA graph.  B
    sequences in cache slots 0..B-1 start at contexts ctx0[b]; the positions
    and the greedy tokens advance on the device, so one captured graph serves
    every step of the decode window."""

    def __init__(self, s, w, K, V, max_ctx, ctx0, window, tok0, dev):
        import torch
        self.s, self.max_ctx, self.window = s, max_ctx, window
        L, D = s.n_layers, s.head_dim
        ctx0 = [int(c) for c in (ctx0 if isinstance(ctx0, (list, tuple)) else [ctx0])]
        self.B = len(ctx0)
        self.ctx0 = torch.tensor(ctx0, dtype=torch.long, device=dev)
        self.K, self.V = K.clone(), V.clone()
        self.embed = w["embed"]
        self.final_norm = w["final_norm"].float()
        self.layers = []
        for l in range(L):
            p = f"layers.{l}."
            self.layers.append({
                "attn_norm": w[p + "attn_norm"].float(), "ffn_norm": w[p + "ffn_norm"].float(),
                "wqkv": torch.cat([w[p + "wq"], w[p + "wk"], w[p + "wv"]], 0), "wo": w[p + "wo"],
                "wgu": torch.cat([w[p + "w_gate"], w[p + "w_up"]], 0), "wd": w[p + "w_down"]})
        i = torch.arange(D // 2, dtype=torch.float64)
        ang = torch.arange(max_ctx, dtype=torch.float64)[:, None] * s.rope_theta ** (-2.0 * i / D)
        self.cos, self.sin = ang.cos().float().to(dev), ang.sin().float().to(dev)
        # attention reads the cache up to the longest context of the window
        # (padded: a captured graph has static shapes), in bf16
        self.T = min(max_ctx, int(max(ctx0)) + window)
        self.keypos = torch.arange(self.T, device=dev)
        self.heads = torch.arange(s.n_kv_heads, device=dev)
        self.tok = torch.full((self.B,), tok0, dtype=torch.long, device=dev)
        self.counter = torch.zeros((), dtype=torch.long, device=dev)
        self.graph = None

    def _rms(self, x, g):
        import torch
        return x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + self.s.eps) * g

    def _rope(self, t, c, sn):
        import torch
        h = t.shape[-1] // 2
        a, b = t[..., :h], t[..., h:]
        return torch.cat([a * c - b * sn, b * c + a * sn], -1)

    def step(self):
        """One greedy decode step for the B sequences (all on the device, graph-capturable)."""
        import torch
        s, B = self.s, self.B
        Hq, Hkv, D = s.n_q_heads, s.n_kv_heads, s.head_dim
        pos = self.ctx0 + torch.remainder(self.counter, self.window)  # [B]
        c = self.cos.index_select(0, pos)[:, None, :]
        sn = self.sin.index_select(0, pos)[:, None, :]
        mask = (self.keypos[None, :] > pos[:, None])[:, None, None, :]  # keys after each new token
        rows = ((torch.arange(B, device=pos.device)[:, None] * Hkv + self.heads[None, :]) * self.max_ctx
                + pos[:, None]).reshape(-1)  # cache rows (slot b, head g, position pos_b)
        x = self.embed.index_select(0, self.tok).float()  # [B, H]
        for l, lw in enumerate(self.layers):
            h = self._rms(x, lw["attn_norm"]).to(torch.bfloat16)
            qkv = (h @ lw["wqkv"].T).float()
            q = self._rope(qkv[:, :Hq * D].view(B, Hq, D), c, sn)
            k = self._rope(qkv[:, Hq * D:(Hq + Hkv) * D].view(B, Hkv, D), c, sn)
            v = qkv[:, (Hq + Hkv) * D:].view(B, Hkv, D)
            self.K[l].view(-1, D).index_copy_(0, rows, k.to(torch.bfloat16).reshape(B * Hkv, D))
            self.V[l].view(-1, D).index_copy_(0, rows, v.to(torch.bfloat16).reshape(B * Hkv, D))
            qg = q.view(B, Hkv, Hq // Hkv, D).to(torch.bfloat16)  # the group's query heads as the query rows
            o = torch.nn.functional.scaled_dot_product_attention(
                qg, self.K[l, :B, :, :self.T], self.V[l, :B, :, :self.T], attn_mask=~mask,
                scale=1.0 / math.sqrt(D)).float().reshape(B, Hq * D)
            x = x + (o.to(torch.bfloat16) @ lw["wo"].T).float()
            h = self._rms(x, lw["ffn_norm"]).to(torch.bfloat16)
            gu = (h @ lw["wgu"].T).float()
            g, u = gu[:, :s.ffn], gu[:, s.ffn:]
            act = (g * torch.sigmoid(g) * u).to(torch.bfloat16)
            x = x + (act @ lw["wd"].T).float()
        logits = self._rms(x, self.final_norm).to(torch.bfloat16) @ self.embed.T
        self.tok.copy_(torch.argmax(logits.float(), -1))
        self.counter.add_(1)

    def capture(self):
        """Capture one step as a CUDA graph; returns the capture time in ms."""
        import torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                self.step()  # warm-up on a side stream, as graph capture requires
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        torch.cuda.synchronize()
        return 1000.0 * (time.perf_counter() - t0)

    def timed(self, n, graph):
        """Mean device ms per step over n steps (CUDA events)."""
        import torch
        run = self.graph.replay if graph else self.step
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            run()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n


def torch_baselines(s, w, K, V, max_ctx, tok0, dev, n_steps):
    """Per-op PyTorch eager and CUDA-graph decode steps on the same model."""
    base = TorchPerOpDecoder(s, w, K, V, max_ctx, CTX0, WINDOW, tok0, dev)
    eager_ms = base.timed(max(10, n_steps // 10), graph=False)
    capture_ms = base.capture()
    graph_ms = base.timed(n_steps, graph=True)
    return {"torch_eager": {"us_per_step": 1000.0 * eager_ms, "tokens_per_s": 1000.0 / eager_ms},
            "torch_cuda_graph": {"us_per_step": 1000.0 * graph_ms, "tokens_per_s": 1000.0 / graph_ms,
                                 "capture_ms": capture_ms},
            "what": "same model, weights and cache on the same GPU: per-op PyTorch (cuBLAS bf16 GEMV, "
                    "fused q/k/v and gate/up weights, masked GQA attention over the padded cache), "
                    "eager and as one captured CUDA graph; device-timed with CUDA events"}


def profile_torch():
    """Five replays of the same-box per-op PyTorch CUDA graph of the 1B B=1
    step (a short command for an ncu launch list of the baseline)."""
    import torch
    dev = "cuda:0"
    s, w_cpu, w, K_cpu, V_cpu, K, V, max_ctx = setup_model(dev)
    base = TorchPerOpDecoder(s, w, K, V, max_ctx, CTX0, WINDOW, 5, dev)
    base.capture()
    for _ in range(5):
        base.graph.replay()
    torch.cuda.synchronize()


def device_kv_cache(s, n_slots, max_ctx, ctx, dev, seed=0):
    """A bf16 N(0, 1) cache drawn on the device (seeded), zero past each
    sequence's context: the symbolic-batch sweep's 64-sequence cache is too
    large to draw on the host in a bench run (parity tests use the host
    generator on smaller cases)."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    shape = (s.n_layers, n_slots, s.n_kv_heads, max_ctx, s.head_dim)
    K = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    V = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    for l in range(s.n_layers):
        for b in range(len(ctx)):
            K[l, b, :, :ctx[b]] = torch.randn(s.n_kv_heads, ctx[b], s.head_dim, generator=gen, device=dev).to(torch.bfloat16)
            V[l, b, :, :ctx[b]] = torch.randn(s.n_kv_heads, ctx[b], s.head_dim, generator=gen, device=dev).to(torch.bfloat16)
    return K, V


def percentiles(ms_list):
    """p10 / p50 / p90 of per-step device times (ms) in us."""
    v = sorted(ms_list)
    pick = lambda q: v[min(len(v) - 1, int(q * (len(v) - 1) + 0.5))]
    return {"p10_us": 1000.0 * pick(0.1), "p50_us": 1000.0 * pick(0.5), "p90_us": 1000.0 * pick(0.9)}


def timed_steps(run, n, start):
    """Run steps start .. start + n - 1 with a CUDA event after each; returns
    (mean ms, per-step ms list)."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    ev[0].record()
    for i in range(n):
        run(1, start + i)
        ev[i + 1].record()
    torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
    return ev[0].elapsed_time(ev[n]) / n, per


def batch_sweep(s, w, dev, n_steps=100, plans=((8, (1, 2, 4, 8)), (64, (1, 2, 4, 8, 16, 32, 64)))):
    """Decode steps of the same 1B model at several batch sizes, each plan
    ONE plan and one compiled kernel for all its batch sizes (no rebuild, no
    graph capture), each sequence at its own context drawn uniform in [128,
    4096] (seeded), next to the per-op PyTorch CUDA graph captured for that
    batch size.  Plans: max_batch 8 (the small-batch GEMV path) and
    max_batch 64 (the wide-batch path: tcgen05 GEMM tasks)."""
    import torch
    import event_tensor_task_b200 as mk
    import workloads as wl
    maxB = max(mb for mb, _ in plans)
    ctx0 = [int(c) for c in wl.context_lengths(maxB, 128, 4096)]
    max_ctx = max(ctx0) + WINDOW + 32
    K, V = device_kv_cache(s, maxB, max_ctx, ctx0, dev)
    peak, _ = peaks()
    slots = torch.arange(maxB, dtype=torch.int32, device=dev)
    out = {"contexts": ctx0, "plans": []}
    graph_us = {}
    for mb, batches in plans:
        dec = mk.DenseDecoder(s, w, K, V, max_batch=mb, max_ctx=max_ctx, n_slots=maxB)
        cases = []
        for B in batches:
            ctx_tab = torch.tensor([[ctx0[b] + i for b in range(B)] for i in range(WINDOW)], dtype=torch.int32,
                                   device=dev)
            toks = torch.full((2, B), 5, dtype=torch.int32, device=dev)

            def run(n, start=0):
                for i in range(start, start + n):
                    dec.step(toks[i % 2], slots[:B], ctx_tab[i % WINDOW], toks[(i + 1) % 2])

            run(5)
            torch.cuda.synchronize()
            ms, per = timed_steps(run, n_steps, 5)
            code, _ = dec.status()
            if code != 0:
                raise SystemExit(f"device status {code} in the batch sweep (max_batch {mb}, B={B})")
            nbytes = statistics.mean(mk.mk_plan_step_bytes(dec.plan, B, [ctx0[b] + i for b in range(B)])
                                     for i in range(WINDOW))
            if B not in graph_us:
                base = TorchPerOpDecoder(s, w, K, V, max_ctx, ctx0[:B], WINDOW, 5, dev)
                base.capture()
                graph_us[B] = 1000.0 * base.timed(n_steps, graph=True)
                del base
            cases.append({"B": B, "us_per_step": 1000.0 * ms, **percentiles(per), "tokens_per_s": B / (ms / 1000.0),
                          "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                          "frac": nbytes / (ms * 1e-3) / 1e9 / peak,
                          "torch_cuda_graph_us_per_step": graph_us[B],
                          "speedup_vs_graph": graph_us[B] / (1000.0 * ms)})
        out["plans"].append({"max_batch": mb, "wide": bool(dec.tiles()["wide"]),
                             "note": "one plan and one kernel for every B of this list (no rebuild, no re-capture)",
                             "cases": cases})
        dec.close()
    return out


def profile_moe(T):
    """Four calls of the 64-expert top-8 MoE layer on T tokens (uniform routing)."""
    import torch
    import event_tensor_task_b200 as mk
    import workloads as wl
    dev = "cuda:0"
    w = {k: v.to(dev) for k, v in wl.moe_weights(wl.MOE_64x8, seed=0).items()}
    layer = mk.MoELayer(wl.MOE_64x8, w, None, max_tokens=max(T, 8))
    x = wl.moe_tokens(T, wl.MOE_64x8.hidden, seed=0).to(dev)
    out = torch.empty(T, wl.MOE_64x8.hidden, dtype=torch.bfloat16, device=dev)
    for _ in range(4):
        layer(x, out)
    torch.cuda.synchronize()
    code, _ = layer.status()
    if code != 0:
        raise SystemExit(f"MoE layer device status {code}")


def profile_wide(B):
    """Four decode steps of the 1B-shaped model at batch B through one
    max_batch 64 plan (the wide-batch path), contexts uniform in [128, 1024]
    (a profiling case: 2.5 GB of weights plus at most 2.2 GB of cache)."""
    import torch
    import event_tensor_task_b200 as mk
    import workloads as wl
    dev = "cuda:0"
    s = wl.LLAMA_1B
    w = {k: v.to(dev) for k, v in wl.dense_weights(s, seed=0).items()}
    ctx0 = [int(c) for c in wl.context_lengths(64, 128, 1024)]
    max_ctx = max(ctx0) + 32
    K, V = device_kv_cache(s, 64, max_ctx, ctx0, dev)
    dec = mk.DenseDecoder(s, w, K, V, max_batch=64, max_ctx=max_ctx, n_slots=64)
    tok = torch.full((B,), 5, dtype=torch.int32, device=dev)
    slots = torch.arange(B, dtype=torch.int32, device=dev)
    ctx = torch.tensor(ctx0[:B], dtype=torch.int32, device=dev)
    nxt = torch.empty(B, dtype=torch.int32, device=dev)
    for _ in range(4):
        dec.step(tok, slots, ctx, nxt)
    torch.cuda.synchronize()
    code, _ = dec.status()
    if code != 0:
        raise SystemExit(f"wide-batch step device status {code}")


def moe_decoder_bench(dev, n_steps=64):
    """The MoE decoder: 16 layers with the 1B attention shape, each FFN the
    64-expert top-8 layer (F 1408), vocab 128256, tied embeddings; Zipf(1.2)
    skewed routing; dynamic schedule; continuous batching with the batch
    size drawn per step from {1, ..., 128} (one plan of max_batch 128: the
    wide-batch attention half and LM head) and contexts starting uniform in
    [256, 4096].  Its 17.7 GB of expert weights
    are drawn on the device (N(0, 0.02) bf16 from a seeded generator): this
    leg times the path; parity is tested on a two-layer model whose weights
    come from the seeded host generators."""
    import torch
    import event_tensor_task_b200 as mk
    import workloads as wl
    s = wl.DenseShape(n_layers=16, hidden=2048, n_q_heads=32, n_kv_heads=8, head_dim=64, ffn=8192, vocab=128256)
    ms = wl.MOE_64x8
    H, D, L = s.hidden, s.head_dim, s.n_layers
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)

    def rnd(*shape):
        return (torch.randn(*shape, generator=gen, device=dev) * 0.02).to(torch.bfloat16)

    w = {"embed": rnd(s.vocab, H), "final_norm": torch.ones(H, dtype=torch.bfloat16, device=dev)}
    mlayers = []
    for l in range(L):
        p = f"layers.{l}."
        w[p + "attn_norm"] = torch.ones(H, dtype=torch.bfloat16, device=dev)
        w[p + "ffn_norm"] = torch.ones(H, dtype=torch.bfloat16, device=dev)
        w[p + "wq"], w[p + "wk"], w[p + "wv"] = rnd(32 * D, H), rnd(8 * D, H), rnd(8 * D, H)
        w[p + "wo"] = rnd(H, 32 * D)
        mlayers.append({"router": rnd(ms.n_experts, H), "w_gate": rnd(ms.n_experts, ms.expert_ffn, H),
                        "w_up": rnd(ms.n_experts, ms.expert_ffn, H), "w_down": rnd(ms.n_experts, H, ms.expert_ffn)})
    bias = wl.zipf_bias(ms.n_experts).to(dev)
    maxB = 128
    ctx0 = [int(c) for c in wl.context_lengths(maxB, 256, 4096, stream="moe-decoder-ctx")]
    max_ctx = max(ctx0) + n_steps + 16
    K = torch.zeros(L, maxB, s.n_kv_heads, max_ctx, D, dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    for b in range(maxB):
        K[:, b, :, :ctx0[b]] = torch.randn(L, s.n_kv_heads, ctx0[b], D, generator=gen, device=dev).to(torch.bfloat16)
        V[:, b, :, :ctx0[b]] = torch.randn(L, s.n_kv_heads, ctx0[b], D, generator=gen, device=dev).to(torch.bfloat16)
    dec = mk.DenseDecoder(s, w, K, V, max_batch=maxB, max_ctx=max_ctx, n_slots=maxB, moe=(ms, mlayers, bias))
    sched = wl.batch_schedule(n_steps + 3, list(range(1, maxB + 1)))
    ran = [0] * maxB
    args = []
    for i, B in enumerate(sched):
        ctx = [ctx0[b] + ran[b] for b in range(B)]
        for b in range(B):
            ran[b] += 1
        args.append((torch.full((B,), 7, dtype=torch.int32, device=dev), torch.arange(B, dtype=torch.int32, device=dev),
                     torch.tensor(ctx, dtype=torch.int32, device=dev), torch.empty(B, dtype=torch.int32, device=dev)))
    for a in args[:3]:
        dec.step(*a)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_steps + 1)]
    ev[0].record()
    for i, a in enumerate(args[3:]):
        dec.step(*a)
        ev[i + 1].record()
    torch.cuda.synchronize()
    code, _ = dec.status()
    if code != 0:
        raise SystemExit(f"MoE decoder device status {code}")
    per = {}
    step_ms = []
    for i, B in enumerate(sched[3:]):
        per.setdefault(B, []).append(ev[i].elapsed_time(ev[i + 1]))
        step_ms.append(ev[i].elapsed_time(ev[i + 1]))
    total_ms = ev[0].elapsed_time(ev[-1])
    tokens = sum(sched[3:])
    # algorithmic bytes of each timed step from its run-time routing: the
    # steps are replayed (same inputs, so the same cache rows and routing) with
    # the per-layer histogram captured, and each layer reads its router and
    # the experts its histogram touched (17.3 MB each)
    E, F = ms.n_experts, ms.expert_ffn
    attn_w = L * ((32 + 2 * 8) * D * H + H * 32 * D) * 2.0
    lm = s.vocab * H * 2.0
    nbytes = []
    hist = torch.empty(L, E, dtype=torch.int32, device=dev)
    for i, a in enumerate(args[3:]):
        B = sched[3 + i]
        dec.step(*a, capture={"hist": hist})
        torch.cuda.synchronize()
        touched = int((hist > 0).sum())
        ctx_sum = float(a[2].sum())
        nbytes.append(attn_w + lm + L * E * H * 2.0 + touched * 3.0 * F * H * 2.0 + B * H * 2.0 +
                      L * s.n_kv_heads * D * 2 * 2.0 * (ctx_sum + B))
    code, _ = dec.status()
    if code != 0:
        raise SystemExit(f"MoE decoder device status {code} in the byte replay")
    peak, _ = peaks()
    achieved = statistics.mean(nbytes) / (total_ms / n_steps * 1e-3) / 1e9
    dec.close()
    buckets = {}
    for B, v in per.items():
        key = "1-8" if B <= 8 else "9-32" if B <= 32 else "33-64" if B <= 64 else "65-128"
        buckets.setdefault(key, []).extend(v)
    return {"workload": "MoE decoder: 16 layers (1B attention shape), 64 experts top-8 F 1408 per layer, vocab 128256, "
                        "Zipf(1.2) routing, dynamic schedule, B per step from {1..128}, contexts from U[256,4096]",
            "us_per_step_by_B_bucket": {k: 1000.0 * statistics.mean(v) for k, v in sorted(buckets.items())},
            "steps": n_steps, "tokens": tokens, "tokens_per_s": tokens / (total_ms / 1000.0),
            "us_per_step": 1000.0 * total_ms / n_steps,

            **percentiles(step_ms),
            "algorithmic_bytes_per_step": statistics.mean(nbytes), "achieved_gbs": achieved, "frac": achieved / peak,
            "bytes_rule": "attention and router weights + the experts each layer's run-time histogram touched "
                          "(3 x 1408 x 2048 bf16 each) + LM head + KV reads and appends + embedding rows",
            "weights": "device-drawn N(0,0.02) bf16 (seeded); parity is tested on a two-layer model"}


def moe_layer_bench(dev, n_iter=10):
    """The MoE FFN layer (64 experts, top-8, F 1408, hidden 2048) for
    T in {1, 8, 64, 512} with uniform and Zipf(1.2)-skewed routing: device
    time per layer call (CUDA events around each call, L2 flushed before
    it), and the HBM roofline of the bytes the call must read (router, the
    distinct experts the routing touched, the tokens in and out)."""
    import torch
    import event_tensor_task_b200 as mk
    import workloads as wl
    shape = wl.MOE_64x8
    H, E, K, F = shape.hidden, shape.n_experts, shape.top_k, shape.expert_ffn
    w = {k: v.to(dev) for k, v in wl.moe_weights(shape, seed=0).items()}
    bias = wl.zipf_bias(E).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # twice the L2
    peak, peak_kind = peaks()
    cases = []
    def timed_call(layer, x, out, hist):
        for _ in range(3):
            layer(x, out, hist=hist)
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(n_iter):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            layer(x, out, hist=hist)
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        code, _ = layer.status()
        if code != 0:
            raise SystemExit(f"MoE layer device status {code}")
        return 1000.0 * total / n_iter

    for regime, b in (("uniform", None), ("zipf", bias)):
        layer = mk.MoELayer(shape, w, b, max_tokens=512)
        fixed = mk.MoELayer(shape, w, b, max_tokens=512, moe_tiles=2)  # (fixed 64-row tiles, for comparison)
        for T in (1, 8, 64, 512):
            x = wl.moe_tokens(T, H, seed=0).to(dev)
            out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
            hist = torch.empty(E, dtype=torch.int32, device=dev)
            us_fixed = timed_call(fixed, x, out, hist)
            us = timed_call(layer, x, out, hist)
            touched = int((hist.cpu() > 0).sum())
            nbytes = E * H * 2 + touched * 3 * F * H * 2 + 2 * T * H * 2
            gbs = nbytes / (us * 1e-6) / 1e9
            flops = 2.0 * T * K * 3 * F * H  # the GroupGEMM: (gate, up, down) x every routed row
            tfs = flops / (us * 1e-6) / 1e12
            cases.append({"T": T, "routing": regime, "us_per_layer": us, "us_fixed_64_row_tiles": us_fixed,
                          "experts_touched": touched,
                          "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "frac": gbs / peak,
                          "groupgemm_tflops": tfs, "frac_of_bf16_peak": tfs / bf16_peak()})
        layer.close()
        fixed.close()
    return {"workload": "MoE FFN layer: hidden 2048, 64 experts, top-8, expert FFN 1408, bf16 N(0,0.02) weights, "
                        "x ~ N(0,1) bf16; L2 flushed before every timed call",
            "peak_gbs": peak, "peak_kind": peak_kind, "cases": cases}


def interpreter_bench(s, w, K, V, max_ctx, dev, n_steps=200):
    """The interpreter alone: the 1B plan at B=1 (context 1024) with empty
    tasks (MK_DEBUG_EMPTY_TASKS: every task keeps its events, waits,
    notifies and queue pushes, but streams no data and runs no body), static
    and dynamic schedule.  Reports the step time, the dispatch rate (tasks
    per microsecond over the whole GPU) and, from one traced step, the
    notify -> wait latency between SMs: per dependency hop of a layer, the
    first consumer's event-ready time minus the last producer's notify time."""
    import collections
    import torch
    import event_tensor_task_b200 as mk
    from event_tensor_task_b200 import trace as mtr
    out = {}
    hops = (("qkv", "attn"), ("merge", "oproj"), ("oproj", "gateup"), ("gateup", "down"))
    for name, sched in (("static", mk.MK_SCHED_STATIC), ("dynamic", mk.MK_SCHED_DYNAMIC)):
        dec = mk.DenseDecoder(s, w, K, V, max_batch=1, max_ctx=max_ctx, n_slots=1, sched=sched, empty_tasks=True,
                              trace=True)
        tok = torch.full((1,), 5, dtype=torch.int32, device=dev)
        slot = torch.zeros(1, dtype=torch.int32, device=dev)
        ctx = torch.tensor([CTX0], dtype=torch.int32, device=dev)
        nxt = torch.empty(1, dtype=torch.int32, device=dev)

        def run(n, start=0):
            for _ in range(n):
                dec.step(tok, slot, ctx, nxt)

        run(5)
        torch.cuda.synchronize()
        ms, per = timed_steps(run, n_steps, 0)
        tr = torch.zeros(148, 400, 16, dtype=torch.int32, device=dev)
        dec.step(tok, slot, ctx, nxt, trace=tr)
        torch.cuda.synchronize()
        code, _ = dec.status()
        if code != 0:
            raise SystemExit(f"device status {code} in the interpreter bench")
        recs = mtr.records(tr, [f.name.decode() for f in dec.families()])
        byfam = collections.defaultdict(list)
        for r in recs:
            byfam[r["family"]].append(r)
        lat = []
        for l in range(s.n_layers):
            for a, b in hops:
                prod = [r["notified"] for r in byfam.get(f"{a}.{l}", []) if r["notified"] is not None]
                cons = [r["ready"] for r in byfam.get(f"{b}.{l}", []) if r["ready"] is not None]
                if prod and cons:
                    lat.append((min(cons) - max(prod)) / 1000.0)
        out[name] = {"us_per_step": 1000.0 * ms, **percentiles(per), "tasks_per_step": len(recs),
                     "tasks_per_us": len(recs) / (1000.0 * ms),
                     "notify_to_ready_us": {"median": statistics.median(lat) if lat else None,
                                            "max": max(lat) if lat else None, "hops": len(lat)}}
        dec.close()
    return out


def cpu_oracle_rate(s, w_cpu, K_cpu, V_cpu, n_steps, n_warm=1):
    """The oracle as it stands: tokens/s over n_steps decode steps after
    n_warm untimed warm-up steps (the first also widens the weights to fp64
    once)."""
    import torch
    import oracle
    import workloads as wl
    o = oracle.DenseOracle(s, w_cpu)
    K, V = K_cpu.clone(), V_cpu.clone()
    tok = int(wl.token_ids(1, s.vocab)[0])
    for i in range(max(1, n_warm)):
        r = o.step(K, V, [tok], [0], [CTX0 + i])
        tok = int(r["next_tokens"][0])
    t0 = time.perf_counter()
    for i in range(n_steps):
        r = o.step(K, V, [tok], [0], [CTX0 + max(1, n_warm) + i])
        tok = int(r["next_tokens"][0])
    dt = time.perf_counter() - t0
    return n_steps / dt, torch.get_num_threads(), dt


def max_over_ranks(x, device):
    """Max of x over the ranks of the default process group (x itself when no
    group is initialised): the timed region of a multi-GPU run is the slowest
    rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, items_per_rank, max_ms):
    """Items per second over all ranks (replicas: every rank does the same
    work) for a timed region of max_ms, the max over ranks."""
    return world * items_per_rank / (max_ms / 1000.0)


def run_reference(args, rank):
    if rank != 0:
        return
    import torch
    import workloads as wl
    s = wl.LLAMA_1B
    w_cpu = wl.dense_weights(s)
    K_cpu, V_cpu = wl.kv_cache(s, 1, CTX0 + WINDOW + 32, [CTX0])
    n = max(1, min(args.steps, 4))
    warm = max(1, min(args.warmup, 3))  # (each oracle step is ~0.1 s of host work)
    rate, cores, dt = cpu_oracle_rate(s, w_cpu, K_cpu, V_cpu, n, warm)
    sample = (f"{n} full decode steps of the 1B model (B=1, positions {CTX0 + warm}..{CTX0 + warm + n - 1}) "
              f"after {warm} untimed warm-up step(s); fp64 CPU oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": n, "warmup": warm, "ms_per_step": 1000.0 * dt / n, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args),
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(args):
    return {"workload": "llama-1b-shaped dense decode (16L, hidden 2048, 32q/8kv x 64, ffn 8192, vocab 128256, "
                        "tied), greedy 32-step window from context 1024",
            "batch": 1, "ctx": f"{CTX0}..{CTX0 + WINDOW - 1}", "sched": args.sched,
            "l2": "2.5 GB weights streamed per step > 126 MB L2; no flush",
            "parallelism": "replicas" if args.gpus > 1 else "single-gpu"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--sched", default="static", choices=["static", "dynamic"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-torch-baseline", action="store_true")
    ap.add_argument("--no-moe", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-moe-decoder", action="store_true")
    ap.add_argument("--no-interp", action="store_true")
    ap.add_argument("--profile-moe", type=int, default=0, metavar="T",
                    help="only run 4 MoE-layer calls on T tokens (a short command for ncu) and exit")
    ap.add_argument("--profile-wide", type=int, default=0, metavar="B",
                    help="only run 4 wide-batch 1B decode steps at batch B (a short command for ncu) and exit")
    ap.add_argument("--profile-torch", action="store_true",
                    help="only replay the per-op PyTorch CUDA graph of the B=1 step 5 times (for ncu) and exit")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.profile_moe:
        profile_moe(args.profile_moe)
        return
    if args.profile_wide:
        profile_wide(args.profile_wide)
        return
    if args.profile_torch:
        profile_torch()
        return

    import torch
    import torch.distributed as dist
    import event_tensor_task_b200 as mk

    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device(dev))

    s, w_cpu, w, K_cpu, V_cpu, K, V, max_ctx = setup_model(dev)
    sched = mk.MK_SCHED_STATIC if args.sched == "static" else mk.MK_SCHED_DYNAMIC
    dec = mk.DenseDecoder(s, w, K, V, max_batch=1, max_ctx=max_ctx, n_slots=1, sched=sched)
    stream = torch.cuda.current_stream()

    import workloads as wl
    tok0 = int(wl.token_ids(1, s.vocab)[0])
    ctx_tab = torch.arange(CTX0, CTX0 + WINDOW, dtype=torch.int32, device=dev)
    slot = torch.zeros(1, dtype=torch.int32, device=dev)
    toks = torch.full((2,), tok0, dtype=torch.int32, device=dev)  # ping-pong greedy tokens

    def run(n, start=0):
        for i in range(start, start + n):
            a, b = toks[i % 2: i % 2 + 1], toks[(i + 1) % 2: (i + 1) % 2 + 1]
            dec.step(a, slot, ctx_tab[i % WINDOW: i % WINDOW + 1], b)

    run(args.warmup)
    torch.cuda.synchronize()
    code, st = dec.status()
    if code != 0:
        raise SystemExit(f"device status {code} after warm-up (family {st.family} index {st.index})")

    # ---- device-timed region: K steps, inputs resident in HBM (an event
    # after every step gives the per-step percentiles)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(torch.cuda.current_device() if world == 1 else local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        evs[0].record(stream)
        for i in range(args.steps):
            run(1, args.warmup + i)
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ms = evs[0].elapsed_time(evs[-1])
    step_pct = percentiles([evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)])
    code, st = dec.status()
    if code != 0:
        raise SystemExit(f"device status {code} in the timed region")
    ms = max_over_ranks(ms, dev)
    ms_step = ms / args.steps
    value = whole_job_rate(world, 1 * args.steps, ms)

    # algorithmic bytes per launch (mean over the context window)
    step_bytes = statistics.mean(mk.mk_plan_step_bytes(dec.plan, 1, [CTX0 + (i % WINDOW)])
                                 for i in range(WINDOW))
    peak, peak_kind = peaks()
    achieved = step_bytes / (ms_step / 1000.0) / 1e9

    # ---- end to end through the public API with host buffers
    h_in = torch.empty(3, dtype=torch.int32, pin_memory=True)
    h_out = torch.empty(1, dtype=torch.int32, pin_memory=True)
    d_in = torch.empty(3, dtype=torch.int32, device=dev)
    d_out = torch.empty(1, dtype=torch.int32, device=dev)
    tok = tok0
    n_e2e = min(args.steps, 1000)

    def e2e_steps(n, start):
        nonlocal tok
        for i in range(start, start + n):
            h_in[0], h_in[1], h_in[2] = tok, 0, CTX0 + (i % WINDOW)
            d_in.copy_(h_in, non_blocking=True)
            dec.step(d_in[0:1], d_in[1:2], d_in[2:3], d_out)
            h_out.copy_(d_out, non_blocking=True)
            stream.synchronize()
            tok = int(h_out[0])

    e2e_steps(args.warmup, 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_steps(n_e2e, args.warmup)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = whole_job_rate(world, n_e2e, e_ms)

    baselines = None
    if world == 1 and not args.no_torch_baseline:
        baselines = torch_baselines(s, w, K, V, max_ctx, tok0, dev, min(args.steps, 500))
        t0 = time.perf_counter()
        tmp = mk.DenseDecoder(s, w, K, V, max_batch=1, max_ctx=max_ctx, n_slots=1, sched=sched)
        torch.cuda.synchronize()
        baselines["megakernel_plan_build_and_bind_ms"] = 1000.0 * (time.perf_counter() - t0)
        tmp.close()

    interp = None
    if world == 1 and not args.no_interp:
        interp = interpreter_bench(s, w, K, V, max_ctx, dev)
    moe = None
    if world == 1 and not args.no_moe:
        moe = moe_layer_bench(dev)
    sweep = None
    if world == 1 and not args.no_sweep:
        sweep = batch_sweep(s, w, dev)
    moe_dec = None
    if world == 1 and not args.no_moe_decoder:
        moe_dec = moe_decoder_bench(dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, dt = cpu_oracle_rate(s, w_cpu, K_cpu, V_cpu, 2)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": "2 full decode steps of the 1B model (B=1, ctx 1025, 1026) after one untimed "
                         "warm-up step; fp64 CPU oracle"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    if baselines:  # the baselines' rate on the same algorithmic bytes as the headline step
        for k in ("torch_eager", "torch_cuda_graph"):
            baselines[k]["achieved_gbs"] = step_bytes / (baselines[k]["us_per_step"] * 1e-6) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "us_per_step": 1000.0 * ms_step, **step_pct,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) KV cache)", "config": workload_config(args),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": ncu_traffic(), "peak_kind": peak_kind,
                     "frac_of_8tbs": achieved / 8000.0, "bytes_per_launch": step_bytes},
        "cpu_baseline": cpu,
        "torch_baselines": baselines,
        "moe_layer": moe,
        "batch_sweep": sweep,
        "moe_decoder": moe_dec,
        "interpreter": interp,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": 12, "d2h_bytes_per_step": 4},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
