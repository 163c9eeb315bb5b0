"""MoE FFN layer: router, top-k, expert histogram, exp_indptr, experts, combine.

Test infrastructure only.  Follows "Event Tensor: A Unified Abstraction for
Compiling Dynamic Megakernel", section "Core method" (data-dependent
dynamism): the runtime top-k decides which expert each (token, slot) pair is
grouped under, and the exclusive prefix sum ``exp_indptr`` of the per-expert
counts decides how many GroupGEMM tiles each expert triggers.

The router logits decide an integer result (the expert ids), so they are
computed in the kernel's precision, fp32, in one fixed order:

* lane ``l`` of a 32-lane group accumulates the products at hidden indices
  ``k = 256*i + 8*l + j`` for ``i = 0, 1, ...`` (outer) and ``j = 0..7``
  (inner), one rounding per addition, starting from +0;
* the 32 lane sums are then combined by a butterfly: for ``s = 16, 8, 4, 2,
  1`` every lane adds the value of lane ``l xor s``; lane 0 holds the logit;
* the router bias (zero, or the skewed-routing prior) is added last, in fp32.

Every product of two bf16 numbers is exact in fp32 (8-bit significands), so
this order fixes the logits bit for bit.  Everything after the selection
(softmax weights, experts, combine) is fp64.
"""
from __future__ import annotations

import torch

from .dense import swiglu, F64

LANES = 32
VEC = 8


def router_logits(x_bf16: torch.Tensor, w_router_bf16: torch.Tensor,
                  bias_f32: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 router logits ``[T, E]`` in the fixed summation order above."""
    T, H = x_bf16.shape
    E = w_router_bf16.shape[0]
    assert H % (LANES * VEC) == 0, "hidden size must be a multiple of 256"
    xf = x_bf16.to(torch.float32)
    wf = w_router_bf16.to(torch.float32)
    n_outer = H // (LANES * VEC)
    # products [T, E, i, l, j]; each product is exact in fp32
    prod = (xf[:, None, :] * wf[None, :, :]).view(T, E, n_outer, LANES, VEC)
    acc = torch.zeros(T, E, LANES, dtype=torch.float32)
    for i in range(n_outer):
        for j in range(VEC):
            acc = acc + prod[:, :, i, :, j]
    lane = torch.arange(LANES)
    for s in (16, 8, 4, 2, 1):
        acc = acc + acc[:, :, lane ^ s]
    logits = acc[:, :, 0].contiguous()
    if bias_f32 is not None:
        logits = logits + bias_f32.to(torch.float32)[None, :]
    return logits


def topk_route(logits_f32: torch.Tensor, k: int):
    """Top-k experts per token and their weights.

    Experts are ordered by logit, largest first; equal logits order by the
    lower expert id.  The weights are the softmax of the ``k`` selected
    logits (fp64), which equals the full softmax renormalised over the
    selection.  Returns ``(idx int32 [T, k], w fp64 [T, k])``.
    """
    T, E = logits_f32.shape
    idx = torch.empty(T, k, dtype=torch.int32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits_f32[t, e]), e))
        idx[t] = torch.tensor(order[:k], dtype=torch.int32)
    sel = torch.gather(logits_f32.to(F64), 1, idx.long())
    w = torch.softmax(sel, dim=1)
    return idx, w


def expert_histogram(idx: torch.Tensor, n_experts: int) -> torch.Tensor:
    """``hist[e]`` = number of (token, slot) pairs routed to expert ``e``."""
    hist = torch.zeros(n_experts, dtype=torch.int32)
    for e in idx.reshape(-1).tolist():
        hist[e] += 1
    return hist


def exp_indptr(hist: torch.Tensor) -> torch.Tensor:
    """Exclusive prefix sum of ``hist``, length ``E + 1``: expert ``e``'s rows
    of the grouped activation matrix are ``[indptr[e], indptr[e+1])``."""
    out = torch.zeros(hist.numel() + 1, dtype=torch.int32)
    run = 0
    for e in range(hist.numel()):
        out[e] = run
        run += int(hist[e])
    out[hist.numel()] = run
    return out


def moe_ffn(x: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
            w_down: torch.Tensor) -> torch.Tensor:
    """One expert's SwiGLU FFN in fp64: ``(silu(x Wg^T) * (x Wu^T)) Wd^T``."""
    x = x.to(F64)
    return swiglu(x @ w_gate.to(F64).T, x @ w_up.to(F64).T) @ w_down.to(F64).T


def moe_layer(x_bf16: torch.Tensor, w: dict, top_k: int,
              bias_f32: torch.Tensor | None = None) -> dict:
    """The whole MoE FFN on ``T`` tokens (no norm, no residual).

    ``out[t] = sum_j w[t, j] * FFN_{idx[t, j]}(x[t])``, accumulated in slot
    order ``j = 0..k-1``.  Returns the fp64 output plus the integer routing
    results (``idx``, ``hist``, ``indptr``) and the fp32 ``logits``.
    """
    E = w["router"].shape[0]
    logits = router_logits(x_bf16, w["router"], bias_f32)
    idx, wts = topk_route(logits, top_k)
    hist = expert_histogram(idx, E)
    indptr = exp_indptr(hist)
    T, H = x_bf16.shape
    xf = x_bf16.to(F64)
    # each expert's FFN on the tokens routed to it
    y = {}
    for e in range(E):
        ts = [t for t in range(T) if e in idx[t].tolist()]
        if ts:
            ye = moe_ffn(xf[torch.tensor(ts)], w["w_gate"][e], w["w_up"][e], w["w_down"][e])
            for r, t in enumerate(ts):
                y[(e, t)] = ye[r]
    # combine in slot order j = 0..k-1
    out = torch.zeros(T, H, dtype=F64)
    for t in range(T):
        for j in range(top_k):
            out[t] += wts[t, j] * y[(int(idx[t, j]), t)]
    return {"out": out, "idx": idx, "weights": wts, "hist": hist, "indptr": indptr,
            "logits": logits}
