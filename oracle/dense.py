"""Dense decode step, plain fp64 on the CPU (test infrastructure only).

Follows the op list of a decoder-only transformer decode step as the Event
Tensor pages use it ("Event Tensor: A Unified Abstraction for Compiling
Dynamic Megakernel", section "Related": attention, continuous batching;
"Lecture 112: Production Megakernels for Real-World Inference", section
"Symbolic Representation of Work": one new token per sequence attending to a
context of length P).  The pages do not spell out the layer maths; the
readings taken (pre-norm Llama block, rotate-half RoPE, GQA with contiguous
head groups, post-RoPE cache, tied LM head, ties in argmax to the lowest id)
are the plainest ones the configurations support.

Nothing here is blocked, fused or reordered: each function is the textbook
definition with a library matmul as its only primitive.
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64


def bf16_round(x: torch.Tensor) -> torch.Tensor:
    """Round to bf16 (RNE) and back to fp64: the value a bf16 store keeps."""
    return x.to(torch.bfloat16).to(F64)


def rms_norm(x: torch.Tensor, gamma: torch.Tensor, eps: float) -> torch.Tensor:
    """RMSNorm over the last axis: ``x / sqrt(mean(x^2) + eps) * gamma``."""
    x = x.to(F64)
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps) * gamma.to(F64)


def rope_cos_sin(pos: int, head_dim: int, theta: float):
    """cos/sin of the rotation angles ``pos * theta^(-2i/head_dim)``, i < head_dim/2.

    The angle of pair ``i`` follows the rotary position embedding of RoFormer
    (Su et al., 2021): frequency ``theta^(-2i/d)``.
    """
    half = head_dim // 2
    ang = [pos * theta ** (-2.0 * i / head_dim) for i in range(half)]
    return (torch.tensor([math.cos(a) for a in ang], dtype=F64),
            torch.tensor([math.sin(a) for a in ang], dtype=F64))


def apply_rope(v: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """Rotate pairs ``(v[i], v[i + d/2])`` by the angle of pair ``i`` ("rotate half").

    ``(a, b) -> (a cos - b sin, b cos + a sin)``, i.e. ``a + i b`` times
    ``exp(i * angle)``.
    """
    half = v.shape[-1] // 2
    a, b = v[..., :half].to(F64), v[..., half:].to(F64)
    return torch.cat([a * cos - b * sin, b * cos + a * sin], dim=-1)


def decode_attention(q: torch.Tensor, keys: torch.Tensor, values: torch.Tensor,
                     scale: float) -> torch.Tensor:
    """One decode token's grouped-query attention.

    ``q`` is ``[Hq, D]``; ``keys``/``values`` are ``[Hkv, n, D]``.  Query head
    ``h`` reads kv head ``h // (Hq / Hkv)``.  Returns ``[Hq, D]``:
    ``softmax(q_h . K_g^T * scale) V_g``.
    """
    Hq, Hkv = q.shape[0], keys.shape[0]
    group = Hq // Hkv
    out = torch.empty(Hq, q.shape[1], dtype=F64)
    for h in range(Hq):
        g = h // group
        s = (keys[g].to(F64) @ q[h].to(F64)) * scale
        a = torch.softmax(s, dim=0)
        out[h] = a @ values[g].to(F64)
    return out


def silu(x: torch.Tensor) -> torch.Tensor:
    return x / (1.0 + torch.exp(-x))


def swiglu(g: torch.Tensor, u: torch.Tensor) -> torch.Tensor:
    """SwiGLU gate: ``silu(g) * u``."""
    return silu(g.to(F64)) * u.to(F64)


def argmax_lowest(v: torch.Tensor) -> int:
    """Index of the maximum; ties resolve to the lowest index."""
    m = torch.max(v)
    return int(torch.nonzero(v == m)[0, 0])


class DenseOracle:
    """fp64 forward pass of one decode step over bf16 weights.

    ``weights`` is the dict of ``workloads.dense_weights``; weights are
    widened to fp64 once per layer on first use and kept.
    """

    def __init__(self, shape, weights: dict):
        self.s = shape
        self.w = weights
        self._cache = {}

    def _f64(self, name: str) -> torch.Tensor:
        t = self._cache.get(name)
        if t is None:
            t = self.w[name].to(F64)
            self._cache[name] = t
        return t

    def lm_head(self) -> torch.Tensor:
        return self._f64("embed" if self.s.tied else "lm_head")

    def step(self, K: torch.Tensor, V: torch.Tensor, tokens, slots, ctx,
             moe=None, capture: bool = False) -> dict:
        """Run one decode step for ``B = len(tokens)`` sequences.

        ``K``/``V`` (bf16 ``[L][slots][Hkv][Tmax][D]``) are updated in place:
        sequence ``b`` appends its rotated key and its value at position
        ``ctx[b]`` of slot ``slots[b]`` and attends to positions
        ``0..ctx[b]`` inclusive.  ``moe`` (optional) maps a layer index to a
        callable ``u_bf16 -> ffn_out`` replacing the dense FFN.

        Returns ``logits`` fp64 ``[B, V]``, ``next_tokens`` ``[B]`` and, with
        ``capture``, the residual stream after every layer.
        """
        s = self.s
        B = len(tokens)
        D, Hq, Hkv = s.head_dim, s.n_q_heads, s.n_kv_heads
        scale = 1.0 / math.sqrt(D)
        x = self._f64("embed")[torch.as_tensor(tokens, dtype=torch.long)].clone()
        resid = []
        for l in range(s.n_layers):
            p = f"layers.{l}."
            u = rms_norm(x, self._f64(p + "attn_norm"), s.eps)
            q = u @ self._f64(p + "wq").T
            k = u @ self._f64(p + "wk").T
            v = u @ self._f64(p + "wv").T
            o = torch.empty(B, Hq * D, dtype=F64)
            for b in range(B):
                pos = int(ctx[b])
                slot = int(slots[b])
                cos, sin = rope_cos_sin(pos, D, s.rope_theta)
                qb = apply_rope(q[b].view(Hq, D), cos, sin)
                kb = apply_rope(k[b].view(Hkv, D), cos, sin)
                K[l, slot, :, pos, :] = kb.to(torch.bfloat16)
                V[l, slot, :, pos, :] = v[b].view(Hkv, D).to(torch.bfloat16)
                keys = K[l, slot, :, : pos + 1, :]
                vals = V[l, slot, :, : pos + 1, :]
                o[b] = decode_attention(qb, keys, vals, scale).reshape(-1)
            x = x + o @ self._f64(p + "wo").T
            u = rms_norm(x, self._f64(p + "ffn_norm"), s.eps)
            if moe is not None:
                x = x + moe(l, u)
            else:
                h = swiglu(u @ self._f64(p + "w_gate").T, u @ self._f64(p + "w_up").T)
                x = x + h @ self._f64(p + "w_down").T
            if capture:
                resid.append(x.clone())
        logits = rms_norm(x, self._f64("final_norm"), s.eps) @ self.lm_head().T
        nxt = torch.tensor([argmax_lowest(logits[b]) for b in range(B)], dtype=torch.int32)
        out = {"logits": logits, "next_tokens": nxt}
        if capture:
            out["residual"] = resid
        return out
