"""Seeded synthetic inputs for the decode-megakernel workloads.

This module draws random numbers and lays them out; it holds none of the
decode step's arithmetic (no norm, projection, attention, routing or
reduction).  It is the one module that both the CPU oracle and the CUDA path
import, so that both see bit-identical inputs.

Every tensor is filled from a fixed-size chunk stream: chunk ``k`` of the
tensor named ``name`` uses ``numpy.random.PCG64(SeedSequence([seed,
crc32(name), k]))``.  The result does not depend on the number of worker
threads.  Normal samples are drawn in fp32 and rounded to bf16 with
round-to-nearest-even (torch's conversion).

Workload shapes follow the decode workloads described for Event Tensor
megakernels ("Event Tensor: A Unified Abstraction for Compiling Dynamic
Megakernel", sections "Problem" and "Core method": continuous batching with a
varying batch size, MoE routing with runtime top-k).
"""
from __future__ import annotations

import math
import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

MASTER_SEED = 0
TOKEN_SEED = 2
SCHEDULE_SEED = 3
ZIPF_PERM_SEED = 1
CHUNK = 1 << 22


@dataclass(frozen=True)
class DenseShape:
    """Decoder-only transformer with GQA attention and a SwiGLU FFN."""
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    eps: float = 1e-5
    rope_theta: float = 10000.0
    tied: bool = True


@dataclass(frozen=True)
class MoEShape:
    """One MoE FFN: a router over ``n_experts`` SwiGLU experts, top-k routing."""
    hidden: int
    n_experts: int
    top_k: int
    expert_ffn: int


# Tiny dense decoder: 2 layers, hidden 256, 4 q / 2 kv heads x 64, FFN 1024.
TINY = DenseShape(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2,
                  head_dim=64, ffn=1024, vocab=1024)
# Llama-1B-shaped decoder: 16 layers, hidden 2048, 32 q / 8 kv heads x 64,
# FFN 8192, vocab 128256, tied embeddings.
LLAMA_1B = DenseShape(n_layers=16, hidden=2048, n_q_heads=32, n_kv_heads=8,
                      head_dim=64, ffn=8192, vocab=128256)
# Single MoE FFN layer: hidden 2048, 64 experts, top-8, expert FFN 1408.
MOE_64x8 = MoEShape(hidden=2048, n_experts=64, top_k=8, expert_ffn=1408)

WEIGHT_STD = 0.02


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _chunk_normal(seed: int, name: str, k: int, n: int, std: float) -> torch.Tensor:
    ss = np.random.SeedSequence([seed, zlib.crc32(name.encode()), k])
    g = np.random.Generator(np.random.PCG64(ss))
    a = g.standard_normal(n, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return torch.from_numpy(a).to(torch.bfloat16)


def normal_bf16(name: str, shape, std: float, seed: int = MASTER_SEED) -> torch.Tensor:
    """N(0, std) samples, fp32 then bf16 (RNE), filled in row-major order."""
    numel = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(numel, dtype=torch.bfloat16)
    nchunks = (numel + CHUNK - 1) // CHUNK

    def job(k):
        lo = k * CHUNK
        hi = min(numel, lo + CHUNK)
        out[lo:hi] = _chunk_normal(seed, name, k, hi - lo, std)

    if nchunks <= 1:
        for k in range(nchunks):
            job(k)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(job, range(nchunks)))
    return out.view(*shape)


def dense_weights(s: DenseShape, seed: int = MASTER_SEED) -> dict:
    """bf16 weights of a dense decoder, all ``[out, in]`` row-major.

    Linear and embedding matrices are N(0, 0.02); RMSNorm gains are ones.
    """
    H, D = s.hidden, s.head_dim
    w = {"embed": normal_bf16("embed", (s.vocab, H), WEIGHT_STD, seed)}
    for l in range(s.n_layers):
        p = f"layers.{l}."
        w[p + "attn_norm"] = torch.ones(H, dtype=torch.bfloat16)
        w[p + "wq"] = normal_bf16(p + "wq", (s.n_q_heads * D, H), WEIGHT_STD, seed)
        w[p + "wk"] = normal_bf16(p + "wk", (s.n_kv_heads * D, H), WEIGHT_STD, seed)
        w[p + "wv"] = normal_bf16(p + "wv", (s.n_kv_heads * D, H), WEIGHT_STD, seed)
        w[p + "wo"] = normal_bf16(p + "wo", (H, s.n_q_heads * D), WEIGHT_STD, seed)
        w[p + "ffn_norm"] = torch.ones(H, dtype=torch.bfloat16)
        w[p + "w_gate"] = normal_bf16(p + "w_gate", (s.ffn, H), WEIGHT_STD, seed)
        w[p + "w_up"] = normal_bf16(p + "w_up", (s.ffn, H), WEIGHT_STD, seed)
        w[p + "w_down"] = normal_bf16(p + "w_down", (H, s.ffn), WEIGHT_STD, seed)
    w["final_norm"] = torch.ones(H, dtype=torch.bfloat16)
    if not s.tied:
        w["lm_head"] = normal_bf16("lm_head", (s.vocab, H), WEIGHT_STD, seed)
    return w


def kv_cache(s: DenseShape, n_slots: int, max_ctx: int, ctx_lens, seed: int = MASTER_SEED):
    """bf16 K and V caches ``[L][n_slots][Hkv][max_ctx][D]``.

    Slot ``b`` holds N(0,1) samples at positions ``< ctx_lens[b]`` and zeros
    after; the cached keys are taken to be already rotated (post-RoPE).
    """
    L, Hkv, D = s.n_layers, s.n_kv_heads, s.head_dim
    K = torch.zeros(L, n_slots, Hkv, max_ctx, D, dtype=torch.bfloat16)
    V = torch.zeros_like(K)
    jobs = []
    for l in range(L):
        for slot, n in enumerate(ctx_lens):
            n = int(n)
            if n > 0:
                jobs.append((l, slot, n))

    def job(j):
        l, slot, n = j
        K[l, slot, :, :n, :] = _slot_rows(seed, f"kcache.{l}.{slot}", Hkv, n, D)
        V[l, slot, :, :n, :] = _slot_rows(seed, f"vcache.{l}.{slot}", Hkv, n, D)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(job, jobs))
    return K, V


def _slot_rows(seed, name, Hkv, n, D):
    numel = Hkv * n * D
    parts = []
    for k in range((numel + CHUNK - 1) // CHUNK):
        lo = k * CHUNK
        parts.append(_chunk_normal(seed, name, k, min(CHUNK, numel - lo), 1.0))
    return torch.cat(parts).view(Hkv, n, D)


def token_ids(n: int, vocab: int, seed: int = TOKEN_SEED, stream: str = "tokens") -> torch.Tensor:
    """``n`` token ids uniform over ``[0, vocab)``, int32."""
    ss = np.random.SeedSequence([seed, zlib.crc32(stream.encode())])
    g = np.random.Generator(np.random.PCG64(ss))
    return torch.from_numpy(g.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32))


def context_lengths(n: int, lo: int, hi: int, seed: int = TOKEN_SEED, stream: str = "ctx") -> torch.Tensor:
    """``n`` context lengths uniform over ``[lo, hi]`` (inclusive), int32."""
    ss = np.random.SeedSequence([seed, zlib.crc32(stream.encode())])
    g = np.random.Generator(np.random.PCG64(ss))
    return torch.from_numpy(g.integers(lo, hi + 1, size=n, dtype=np.int64).astype(np.int32))


def batch_schedule(n_steps: int, choices, seed: int = SCHEDULE_SEED) -> list:
    """Per-step batch sizes for continuous batching: a seeded walk over ``choices``.

    The choices are cycled through in seeded shuffles, so each size appears
    once per ``len(choices)`` steps.
    """
    ss = np.random.SeedSequence([seed])
    g = np.random.Generator(np.random.PCG64(ss))
    out = []
    while len(out) < n_steps:
        out.extend(int(c) for c in g.permutation(np.asarray(choices)))
    return out[:n_steps]


def moe_weights(m: MoEShape, seed: int = MASTER_SEED, prefix: str = "moe.") -> dict:
    """bf16 router ``[E, H]`` and expert SwiGLU weights, N(0, 0.02).

    ``w_gate``/``w_up`` are ``[E, F, H]`` and ``w_down`` is ``[E, H, F]``.
    """
    E, H, F = m.n_experts, m.hidden, m.expert_ffn
    return {
        "router": normal_bf16(prefix + "router", (E, H), WEIGHT_STD, seed),
        "w_gate": normal_bf16(prefix + "w_gate", (E, F, H), WEIGHT_STD, seed),
        "w_up": normal_bf16(prefix + "w_up", (E, F, H), WEIGHT_STD, seed),
        "w_down": normal_bf16(prefix + "w_down", (E, H, F), WEIGHT_STD, seed),
    }


def moe_tokens(T: int, hidden: int, seed: int = MASTER_SEED, stream: str = "moe.x") -> torch.Tensor:
    """``T`` activations N(0,1) bf16 ``[T, hidden]``."""
    return normal_bf16(f"{stream}.{T}", (T, hidden), 1.0, seed)


def zipf_bias(n_experts: int, s: float = 1.2, seed: int = ZIPF_PERM_SEED) -> torch.Tensor:
    """Per-expert router-logit bias for skewed routing: ``-s * ln(rank)``.

    ``rank_e = 1 + perm[e]`` for a seeded permutation ``perm``; adding
    ``-s ln(rank)`` to a logit multiplies its softmax weight by
    ``rank^-s``, i.e. a Zipf(s) prior over experts.  Returned as fp32.
    """
    ss = np.random.SeedSequence([seed, zlib.crc32(b"zipf")])
    g = np.random.Generator(np.random.PCG64(ss))
    perm = g.permutation(n_experts)
    bias = np.array([-s * math.log(1 + int(perm[e])) for e in range(n_experts)], dtype=np.float64)
    return torch.from_numpy(bias.astype(np.float32))


def no_bias(n_experts: int) -> torch.Tensor:
    """All-zero router bias (uniform routing regime)."""
    return torch.zeros(n_experts, dtype=torch.float32)
