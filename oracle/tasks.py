"""Expected task set of one decode step — test infrastructure only.

"Event Tensor: A Unified Abstraction for Compiling Dynamic Megakernel",
section "Core method": an event is the completion of a set of SM-granular
tasks, and its dimensions may be symbolic (the batch size); "Lecture 112:
Production Megakernels for Real-World Inference", section "Symbolic
Representation of Work": extents are expressions of the runtime sizes (the
context length).  The set of tasks one step must run is therefore a function
of the step's batch size and per-sequence context lengths plus the tile
sizes, which are passed in here as plain numbers.

Task families of one dense layer, in the order a layer runs them:

* ``qkv``    — one per ``tile_qkv`` output rows of the stacked Q/K/V weights;
* ``attn``   — one per (sequence b, kv head g, key chunk c),
  ``c < ceil((ctx_b + 1) / chunk)``;
  (the last attention task of a (b, g) to finish merges that pair's partials
  itself: no task of its own);
* ``oproj``  — one per ``tile_o`` rows of the output projection;
* ``gateup`` — one per ``tile_gu`` rows of the gate (and the same rows of up);
* ``down``   — one per (``tile_down`` rows, K segment of ``kseg`` columns).

After the last layer: ``lm`` (``tile_lm`` vocabulary rows each) and
``lmfin`` (one: the greedy token from the LM tiles' running maximum).

An attention task may take ``split`` consecutive key chunks (``tiles["split"]``,
default 1): sequence b then has ``nch_b = ceil(ceil((ctx_b + 1) / chunk) /
split)`` attention tasks per kv head.  With ``tiles["split_auto"]`` the split
is chosen per step (``step_split``): the step's chunk units
``C = Hkv * sum_b ceil((ctx_b + 1) / chunk)`` over about two thirds of
``tiles["n_sm"]`` tasks, ``ceil(C / ceil(2 n_sm / 3))``, kept between
``min(3, split)`` and ``split``; in the wide-batch layout only at steps of at
most 8 rows (above that the split is ``split``).  Linear index of an ``attn`` task:
``Hkv * sum_{b'<b} nch_{b'} + g * nch_b + c``.  ``down`` tasks are numbered
K-segment-major: ``kc * (H / tile_down) + n``.

With ``tiles["wide"]`` (the wide-batch layout, where the normalised
activations are materialised) a layer also runs ``norm`` before ``qkv`` and
``norm2`` before ``gateup``, and ``normf`` runs before ``lm``: one task per
batch row each.  Its ``qkv``, ``oproj`` and ``gateup`` tiles may run as
``tiles["gseg"]`` = (q, o, g) tasks each, one per K segment (task i is
segment i % s of tile i // s).
"""
from __future__ import annotations


def _ceil(a: int, b: int) -> int:
    return -(-a // b)


def step_split(shape, B: int, ctx, tiles: dict) -> int:
    """Key chunks per attention task in a step with these contexts."""
    split = tiles.get("split", 1)
    if not tiles.get("split_auto") or (tiles.get("wide") and B > 8):
        return split
    units = shape.n_kv_heads * sum(_ceil(int(ctx[b]) + 1, tiles["chunk"]) for b in range(B))
    target = _ceil(2 * tiles["n_sm"], 3)
    return max(min(3, split), min(split, _ceil(units, target)))


def dense_family_extents(shape, B: int, ctx, tiles: dict) -> dict:
    """Number of tasks of each family in one layer (and after the last)."""
    H, D = shape.hidden, shape.head_dim
    Hq, Hkv = shape.n_q_heads, shape.n_kv_heads
    split = step_split(shape, B, ctx, tiles)
    nch = [_ceil(_ceil(int(ctx[b]) + 1, tiles["chunk"]), split) for b in range(B)]
    n_lm = _ceil(shape.vocab, tiles["tile_lm"])
    norms = {"norm": B, "norm2": B, "normf": B} if tiles.get("wide") else {}
    sq, so, sg = tiles.get("gseg", (1, 1, 1))  # K segments per tile, each its own task
    return {
        **norms,
        "qkv": (Hq + 2 * Hkv) * D // tiles["tile_qkv"] * sq,
        "attn": Hkv * sum(nch),
        "oproj": H // tiles["tile_o"] * so,
        "gateup": shape.ffn // tiles["tile_gu"] * sg,
        "down": (H // tiles["tile_down"]) * (shape.ffn // tiles["kseg"]),
        "lm": n_lm,
        "lmfin": 1,
    }


def expected_dense_tasks(shape, B: int, ctx, tiles: dict) -> set:
    """The set of ``(family, layer, index)`` one decode step runs exactly once.

    Per-layer families carry their layer; ``lm`` and ``lmfin``
    carry layer ``-1``.  ``attn`` indices are enumerated from the (b, g, c)
    triples, so the set also pins the linear numbering stated above.
    """
    ext = dense_family_extents(shape, B, ctx, tiles)
    Hkv = shape.n_kv_heads
    wide = bool(tiles.get("wide"))
    split = step_split(shape, B, ctx, tiles)
    out = set()
    for l in range(shape.n_layers):
        for fam in ("qkv", "oproj", "gateup", "down") + (("norm", "norm2") if wide else ()):
            out.update((fam, l, i) for i in range(ext[fam]))
        base = 0
        for b in range(B):
            nch = _ceil(_ceil(int(ctx[b]) + 1, tiles["chunk"]), split)
            for g in range(Hkv):
                for c in range(nch):
                    out.add(("attn", l, Hkv * base + g * nch + c))
            base += nch
    for fam in ("lm", "lmfin") + (("normf",) if wide else ()):
        out.update((fam, -1, i) for i in range(ext[fam]))
    return out


def moe_tiles(hist, tm: int, big: int = 0):
    """GroupGEMM tiles of an MoE layer: expert ``e``'s ``hist[e]`` rows split
    into ``ceil(hist[e] / tm_e)`` tiles of at most ``tm_e`` rows, numbered
    expert by expert in increasing expert id ("Event Tensor: A Unified
    Abstraction for Compiling Dynamic Megakernel", section "Core method": the
    prefix sum of the per-expert counts decides how many GroupGEMM tiles each
    expert triggers).  ``tm_e = tm``, or with routing-aware tiles (``big`` > 0;
    "RaMP: Runtime-Aware Megakernel Polymorphism for Mixture-of-Experts": the
    tile configuration follows the run-time histogram) ``tm_e = big`` for an
    expert with more than ``tm`` rows.  Returns ``[(expert, first row, rows),
    ...]`` with rows counted from ``exp_indptr[e]``."""
    tiles, row = [], 0
    for e, h in enumerate(int(v) for v in hist):
        te = big if (big and h > tm) else tm
        for m in range(_ceil(h, te)):
            tiles.append((e, row + m * te, min(te, h - m * te)))
        row += h
    return tiles


def expected_moe_tasks(T: int, hist, hidden: int, expert_ffn: int, tiles: dict) -> set:
    """The set of ``(family, -1, index)`` one MoE layer call runs exactly once.

    ``route`` and ``combine``: ``ceil(T / 8)`` each (8 tokens per task);
    ``mindptr`` and ``mfin``: one each; ``egu``: ``tiles * ceil(F / tn)``
    numbered ``tile * ceil(F / tn) + n``; ``edown``: ``tiles * (H / td)``
    numbered ``tile * (H / td) + n``.
    """
    n_tiles = len(moe_tiles(hist, tiles["tm"], tiles.get("big", 0)))
    nt_gu = _ceil(expert_ffn, tiles["tn"])
    nt_d = hidden // tiles["td"]
    out = set()
    for i in range(_ceil(T, 8)):
        out.add(("route", -1, i))
        out.add(("combine", -1, i))
    out.add(("mindptr", -1, 0))
    out.add(("mfin", -1, 0))
    for i in range(n_tiles * nt_gu):
        out.add(("egu", -1, i))
    for i in range(n_tiles * nt_d):
        out.add(("edown", -1, i))
    return out
