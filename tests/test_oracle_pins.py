"""Pins of the CPU oracle against things other than itself.

Closed forms, hand-derived fixtures (tests/golden), invariants, special cases
that reduce to a library routine, and a scalar brute force on tiny inputs.
Each pin is chosen so that a plausible slip (a dropped term, a wrong sign, a
wrong head/expert index, a transposed operand) fails at least one of them.
"""
import math
import random

import pytest
import torch

import oracle
from oracle import dense as od
from oracle import moe as om
from oracle import tasks as ot
import workloads as wl
from conftest import read_golden

F64 = torch.float64


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_golden():
    want = [float(v) for v in read_golden("rmsnorm_3_4.txt")[0]]
    got = od.rms_norm(torch.tensor([[3.0, 4.0]]), torch.ones(2), 0.0)[0]
    assert torch.allclose(got, torch.tensor(want, dtype=F64), rtol=0, atol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(3, 64, generator=g, dtype=F64)
    y = od.rms_norm(x, torch.ones(64), 0.0)
    assert torch.allclose((y * y).mean(-1), torch.ones(3, dtype=F64), atol=1e-14)
    assert torch.allclose(od.rms_norm(7.5 * x, torch.ones(64), 0.0), y, atol=1e-14)
    gamma = torch.linspace(-2, 2, 64, dtype=F64)
    assert torch.allclose(od.rms_norm(x, gamma, 0.0), y * gamma, atol=1e-14)
    # eps enters under the root: a constant vector c maps to c / sqrt(c^2 + eps)
    c = torch.full((1, 8), 0.01, dtype=F64)
    assert torch.allclose(od.rms_norm(c, torch.ones(8), 1e-5),
                          c / math.sqrt(1e-4 + 1e-5), atol=1e-14)


# ---------------------------------------------------------------- RoPE
def test_rope_golden():
    want = torch.tensor([float(v) for v in read_golden("rope_d4_pos1.txt")[0]], dtype=F64)
    cos, sin = od.rope_cos_sin(1, 4, 10000.0)
    got = od.apply_rope(torch.tensor([1.0, 2.0, 3.0, 4.0], dtype=F64), cos, sin)
    assert torch.allclose(got, want, atol=1e-15)


def test_rope_equals_complex_multiplication():
    g = torch.Generator().manual_seed(2)
    v = torch.randn(5, 64, generator=g, dtype=F64)
    for pos in (0, 1, 17, 1023, 4095):
        cos, sin = od.rope_cos_sin(pos, 64, 10000.0)
        z = torch.complex(v[:, :32], v[:, 32:]) * torch.polar(torch.ones(32, dtype=F64),
                                                              torch.atan2(sin, cos))
        want = torch.cat([z.real, z.imag], dim=-1)
        assert torch.allclose(od.apply_rope(v, cos, sin), want, atol=1e-12)


def test_rope_invariants():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(64, generator=g, dtype=F64)
    k = torch.randn(64, generator=g, dtype=F64)
    c0, s0 = od.rope_cos_sin(0, 64, 10000.0)
    assert torch.equal(od.apply_rope(q, c0, s0), q)
    ca, sa = od.rope_cos_sin(5, 64, 10000.0)
    cb, sb = od.rope_cos_sin(11, 64, 10000.0)
    cab, sab = od.rope_cos_sin(16, 64, 10000.0)
    assert torch.allclose(od.apply_rope(od.apply_rope(q, ca, sa), cb, sb),
                          od.apply_rope(q, cab, sab), atol=1e-12)
    r = od.apply_rope(q, cab, sab)
    assert torch.allclose(r[:32] ** 2 + r[32:] ** 2, q[:32] ** 2 + q[32:] ** 2, atol=1e-12)
    # scores depend on the position difference only
    cm, sm = od.rope_cos_sin(40, 64, 10000.0)
    cn, sn = od.rope_cos_sin(29, 64, 10000.0)
    cd, sd = od.rope_cos_sin(11, 64, 10000.0)
    lhs = od.apply_rope(q, cm, sm) @ od.apply_rope(k, cn, sn)
    assert abs(float(lhs - od.apply_rope(q, cd, sd) @ k)) < 1e-11


# ---------------------------------------------------------------- attention
def test_attention_single_key_returns_value():
    g = torch.Generator().manual_seed(4)
    q = torch.randn(4, 64, generator=g, dtype=F64)
    K = torch.randn(2, 1, 64, generator=g, dtype=F64)
    V = torch.randn(2, 1, 64, generator=g, dtype=F64)
    o = od.decode_attention(q, K, V, 0.125)
    assert torch.allclose(o, V[[0, 0, 1, 1], 0], atol=1e-15)


def test_attention_equal_keys_mean_of_values():
    g = torch.Generator().manual_seed(5)
    q = torch.randn(2, 64, generator=g, dtype=F64)
    K = torch.randn(1, 1, 64, generator=g, dtype=F64).expand(1, 9, 64)
    V = torch.randn(1, 9, 64, generator=g, dtype=F64)
    o = od.decode_attention(q, K, V, 0.125)
    assert torch.allclose(o, V[0].mean(0).expand(2, 64), atol=1e-14)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (32, 8)])
def test_attention_matches_library_sdpa(hq, hkv):
    g = torch.Generator().manual_seed(6)
    n = 37
    q = torch.randn(hq, 64, generator=g, dtype=F64)
    K = torch.randn(hkv, n, 64, generator=g, dtype=F64)
    V = torch.randn(hkv, n, 64, generator=g, dtype=F64)
    rep = hq // hkv
    Ke = K.repeat_interleave(rep, dim=0)
    Ve = V.repeat_interleave(rep, dim=0)
    want = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], Ke, Ve, scale=0.125)[:, 0, :]
    assert torch.allclose(od.decode_attention(q, K, V, 0.125), want, atol=1e-12)


def test_attention_gqa_groups_are_contiguous():
    # only kv head 0 carries nonzero values: q heads 0..3 see it, 4..7 do not
    g = torch.Generator().manual_seed(7)
    q = torch.randn(8, 64, generator=g, dtype=F64)
    K = torch.randn(2, 5, 64, generator=g, dtype=F64)
    V = torch.zeros(2, 5, 64, dtype=F64)
    V[0] = torch.randn(5, 64, generator=g, dtype=F64)
    o = od.decode_attention(q, K, V, 0.125)
    assert (o[:4].abs().sum(-1) > 0).all() and (o[4:] == 0).all()


# ---------------------------------------------------------------- SwiGLU
def test_swiglu_closed_forms():
    x = torch.tensor([0.0, 1.0, -1.0, 40.0, -40.0], dtype=F64)
    s = od.swiglu(x, torch.ones(5, dtype=F64))
    assert s[0] == 0
    assert abs(float(s[1]) - 1 / (1 + math.exp(-1))) < 1e-15
    assert abs(float(s[2]) + 1 / (1 + math.e)) < 1e-15
    assert abs(float(s[3]) - 40.0) < 1e-12 and abs(float(s[4])) < 1e-15
    assert torch.allclose(od.swiglu(x, 3 * torch.ones(5, dtype=F64)), 3 * s)


# ---------------------------------------------------------------- full step
MICRO = wl.DenseShape(n_layers=2, hidden=16, n_q_heads=4, n_kv_heads=2, head_dim=8,
                      ffn=24, vocab=20)


def _micro_inputs(seed=0):
    w = wl.dense_weights(MICRO, seed=seed)
    # non-trivial gains, so that a dropped gamma shows
    for k in list(w):
        if k.endswith("norm"):
            w[k] = (1.0 + 0.25 * torch.arange(MICRO.hidden, dtype=F64) / MICRO.hidden).to(torch.bfloat16)
    ctx = [3, 6]
    K, V = wl.kv_cache(MICRO, 2, 8, ctx, seed=seed)
    return w, K, V, ctx


def _scalar_decode(s, w, K, V, tokens, slots, ctx):
    """Brute force with Python floats and loops; independent of oracle.dense."""
    H, D, Hq, Hkv = s.hidden, s.head_dim, s.n_q_heads, s.n_kv_heads
    f = lambda t: t.to(F64).tolist()
    E = f(w["embed"])
    Kc = K.clone()
    Vc = V.clone()
    out_logits = []
    for b, tok in enumerate(tokens):
        x = list(E[tok])
        p = ctx[b]
        for l in range(s.n_layers):
            P = f"layers.{l}."

            def norm(v, gname):
                gm = f(w[P + gname] if gname != "final_norm" else w["final_norm"])
                r = math.sqrt(sum(a * a for a in v) / len(v) + s.eps)
                return [v[i] / r * gm[i] for i in range(len(v))]

            def lin(W, v):
                return [sum(W[o][i] * v[i] for i in range(len(v))) for o in range(len(W))]

            u = norm(x, "attn_norm")
            q = lin(f(w[P + "wq"]), u)
            k = lin(f(w[P + "wk"]), u)
            v = lin(f(w[P + "wv"]), u)

            def rot(vec):
                o = list(vec)
                for i in range(D // 2):
                    a = p * s.rope_theta ** (-2 * i / D)
                    x0, x1 = vec[i], vec[i + D // 2]
                    o[i] = x0 * math.cos(a) - x1 * math.sin(a)
                    o[i + D // 2] = x1 * math.cos(a) + x0 * math.sin(a)
                return o

            for g in range(Hkv):
                kr = rot(k[g * D:(g + 1) * D])
                for i in range(D):
                    Kc[l, slots[b], g, p, i] = kr[i]
                    Vc[l, slots[b], g, p, i] = v[g * D + i]
            att = []
            for h in range(Hq):
                g = h // (Hq // Hkv)
                qh = rot(q[h * D:(h + 1) * D])
                keys = f(Kc[l, slots[b], g, :p + 1])
                vals = f(Vc[l, slots[b], g, :p + 1])
                sc = [sum(qh[i] * kk[i] for i in range(D)) / math.sqrt(D) for kk in keys]
                m = max(sc)
                e = [math.exp(z - m) for z in sc]
                z = sum(e)
                att += [sum(e[t] * vals[t][i] for t in range(p + 1)) / z for i in range(D)]
            o = lin(f(w[P + "wo"]), att)
            x = [x[i] + o[i] for i in range(H)]
            u = norm(x, "ffn_norm")
            gt = lin(f(w[P + "w_gate"]), u)
            up = lin(f(w[P + "w_up"]), u)
            hh = [gt[j] / (1 + math.exp(-gt[j])) * up[j] for j in range(len(gt))]
            d = lin(f(w[P + "w_down"]), hh)
            x = [x[i] + d[i] for i in range(H)]
        gm = f(w["final_norm"])
        r = math.sqrt(sum(a * a for a in x) / H + s.eps)
        xn = [x[i] / r * gm[i] for i in range(H)]
        out_logits.append([sum(E[vv][i] * xn[i] for i in range(H)) for vv in range(s.vocab)])
    return torch.tensor(out_logits, dtype=F64), Kc, Vc


def test_decode_step_matches_scalar_brute_force():
    w, K, V, ctx = _micro_inputs()
    tokens, slots = [5, 17], [0, 1]
    K1, V1 = K.clone(), V.clone()
    res = od.DenseOracle(MICRO, w).step(K1, V1, tokens, slots, ctx)
    want, Kw, Vw = _scalar_decode(MICRO, w, K, V, tokens, slots, ctx)
    assert torch.allclose(res["logits"], want, rtol=1e-10, atol=1e-12)
    assert torch.equal(K1, Kw) and torch.equal(V1, Vw)
    assert res["next_tokens"].tolist() == [int(torch.argmax(want[b])) for b in range(2)]


def test_decode_step_batch_independence_and_cache_tail():
    w, K, V, ctx = _micro_inputs()
    o = od.DenseOracle(MICRO, w)
    KA, VA = K.clone(), V.clone()
    both = o.step(KA, VA, [5, 17], [0, 1], ctx)["logits"]
    KB, VB = K.clone(), V.clone()
    # garbage beyond each sequence's context must not be read
    KB[:, 0, :, ctx[0] + 1:] = 99.0
    VB[:, 1, :, ctx[1] + 1:] = -99.0
    one = o.step(KB, VB, [5], [0], [ctx[0]])["logits"]
    two = o.step(KB, VB, [17], [1], [ctx[1]])["logits"]
    assert torch.allclose(both, torch.cat([one, two]), atol=1e-13)


def test_zero_mixing_predicts_input_token():
    # with W_o = W_down = 0 the residual stays the embedding; with tied
    # embeddings the logits are E . norm(E[tok]) and the input token wins
    s = wl.TINY
    w = wl.dense_weights(s)
    for l in range(s.n_layers):
        w[f"layers.{l}.wo"] = torch.zeros_like(w[f"layers.{l}.wo"])
        w[f"layers.{l}.w_down"] = torch.zeros_like(w[f"layers.{l}.w_down"])
    K, V = wl.kv_cache(s, 1, 80, [64])
    toks = [3, 500, 1023]
    for t in toks:
        r = od.DenseOracle(s, w).step(K.clone(), V.clone(), [t], [0], [64])
        e = w["embed"].to(F64)
        want = e @ (e[t] / torch.sqrt((e[t] ** 2).mean() + s.eps))
        assert torch.allclose(r["logits"][0], want, atol=1e-12)
        assert int(r["next_tokens"][0]) == t


def test_argmax_ties_golden():
    # hand-worked rows with tied maxima (tests/golden/argmax_ties.txt)
    for row in read_golden("argmax_ties.txt"):
        assert row[0] == "case"
        arrow = row.index("->")
        vals = torch.tensor([float(v) for v in row[1:arrow]], dtype=F64)
        assert od.argmax_lowest(vals) == int(row[arrow + 1]), row


def test_decode_step_tied_logits_pick_lowest_id():
    # two identical rows of the tied embedding give two identical logits; when
    # they are the maximum the step returns the lower id
    s = wl.TINY
    w = wl.dense_weights(s)
    K, V = wl.kv_cache(s, 1, 80, [64])
    tok = 500
    best = int(od.DenseOracle(s, w).step(K.clone(), V.clone(), [tok], [0], [64])["next_tokens"][0])
    low = 0 if best != 0 else 1
    assert tok != low  # (the input row itself is unchanged)
    w2 = dict(w)
    e = w["embed"].clone()
    e[low] = e[best]
    w2["embed"] = e
    r = od.DenseOracle(s, w2).step(K.clone(), V.clone(), [tok], [0], [64])
    lg = r["logits"][0]
    assert float(lg[low]) == float(lg[best]) and float(lg[best]) == float(lg.max())
    assert int(r["next_tokens"][0]) == min(low, best)


# ---------------------------------------------------------------- MoE decoder block
def _dense_ffn_hook(w, s, round_input=False):
    """The dense FFN of each layer as a replacement FFN callable (fp64)."""
    def hook(l, u):
        P = f"layers.{l}."
        if round_input:
            u = od.bf16_round(u)
        return od.swiglu(u @ w[P + "w_gate"].double().T, u @ w[P + "w_up"].double().T) @ w[P + "w_down"].double().T
    return hook


def test_decoder_ffn_hook_reproduces_dense_step():
    # the replacement-FFN path (the MoE decoder's block) must see the
    # ffn-normed residual u and add its output to the residual: with the dense
    # FFN as the hook the step equals the dense step, residual captures included
    w, K, V, ctx = _micro_inputs()
    o = od.DenseOracle(MICRO, w)
    ref = o.step(K.clone(), V.clone(), [5, 17], [0, 1], ctx, capture=True)
    got = o.step(K.clone(), V.clone(), [5, 17], [0, 1], ctx, moe=_dense_ffn_hook(w, MICRO), capture=True)
    assert torch.allclose(got["logits"], ref["logits"], rtol=0, atol=1e-12)
    for a, b in zip(got["residual"], ref["residual"]):
        assert torch.allclose(a, b, rtol=0, atol=1e-12)
    # a hook fed x instead of u, or a dropped residual add, changes the result
    def bad_input(l, u):
        return _dense_ffn_hook(w, MICRO)(l, u * 2.0)
    bad = o.step(K.clone(), V.clone(), [5, 17], [0, 1], ctx, moe=bad_input)
    assert not torch.allclose(bad["logits"], ref["logits"], atol=1e-6)


def _moe_from_dense(w, s, l, E):
    """E identical experts, each the dense FFN of layer l; router zeros."""
    P = f"layers.{l}."
    return {"router": torch.zeros(E, s.hidden, dtype=torch.bfloat16),
            "w_gate": w[P + "w_gate"][None].expand(E, -1, -1).contiguous(),
            "w_up": w[P + "w_up"][None].expand(E, -1, -1).contiguous(),
            "w_down": w[P + "w_down"][None].expand(E, -1, -1).contiguous()}


@pytest.mark.parametrize("E,k", [(1, 1), (4, 2)])
def test_decoder_moe_block_equals_dense_on_rounded_input(E, k):
    # the MoE decoder block as the GPU tests build it (MoE layer on the
    # bf16-rounded normalised residual): E = k = 1 with the dense FFN as the
    # expert, and E identical experts with top-k > 1 (weights sum to one), both
    # equal the dense FFN applied to the rounded input
    s = wl.DenseShape(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=64, vocab=40)
    w = wl.dense_weights(s, seed=3)
    K, V = wl.kv_cache(s, 2, 16, [5, 9], seed=3)
    o = od.DenseOracle(s, w)
    experts = [_moe_from_dense(w, s, l, E) for l in range(s.n_layers)]
    hook = lambda l, u: om.moe_layer(u.to(torch.bfloat16), experts[l], k)["out"]
    got = o.step(K.clone(), V.clone(), [3, 11], [0, 1], [5, 9], moe=hook, capture=True)
    ref = o.step(K.clone(), V.clone(), [3, 11], [0, 1], [5, 9], moe=_dense_ffn_hook(w, s, round_input=True),
                 capture=True)
    assert torch.allclose(got["logits"], ref["logits"], rtol=0, atol=1e-12)
    for a, b in zip(got["residual"], ref["residual"]):
        assert torch.allclose(a, b, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- MoE router
def test_router_order_golden():
    rows = read_golden("router_order.txt")
    x = torch.zeros(1, 256)
    w = torch.zeros(1, 256)
    want = None
    for r in rows:
        if r[0] == "expected":
            want = float(r[1])
        else:
            x[0, int(r[0])] = float(r[1])
            w[0, int(r[0])] = float(r[2])
    got = om.router_logits(x.to(torch.bfloat16), w.to(torch.bfloat16))
    assert float(got[0, 0]) == want
    # the exact sum is 2: the fixed order is what makes the result 0
    assert float((x.double() * w.double()).sum()) == 2.0


def test_router_integer_inputs_exact():
    g = torch.Generator().manual_seed(8)
    x = torch.randint(-3, 4, (5, 512), generator=g).to(torch.bfloat16)
    w = torch.randint(-3, 4, (16, 512), generator=g).to(torch.bfloat16)
    exact = x.double() @ w.double().T
    assert torch.equal(om.router_logits(x, w).double(), exact)


def test_router_within_fp32_error_bound():
    m = wl.MOE_64x8
    w = wl.moe_weights(m)
    x = wl.moe_tokens(8, m.hidden)
    got = om.router_logits(x, w["router"]).double()
    exact = x.double() @ w["router"].double().T
    bound = m.hidden * 2.0 ** -24 * (x.double().abs() @ w["router"].double().abs().T)
    assert ((got - exact).abs() <= bound).all()
    bias = wl.zipf_bias(m.n_experts)
    gb = om.router_logits(x, w["router"], bias)
    assert torch.equal(gb, om.router_logits(x, w["router"]) + bias)


# ---------------------------------------------------------------- top-k, hist, indptr
def test_topk_golden_ties_and_indptr():
    rows = {r[0]: r[1:] for r in read_golden("topk_ties.txt")}
    logits = torch.tensor([[float(v) for v in rows["logits"]]])
    idx, wts = om.topk_route(logits, int(rows["k"][0]))
    assert idx[0].tolist() == [int(v) for v in rows["idx"]]
    assert abs(float(wts.sum()) - 1.0) < 1e-15
    hist = torch.tensor([int(v) for v in rows["hist"]], dtype=torch.int32)
    assert om.exp_indptr(hist).tolist() == [int(v) for v in rows["indptr"]]


def test_topk_all_equal_logits():
    idx, wts = om.topk_route(torch.zeros(3, 64), 8)
    assert idx.tolist() == [list(range(8))] * 3
    assert torch.allclose(wts, torch.full((3, 8), 1 / 8, dtype=F64))


def test_topk_matches_library_topk_and_invariants():
    g = torch.Generator().manual_seed(9)
    logits = torch.randn(50, 64, generator=g)
    idx, wts = om.topk_route(logits, 8)
    lib_v, lib_i = torch.topk(logits.double(), 8, dim=1)  # distinct values: order unique
    assert torch.equal(idx.long(), lib_i)
    full = torch.softmax(logits.double(), dim=1)
    renorm = torch.gather(full, 1, lib_i) / torch.gather(full, 1, lib_i).sum(1, keepdim=True)
    assert torch.allclose(wts, renorm, atol=1e-14)
    hist = om.expert_histogram(idx, 64)
    assert int(hist.sum()) == 50 * 8
    ind = om.exp_indptr(hist)
    assert ind[0] == 0 and ind[-1] == 400 and torch.equal(ind[1:] - ind[:-1], hist)
    assert all(len(set(r)) == 8 for r in idx.tolist())
    want = torch.bincount(idx.reshape(-1).long(), minlength=64).to(torch.int32)
    assert torch.equal(hist, want)


# ---------------------------------------------------------------- MoE layer
def _tiny_moe(E=8, H=256, F=64, seed=0):
    m = wl.MoEShape(hidden=H, n_experts=E, top_k=min(4, E), expert_ffn=F)
    return m, wl.moe_weights(m, seed=seed, prefix="tinymoe.")


def test_moe_identical_experts_is_one_ffn():
    m, w = _tiny_moe()
    for k in ("w_gate", "w_up", "w_down"):
        w[k] = w[k][:1].expand_as(w[k]).contiguous()
    x = wl.moe_tokens(6, m.hidden)
    r = om.moe_layer(x, w, m.top_k)
    want = om.moe_ffn(x.double(), w["w_gate"][0], w["w_up"][0], w["w_down"][0])
    assert torch.allclose(r["out"], want, atol=1e-13)


def test_moe_single_expert_is_dense_swiglu():
    m, w = _tiny_moe(E=1)
    x = wl.moe_tokens(3, m.hidden)
    r = om.moe_layer(x, w, 1)
    u = x.double()
    want = od.swiglu(u @ w["w_gate"][0].double().T, u @ w["w_up"][0].double().T) @ w["w_down"][0].double().T
    assert torch.allclose(r["out"], want, atol=1e-13)
    assert r["idx"].tolist() == [[0]] * 3 and r["hist"].tolist() == [3]


def test_moe_weight_expert_pairing():
    # expert e's down projection is alpha_e times expert 0's: the layer output is
    # (sum_j w_j alpha_{idx_j}) * FFN_0(x); a mispaired weight or expert fails
    m, w = _tiny_moe()
    alpha = torch.tensor([1.0, -2.0, 0.5, 4.0, -1.0, 0.25, 2.0, -0.5])  # powers of two: exact in bf16
    for k in ("w_gate", "w_up"):
        w[k] = w[k][:1].expand_as(w[k]).contiguous()
    w["w_down"] = (w["w_down"][:1].double() * alpha[:, None, None].double()).to(torch.bfloat16)
    x = wl.moe_tokens(5, m.hidden)
    r = om.moe_layer(x, w, m.top_k)
    base = om.moe_ffn(x.double(), w["w_gate"][0], w["w_up"][0], w["w_down"][0])
    coef = (r["weights"] * alpha.double()[r["idx"].long()]).sum(1)
    assert torch.allclose(r["out"], coef[:, None] * base, atol=1e-12)


def test_moe_skewed_bias_concentrates_routing():
    m = wl.MOE_64x8
    w = wl.moe_weights(m)
    x = wl.moe_tokens(64, m.hidden)
    bias = wl.zipf_bias(m.n_experts)
    lu = om.router_logits(x, w["router"])
    ls = om.router_logits(x, w["router"], bias)
    hu = om.expert_histogram(om.topk_route(lu, 8)[0], 64)
    hs = om.expert_histogram(om.topk_route(ls, 8)[0], 64)
    assert int((hs > 0).sum()) < int((hu > 0).sum())
    top = int(torch.argmax(bias))  # rank-1 expert has bias 0, the largest
    assert int(hs[top]) >= int(hu[top])


# ---------------------------------------------------------------- task set
TILES_TINY = dict(tile_qkv=8, chunk=64, tile_o=8, tile_gu=4, tile_down=8, kseg=1024,
                  tile_lm=16)


def test_task_counts_golden():
    rows = {r[0]: int(r[1]) for r in read_golden("task_counts_tiny.txt")}
    ext = ot.dense_family_extents(wl.TINY, 1, [64], TILES_TINY)
    for fam, n in ext.items():
        assert n == rows[fam], fam
    tasks = ot.expected_dense_tasks(wl.TINY, 1, [64], TILES_TINY)
    assert len(tasks) == rows["total"]


def test_step_split_by_hand():
    # the per-step attention split on the 1B shape (8 kv heads, 64-key
    # chunks) with 148 SMs: T = ceil(2 * 148 / 3) = 99 tasks
    tiles = dict(chunk=64, split=32, split_auto=True, n_sm=148)
    s = wl.LLAMA_1B
    # B=1 at 1024: 8 * ceil(1025 / 64) = 8 * 17 = 136 units, ceil(136 / 99) = 2, floor 3
    assert ot.step_split(s, 1, [1024], tiles) == 3
    # chunks 11, 39, 33, 4: 8 * 87 = 696 units, ceil(696 / 99) = 8 (7 * 99 = 693)
    assert ot.step_split(s, 4, [696, 2450, 2106, 216], tiles) == 8
    # chunks 11, 39, 33, 4, 21, 59, 7, 15: 8 * 189 = 1512, ceil(1512 / 99) = 16 (15 * 99 = 1485)
    assert ot.step_split(s, 8, [696, 2450, 2106, 216, 1316, 3764, 443, 949], tiles) == 16
    # 8 * 8 * 64 = 4096 units, ceil(4096 / 99) = 42, capped at 32
    assert ot.step_split(s, 8, [4095] * 8, tiles) == 32
    # the wide-batch layout: adaptive up to 8 rows (cap 24), fixed above
    wide = dict(tiles, split=24, wide=True)
    assert ot.step_split(s, 8, [4095] * 8, wide) == 24
    assert ot.step_split(s, 4, [696, 2450, 2106, 216], wide) == 8
    assert ot.step_split(s, 9, [0] * 9, wide) == 24
    # a cap below the floor of 3 wins; without split_auto the split is fixed
    assert ot.step_split(s, 1, [1024], dict(tiles, split=2)) == 2
    assert ot.step_split(s, 8, [4095] * 8, dict(tiles, split_auto=False)) == 32
    # the task set follows: B=1 at 1024 with split 3 has ceil(17 / 3) = 6 tasks per kv head
    ext = ot.dense_family_extents(s, 1, [1024], dict(TILES_TINY, **tiles))
    assert ext["attn"] == 8 * 6


def test_task_set_brute_force_attn_numbering():
    ctx = [0, 63, 64, 200]
    tasks = ot.expected_dense_tasks(wl.TINY, 4, ctx, TILES_TINY)
    attn = sorted(i for f, l, i in tasks if f == "attn" and l == 0)
    # indices are exactly 0..(total-1): a bijection with the (b, g, c) triples
    n = sum(2 * (-(-(c + 1) // 64)) for c in ctx)
    assert attn == list(range(n))


def test_task_set_wide_layout_by_hand():
    # TINY (2 layers, H 256, 4 q / 2 kv heads, F 1024, V 1024), wide layout,
    # 128-row tiles, kseg 1024, split 8; B = 9 at contexts 0..8 except one at
    # 600 (ceil(601 / 64) = 10 chunks -> 2 tasks), the others 1 task each.
    # Per layer: norm 9 (one per row), qkv (4 + 4) * 64 / 128 = 4 tiles x 2
    # K segments = 8, attn 2 * (8 + 2) = 20 (a pair's last task merges its
    # partials: no merge tasks), oproj 2 x 2 = 4, norm2 9, gateup 8 x 2 = 16,
    # down 2; then normf 9, lm 8, lmfin 1.
    tiles = dict(tile_qkv=128, chunk=64, tile_o=128, tile_gu=128, tile_down=128, kseg=1024, tile_lm=128,
                 split=8, wide=True, gseg=(2, 2, 2))
    ctx = [0, 1, 2, 3, 4, 5, 6, 7, 600]
    tasks = ot.expected_dense_tasks(wl.TINY, 9, ctx, tiles)
    fams = {}
    for f, l, i in tasks:
        fams[(f, l)] = fams.get((f, l), 0) + 1
    for l in range(2):
        assert {k[0]: v for k, v in fams.items() if k[1] == l} == {
            "norm": 9, "qkv": 8, "attn": 20, "oproj": 4, "norm2": 9, "gateup": 16, "down": 2}
    assert fams[("normf", -1)] == 9 and fams[("lm", -1)] == 8 and fams[("lmfin", -1)] == 1
    # the last sequence's two tasks per kv head: Hkv * 8 + g * 2 + c
    assert {i for f, l, i in tasks if f == "attn" and l == 0 and i >= 16} == {16, 17, 18, 19}


def test_moe_tiles_and_task_set_by_hand():
    # hist = [3, 0, 130, 64], tm = 64: expert 0 -> one tile of 3 rows; expert 2
    # -> tiles of 64, 64, 2 rows starting at rows 3, 67, 131; expert 3 -> one
    # tile of 64 rows at row 133.  5 tiles.
    assert ot.moe_tiles([3, 0, 130, 64], 64) == [(0, 0, 3), (2, 3, 64), (2, 67, 64), (2, 131, 2), (3, 133, 64)]
    # routing-aware heights: expert 2 (130 > 64 rows) -> tiles of 128, 2 rows;
    # expert 3 (exactly 64) keeps one 64-row tile
    assert ot.moe_tiles([3, 0, 130, 64], 64, big=128) == [(0, 0, 3), (2, 3, 128), (2, 131, 2), (3, 133, 64)]
    # T = 25 tokens: 4 route + 4 combine tasks; F = 1408, tn = 8 -> 176 gate/up
    # tasks per tile; H = 2048, td = 8 -> 256 down tasks per tile
    tasks = ot.expected_moe_tasks(25, [3, 0, 130, 64], 2048, 1408, {"tm": 64, "tn": 8, "td": 8})
    fams = {}
    for f, _, i in tasks:
        fams[f] = fams.get(f, 0) + 1
    assert fams == {"route": 4, "combine": 4, "mindptr": 1, "mfin": 1, "egu": 5 * 176, "edown": 5 * 256}
