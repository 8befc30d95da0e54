"""Checks that pin the fp64 oracle to things other than itself.

Each function raises AssertionError when the oracle disagrees with what the
documentation pages or the mathematics fix: high-precision closed forms
(Python's decimal module at 50 digits), textbook/library routines (torch fp64
dense layers, torch's tanh-GELU and SiLU), brute force on tiny inputs and
invariants.  They are called by test_oracle_pins.py and, against deliberately
broken copies of the oracle, by test_oracle_mutants.py.
"""
import json
import math
import os
import random
from decimal import Decimal, getcontext

import numpy as np
import torch
import torch.nn.functional as F

import oracle

getcontext().prec = 50
GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))
C_GELU = GOLDEN["gelu_tanh_sqrt_2_over_pi"]["value"]
C_CUBIC = GOLDEN["gelu_tanh_cubic"]["value"]
ALPHA = GOLDEN["swigluoai_alpha"]["value"]
LIMIT = GOLDEN["swigluoai_limit"]["value"]


# ----------------------------------------------------------------- helpers
def d_exp(x):
    return Decimal(x).exp()


def d_sigmoid(x):
    return Decimal(1) / (Decimal(1) + d_exp(-Decimal(x)))


def d_tanh(x):
    e2 = d_exp(2 * Decimal(x))
    return (e2 - 1) / (e2 + 1)


def close(a, b, rel=1e-14, abs_=0.0):
    a, b = float(a), float(b)
    return abs(a - b) <= rel * abs(b) + abs_


def bf16(t):
    """Round a float tensor to bf16 and return (torch bf16 tensor, uint16 bits)."""
    tb = t.to(torch.bfloat16)
    return tb, tb.view(torch.int16).numpy().view(np.uint16)


def rand_layer(T, H, E, k, D, seed, bias=False, scale_w=0.2):
    g = torch.Generator().manual_seed(seed)
    x, xb = bf16(torch.randn(T, H, generator=g))
    Wgu, Wgub = bf16(torch.randn(E, H, 2 * D, generator=g) * scale_w)
    Wd, Wdb = bf16(torch.randn(E, D, H, generator=g) * scale_w)
    bgu = bgub = bd = bdb = None
    if bias:
        bgu, bgub = bf16(torch.randn(E, 2 * D, generator=g) * 0.3)
        bd, bdb = bf16(torch.randn(E, H, generator=g) * 0.3)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    w = torch.rand(T, k, generator=g, dtype=torch.float64)
    return dict(x=x, xb=xb, Wgu=Wgu, Wgub=Wgub, Wd=Wd, Wdb=Wdb, bgu=bgu, bgub=bgub, bd=bd, bdb=bdb,
                idx=idx, w=w)


# -------------------------------------------------------------- activations
def pin_activation_closed_forms():
    # gelu_tanh with the page's two constants, at hand-picked points.
    for g in (-3.0, -1.0, -0.25, 0.0, 0.5, 1.0, 2.0, 4.5):
        for u in (1.0, -0.75):
            dg = Decimal(g)
            ref = Decimal("0.5") * dg * (1 + d_tanh(Decimal(C_GELU) * (dg + Decimal(C_CUBIC) * dg ** 3))) * Decimal(u)
            got = oracle.activation("gelu_tanh", g, u)
            assert close(got, ref, 1e-14, 1e-300), ("gelu_tanh", g, u, got, ref)
    # swigluoai at g=2, u=0.5, alpha=1.702: 2 * sigmoid(3.404) * 1.5
    ref = Decimal(2) * d_sigmoid(Decimal("3.404")) * Decimal("1.5")
    got = oracle.activation("swigluoai", 2.0, 0.5, ALPHA, LIMIT)
    assert close(got, ref), ("swigluoai", got, ref)
    # clamps: gate 10 -> 7 (max only), up -9 -> -7, so 7 * sigmoid(11.914) * (-6)
    ref = Decimal(7) * d_sigmoid(Decimal("11.914")) * Decimal(-6)
    got = oracle.activation("swigluoai", 10.0, -9.0, ALPHA, LIMIT)
    assert close(got, ref), ("swigluoai clamp", got, ref)
    # gate is clamped from above only: g=-10 stays -10
    ref = Decimal(-10) * d_sigmoid(Decimal("-17.02")) * Decimal("1.5")
    got = oracle.activation("swigluoai", -10.0, 0.5, ALPHA, LIMIT)
    assert close(got, ref), ("swigluoai negative gate", got, ref)
    # silu: unclamped with limit 0, clamped with limit 7
    ref = Decimal(10) * d_sigmoid(10) * Decimal(-9)
    assert close(oracle.activation("silu", 10.0, -9.0, 0.0, 0.0), ref)
    ref = Decimal(7) * d_sigmoid(7) * Decimal(-7)
    assert close(oracle.activation("silu", 10.0, -9.0, 0.0, 7.0), ref)
    ref = Decimal(-2) * d_sigmoid(-2) * Decimal(3)
    assert close(oracle.activation("silu", -2.0, 3.0, 0.0, 7.0), ref)


def pin_activation_library_routines():
    g = torch.linspace(-8, 8, 401, dtype=torch.float64)
    u = torch.linspace(-3, 5, 401, dtype=torch.float64)
    got = torch.tensor([oracle.activation("gelu_tanh", float(a), float(b)) for a, b in zip(g, u)], dtype=torch.float64)
    assert torch.allclose(got, F.gelu(g, approximate="tanh") * u, rtol=1e-13, atol=1e-14)
    got = torch.tensor([oracle.activation("silu", float(a), float(b)) for a, b in zip(g, u)], dtype=torch.float64)
    assert torch.allclose(got, F.silu(g) * u, rtol=1e-13, atol=1e-14)
    # swigluoai with alpha = 1 and no clamp is silu(g) * (u + 1)
    got = torch.tensor([oracle.activation("swigluoai", float(a), float(b), 1.0, 0.0) for a, b in zip(g, u)], dtype=torch.float64)
    assert torch.allclose(got, F.silu(g) * (u + 1), rtol=1e-13, atol=1e-14)
    # the tanh form stays within 1e-3 of the exact (erf) GELU
    got = torch.tensor([oracle.activation("gelu_tanh", float(a), 1.0) for a in g])
    assert (got - F.gelu(g)).abs().max() < 1e-3
    assert abs(C_GELU - math.sqrt(2 / math.pi)) < 1e-16


# ---------------------------------------------------------- softmax router
def pin_softmax_router():
    z = np.array([[1.0, 3.0, 2.0, 3.0]], np.float32)
    idx, w = oracle.route_softmax_topk(z, 4, 2)
    assert idx.tolist() == [[1, 3]], idx            # tie -> lower index first
    assert np.allclose(w, 0.5, rtol=0, atol=1e-15)
    z = np.log(np.array([[1.0, 2.0, 3.0, 4.0]])).astype(np.float32)
    idx, w = oracle.route_softmax_topk(z, 4, 3)
    assert idx.tolist() == [[3, 2, 1]]
    e = np.exp(z.astype(np.float64)[0, [3, 2, 1]])
    assert np.allclose(w[0], e / e.sum(), rtol=1e-15)
    assert abs(w[0, 0] - 4 / 9) < 1e-7 and abs(w[0, 2] - 2 / 9) < 1e-7
    # random: equals the full softmax restricted to the top-k and renormalised
    g = torch.Generator().manual_seed(3)
    for E, k in ((8, 2), (37, 5), (128, 4)):
        zt = torch.randn(50, E + 3, generator=g) * 2
        idx, w = oracle.route_softmax_topk(zt.numpy(), E, k)
        p = torch.softmax(zt[:, :E].double(), dim=-1)
        top = torch.topk(zt[:, :E], k, dim=-1)
        assert (torch.from_numpy(idx).long() == top.indices).all()
        ref = torch.gather(p, 1, top.indices)
        ref = ref / ref.sum(-1, keepdim=True)
        assert torch.allclose(torch.from_numpy(w), ref, rtol=1e-13, atol=0)
    # bf16 logits are read as their exact values
    zb = torch.randn(7, 16, generator=g).to(torch.bfloat16)
    i1, w1 = oracle.route_softmax_topk(zb.view(torch.int16).numpy().view(np.uint16), 16, 3)
    i2, w2 = oracle.route_softmax_topk(zb.float().numpy(), 16, 3)
    assert (i1 == i2).all() and (w1 == w2).all()


# ------------------------------------------------------------- sink router
def d_sink_weights(z_sel, z_sink, scale):
    s = [d_sigmoid(z) for z in list(z_sel) + list(z_sink)]
    # equal to sigmoid_i / sum sigmoid_j; for very negative z use exp(z)
    # ratios, which is the same quantity to 50 digits
    tot = sum(s)
    return [float(v / tot * Decimal(scale)) for v in s]


def d_sink_weights_logspace(z_all, scale):
    # log sigmoid(z) = z - ln(1 + e^z): exact in decimal even where the
    # sigmoid underflows double precision
    ls = [Decimal(z) - (1 + d_exp(Decimal(z))).ln() for z in z_all]
    m = max(ls)
    ex = [(v - m).exp() for v in ls]
    tot = sum(ex)
    return [float(v / tot * Decimal(scale)) for v in ex]


def pin_sink_router():
    # hand example: selection uses sigmoid(z) + b, not z + b
    z = np.array([[5.0, 4.0, -1.0, 0.0, 0.5, 0.25]], np.float32)   # E=4, S=2
    b = np.array([0.0, 0.05, 0.0, 0.0], np.float32)
    idx, w, sw = oracle.route_sigmoid_sink(z, 4, 2, 1, b, 2.5, 1.0)
    assert idx.tolist() == [[1]], idx    # sigmoid(4)+0.05 = 1.032 > sigmoid(5) = 0.9933
    ref = d_sink_weights([4.0], [0.5, 0.25], 2.5)    # raw (unbiased) logit of the selected expert
    assert close(w[0, 0], ref[0]) and close(sw[0, 0], ref[1]) and close(sw[0, 1], ref[2])
    # random moderate logits: sigmoid_i / sum_j sigmoid_j, scaled
    g = torch.Generator().manual_seed(5)
    E, S, k = 16, 2, 6
    zt = (torch.randn(20, E + S + 3, generator=g) * 3).numpy()
    zt[:, E + S:] = np.nan                                 # a wider row's tail is never read
    bias = (torch.rand(E, generator=g) * 0.2 - 0.1).numpy()
    idx, w, sw = oracle.route_sigmoid_sink(zt, E, S, k, bias, 2.5, 0.8)
    for t in range(20):
        ref = d_sink_weights([float(zt[t, e]) for e in idx[t]], [float(v) for v in zt[t, E:E + S]], 2.0)
        got = list(w[t]) + list(sw[t])
        assert all(close(a, r, 1e-13) for a, r in zip(got, ref)), (t, got, ref)
        assert close(sum(got), 2.0, 1e-14)                # route_scale * global_scale
        # selection: top-k of the float score, descending, ties to lower index
        sig = (1.0 / (1.0 + np.exp(-zt[t, :E].astype(np.float64)))).astype(np.float32)
        score = sig + bias
        order = sorted(range(E), key=lambda e: (-float(score[e]), e))[:k]
        assert idx[t].tolist() == order
    # extreme logits where sigmoid underflows double: log-space form stays finite
    z = np.array([[-800.0, -801.0, -790.0, -805.0, -799.0, -900.0]], np.float64).astype(np.float32)
    idx, w, sw = oracle.route_sigmoid_sink(z, 4, 2, 2, None, 1.0, 1.0)
    assert idx.tolist() == [[0, 1]]     # every sigmoid rounds to 0 in float: ties -> lowest indices
    ref = d_sink_weights_logspace([-800.0, -801.0, -799.0, -900.0], 1.0)
    got = list(w[0]) + list(sw[0])
    assert all(close(a, r, 1e-12) for a, r in zip(got, ref)), (got, ref)
    z = np.array([[80.0, -80.0, 3.0, 60.0, -80.0]], np.float32)
    idx, w, sw = oracle.route_sigmoid_sink(z, 4, 1, 2, None, 1.0, 1.0)
    ref = d_sink_weights_logspace([float(z[0, e]) for e in idx[0]] + [-80.0], 1.0)
    assert all(close(a, r, 1e-12, 1e-300) for a, r in zip(list(w[0]) + list(sw[0]), ref))
    # bias changes the selection but never the weight values
    zt = (torch.randn(30, 10, generator=g)).numpy()
    i0, w0, s0 = oracle.route_sigmoid_sink(zt, 8, 2, 3, None, 1.5, 1.0)
    b = np.zeros(8, np.float32)
    i1, w1, s1 = oracle.route_sigmoid_sink(zt, 8, 2, 3, b + 0.0, 1.5, 1.0)
    assert (i0 == i1).all() and (w0 == w1).all() and (s0 == s1).all()
    b = np.full(8, 0.125, np.float32)                     # uniform shift: same set
    i2, w2, s2 = oracle.route_sigmoid_sink(zt, 8, 2, 3, b, 1.5, 1.0)
    assert (i0 == i2).all() and (w0 == w2).all() and (s0 == s2).all()
    b = np.zeros(8, np.float32); b[7] = 2.0               # forces expert 7 into every set
    i3, w3, s3 = oracle.route_sigmoid_sink(zt, 8, 2, 3, b, 1.5, 1.0)
    assert (i3[:, 0] == 7).all()
    ref = [d_sink_weights([float(zt[t, e]) for e in i3[t]], [float(zt[t, 8]), float(zt[t, 9])], 1.5) for t in range(30)]
    assert np.allclose(np.concatenate([w3, s3], 1), np.array(ref), rtol=1e-13, atol=0)
    # all-equal scores: ties go to the lowest indices
    idx, _, _ = oracle.route_sigmoid_sink(np.zeros((1, 7), np.float32), 5, 2, 3, None)
    assert idx.tolist() == [[0, 1, 2]]


# ---------------------------------------------------------------------- CSR
def pin_csr():
    g = torch.Generator().manual_seed(7)
    for T, E, k in ((1, 1, 1), (13, 5, 2), (200, 16, 4), (64, 8, 8)):
        idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32).numpy()
        counts, offsets, perm, inv = oracle.create_indices(idx, E)
        flat = idx.reshape(-1)
        assert (counts == np.bincount(flat, minlength=E)).all()
        assert counts.sum() == T * k
        assert offsets[0] == 0 and (np.diff(offsets) == counts).all()
        ref = sorted(range(flat.size), key=lambda s: (flat[s], s))
        assert perm.tolist() == ref
        assert (inv[perm] == np.arange(flat.size)).all()
    # all slots on one expert: every other segment empty
    idx = np.full((9, 1), 3, np.int32)
    counts, offsets, perm, _ = oracle.create_indices(idx, 6)
    assert counts.tolist() == [0, 0, 0, 9, 0, 0] and offsets.tolist() == [0, 0, 0, 0, 9, 9, 9]
    assert perm.tolist() == list(range(9))
    try:
        oracle.create_indices(np.array([[0, 6]], np.int32), 6)
        raise AssertionError("out-of-range index accepted")
    except ValueError:
        pass


# ---------------------------------------------------------------------- FFN
def dense_ffn(x, Wg, Wu, Wd, act, alpha=0.0, limit=0.0, bg=None, bu=None, bd=None):
    """A textbook gated MLP in torch fp64 with torch's own activations."""
    g = x @ Wg + (0 if bg is None else bg)
    u = x @ Wu + (0 if bu is None else bu)
    if limit > 0:
        g = torch.clamp(g, max=limit)
        u = torch.clamp(u, -limit, limit)
    if act == "silu":
        h = F.silu(g) * u
    elif act == "gelu_tanh":
        h = F.gelu(g, approximate="tanh") * u
    else:
        h = g * torch.sigmoid(alpha * g) * (u + 1)
    return h @ Wd + (0 if bd is None else bd)


def pin_ffn_dense_reduction():
    """top_k = 1 with every expert identical equals one dense gated FFN."""
    g = torch.Generator().manual_seed(11)
    T, H, E, D = 9, 24, 3, 16
    x, xb = bf16(torch.randn(T, H, generator=g))
    one_gu, _ = bf16(torch.randn(H, 2 * D, generator=g) * 0.3)
    one_d, _ = bf16(torch.randn(D, H, generator=g) * 0.3)
    bgu, _ = bf16(torch.randn(2 * D, generator=g) * 0.2)
    bd, _ = bf16(torch.randn(H, generator=g) * 0.2)
    Wgu = one_gu.expand(E, H, 2 * D).contiguous()
    Wd = one_d.expand(E, D, H).contiguous()
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    idx = (torch.arange(T) % E).to(torch.int32).reshape(T, 1).numpy()
    w = np.ones((T, 1))
    X, G, U, Dn = x.double(), one_gu[:, :D].double(), one_gu[:, D:].double(), one_d.double()
    for act, alpha, limit in (("silu", 0.0, 0.0), ("silu", 0.0, 0.5), ("gelu_tanh", 0.0, 0.0),
                              ("swigluoai", ALPHA, LIMIT), ("swigluoai", ALPHA, 0.3)):
        got = oracle.expert_ffn(xb, idx, w, bits(Wgu), bits(Wd), activation=act, alpha=alpha, limit=limit)
        ref = dense_ffn(X, G, U, Dn, act, alpha, limit)
        assert torch.allclose(torch.from_numpy(got), ref, rtol=1e-12, atol=1e-12), act
        # with biases
        got = oracle.expert_ffn(xb, idx, w, bits(Wgu), bits(Wd), bits(bgu.expand(E, 2 * D)),
                                bits(bd.expand(E, H)), activation=act, alpha=alpha, limit=limit)
        ref = dense_ffn(X, G, U, Dn, act, alpha, limit, bgu[:D].double(), bgu[D:].double(), bd.double())
        assert torch.allclose(torch.from_numpy(got), ref, rtol=1e-12, atol=1e-12), act + "+bias"


def brute_force_layer(L, act, fmt, alpha=0.0, limit=0.0):
    """Per-token loop over the selected experts, each a dense torch fp64 MLP."""
    T, k = L["idx"].shape
    D = L["Wgu"].shape[2] // 2
    out = torch.zeros(T, L["x"].shape[1], dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(L["idx"][t, j])
            W = L["Wgu"][e].double()
            bgu = None if L["bgu"] is None else L["bgu"][e].double()
            if fmt == "concatenated":
                Wg, Wu = W[:, :D], W[:, D:]
                bg, bu = (None, None) if bgu is None else (bgu[:D], bgu[D:])
            else:
                Wg, Wu = W[:, 0::2], W[:, 1::2]
                bg, bu = (None, None) if bgu is None else (bgu[0::2], bgu[1::2])
            bd = None if L["bd"] is None else L["bd"][e].double()
            y = dense_ffn(L["x"][t:t + 1].double(), Wg, Wu, L["Wd"][e].double(), act, alpha, limit, bg, bu, bd)
            out[t] += float(L["w"][t, j]) * y[0]
    return out


def pin_ffn_brute_force():
    for fmt, act, alpha, limit, bias in (("concatenated", "silu", 0.0, 0.0, False),
                                         ("interleaved", "swigluoai", ALPHA, LIMIT, True),
                                         ("concatenated", "gelu_tanh", 0.0, 0.0, True),
                                         ("interleaved", "silu", 0.0, 0.4, False)):
        L = rand_layer(T=6, H=16, E=4, k=2, D=8, seed=13, bias=bias)
        got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"],
                                fmt, act, alpha, limit)
        ref = brute_force_layer(L, act, fmt, alpha, limit)
        assert torch.allclose(torch.from_numpy(got), ref, rtol=1e-12, atol=1e-12), (fmt, act)


def pin_ffn_invariants():
    L = rand_layer(T=12, H=16, E=5, k=3, D=8, seed=17, bias=True)
    args = dict(gate_up_format="concatenated", activation="swigluoai", alpha=ALPHA, limit=LIMIT)
    base = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"], **args)
    # token permutation equivariance
    p = torch.randperm(12, generator=torch.Generator().manual_seed(1)).numpy()
    got = oracle.expert_ffn(L["xb"][p], L["idx"].numpy()[p], L["w"].numpy()[p], L["Wgub"], L["Wdb"], L["bgub"], L["bdb"], **args)
    assert np.array_equal(got, base[p])
    # expert relabelling equivariance
    q = torch.randperm(5, generator=torch.Generator().manual_seed(2)).numpy()     # new label of old expert e is q[e]
    inv_q = np.argsort(q)
    got = oracle.expert_ffn(L["xb"], q[L["idx"].numpy()].astype(np.int32), L["w"].numpy(), L["Wgub"][inv_q],
                            L["Wdb"][inv_q], L["bgub"][inv_q], L["bdb"][inv_q], **args)
    assert np.allclose(got, base, rtol=1e-13, atol=1e-13)
    # concatenated and interleaved layouts of the same expert give the same layer
    D = 8
    perm_cols = np.empty(2 * D, np.int64)
    perm_cols[0::2] = np.arange(D)
    perm_cols[1::2] = D + np.arange(D)
    got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), np.ascontiguousarray(L["Wgub"][:, :, perm_cols]),
                            L["Wdb"], np.ascontiguousarray(L["bgub"][:, perm_cols]), L["bdb"],
                            "interleaved", "swigluoai", ALPHA, LIMIT)
    assert np.allclose(got, base, rtol=1e-13, atol=1e-13)
    # a token subset gives exactly those rows
    sel = np.array([5, 0, 11, 5])
    got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"],
                            tokens=sel, **args)
    assert np.array_equal(got, base[sel])
    # the down bias is weighted by the routing weight: W_d = 0 leaves sum_j w_j b_d[e_j]
    zeros_d = np.zeros_like(L["Wdb"])
    got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], zeros_d, L["bgub"], L["bdb"], **args)
    bd = L["bd"].double().numpy()
    ref = np.einsum("tk,tkh->th", L["w"].numpy(), bd[L["idx"].numpy()])
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-14)
    # the gate_up bias enters before the activation: W_gu = 0 leaves act(b_g, b_u) . W_d + b_d
    zeros_gu = np.zeros_like(L["Wgub"])
    got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), zeros_gu, L["Wdb"], L["bgub"], L["bdb"], **args)
    bg = L["bgu"].double()
    h = dense_ffn(torch.ones(1, 1, dtype=torch.float64), bg[:, None, :D], bg[:, None, D:],
                  L["Wd"].double(), "swigluoai", ALPHA, LIMIT, bd=L["bd"].double()[:, None, :])[:, 0, :]
    ref = np.einsum("tk,tkh->th", L["w"].numpy(), h.numpy()[L["idx"].numpy()])
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-13)


def pin_ffn_empty_experts():
    """An expert that no token selects contributes nothing, even if its weights are NaN."""
    L = rand_layer(T=8, H=16, E=6, k=2, D=8, seed=19)
    idx = L["idx"].numpy() % 3                            # experts 3..5 are never chosen
    idx[:, 1] = (idx[:, 0] + 1) % 3
    Wgu, Wd = L["Wgub"].copy(), L["Wdb"].copy()
    nan_bits = np.uint16(0x7FC0)
    Wgu[3:] = nan_bits
    Wd[3:] = nan_bits
    got = oracle.expert_ffn(L["xb"], idx, L["w"].numpy(), Wgu, Wd)
    ref = oracle.expert_ffn(L["xb"], idx, L["w"].numpy(), L["Wgub"], L["Wdb"])
    assert np.isfinite(got).all() and np.array_equal(got, ref)


def brute_force_weight_first(L, act, fmt, alpha=0.0, limit=0.0):
    """Per-token loop: sum_j FFN_e(w_j * x[t]) with dense torch fp64 MLPs."""
    T, k = L["idx"].shape
    D = L["Wgu"].shape[2] // 2
    out = torch.zeros(T, L["x"].shape[1], dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(L["idx"][t, j])
            W = L["Wgu"][e].double()
            Wg, Wu = (W[:, :D], W[:, D:]) if fmt == "concatenated" else (W[:, 0::2], W[:, 1::2])
            bgu = None if L["bgu"] is None else L["bgu"][e].double()
            bg, bu = (None, None) if bgu is None else ((bgu[:D], bgu[D:]) if fmt == "concatenated"
                                                       else (bgu[0::2], bgu[1::2]))
            bd = None if L["bd"] is None else L["bd"][e].double()
            xin = float(L["w"][t, j]) * L["x"][t:t + 1].double()
            out[t] += dense_ffn(xin, Wg, Wu, L["Wd"][e].double(), act, alpha, limit, bg, bu, bd)[0]
    return out


def pin_weight_first():
    """apply_router_weight_first: the weight scales the input, so the down bias is unweighted."""
    for fmt, act, alpha, limit, bias in (("concatenated", "silu", 0.0, 0.0, True),
                                         ("interleaved", "swigluoai", ALPHA, LIMIT, True),
                                         ("concatenated", "gelu_tanh", 0.0, 0.0, False)):
        L = rand_layer(T=6, H=16, E=4, k=2, D=8, seed=23, bias=bias)
        got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"],
                                fmt, act, alpha, limit, weight_first=True)
        ref = brute_force_weight_first(L, act, fmt, alpha, limit)
        assert torch.allclose(torch.from_numpy(got), ref, rtol=1e-12, atol=1e-12), (fmt, act)
    # with every weight 1 the two orders agree
    L = rand_layer(T=5, H=16, E=4, k=2, D=8, seed=24, bias=True)
    ones = np.ones((5, 2))
    a = oracle.expert_ffn(L["xb"], L["idx"].numpy(), ones, L["Wgub"], L["Wdb"], L["bgub"], L["bdb"], weight_first=True)
    b = oracle.expert_ffn(L["xb"], L["idx"].numpy(), ones, L["Wgub"], L["Wdb"], L["bgub"], L["bdb"])
    assert np.array_equal(a, b)


def pin_token_mask():
    L = rand_layer(T=10, H=16, E=4, k=2, D=8, seed=25, bias=True)
    mask = np.array([1, 0, 1, 1, 0, 0, 1, 1, 1, 0], np.uint8)
    full = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"])
    got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"],
                            token_mask=mask)
    assert np.array_equal(got[mask == 1], full[mask == 1])       # valid tokens unchanged
    assert (got[mask == 0] == 0).all()                           # masked tokens give zero rows
    none = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"],
                             token_mask=np.zeros(10, np.uint8))
    assert (none == 0).all()


def pin_shared_experts():
    """One shared expert with gate 1 adds one dense gated MLP (torch fp64)."""
    g = torch.Generator().manual_seed(26)
    T, H, Ds = 7, 24, 16
    x, xb = bf16(torch.randn(T, H, generator=g))
    Wgu, Wgub = bf16(torch.randn(1, H, 2 * Ds, generator=g) * 0.3)
    Wd, Wdb = bf16(torch.randn(1, Ds, H, generator=g) * 0.3)
    got = oracle.shared_expert_ffn(xb, np.ones((T, 1)), Wgub, Wdb, activation="silu")
    ref = dense_ffn(x.double(), Wgu[0, :, :Ds].double(), Wgu[0, :, Ds:].double(), Wd[0].double(), "silu")
    assert torch.allclose(torch.from_numpy(got), ref, rtol=1e-12, atol=1e-12)
    # gates scale the shared outputs (sink lanes are gated shared experts)
    gates = np.linspace(0.1, 1.3, T).reshape(T, 1)
    got = oracle.shared_expert_ffn(xb, gates, Wgub, Wdb, activation="silu")
    assert torch.allclose(torch.from_numpy(got), ref * torch.from_numpy(gates), rtol=1e-12, atol=1e-12)


def pin_random_brute_force():
    """Seeded random shapes and options, each part against its brute-force
    form: the FFN (with the router weight first and a token mask on some
    draws) against the per-token loop of dense torch MLPs, the sink router
    against the decimal sigma_i / sum sigma_j with a sorted selection, the
    softmax router on tie-prone logits against a sort by (-z, e) and the
    renormalised exponentials, the CSR against a sort by (expert, slot)."""
    r = random.Random(2024)
    for case in range(150):
        T, H, E, D = r.randint(1, 8), r.randint(1, 20), r.randint(1, 6), r.randint(1, 10)
        k = r.randint(1, E)
        fmt = r.choice(["concatenated", "interleaved"])
        act = r.choice(["silu", "swigluoai", "gelu_tanh"])
        alpha = ALPHA if act == "swigluoai" else 0.0
        limit = 0.0 if act == "gelu_tanh" else r.choice([0.0, 0.3, LIMIT])
        L = rand_layer(T=T, H=H, E=E, k=k, D=D, seed=1000 + case, bias=r.random() < 0.5)
        weight_first = r.random() < 0.3
        mask = np.array([r.random() < 0.7 for _ in range(T)], np.uint8) if r.random() < 0.3 else None
        got = oracle.expert_ffn(L["xb"], L["idx"].numpy(), L["w"].numpy(), L["Wgub"], L["Wdb"], L["bgub"], L["bdb"],
                                fmt, act, alpha, limit, weight_first=weight_first, token_mask=mask)
        ref = (brute_force_weight_first if weight_first else brute_force_layer)(L, act, fmt, alpha, limit)
        if mask is not None:
            ref[torch.from_numpy(mask == 0)] = 0.0        # a masked token's row is zero
        assert torch.allclose(torch.from_numpy(got), ref, rtol=1e-12, atol=1e-12), (case, fmt, act, limit)
    g = torch.Generator().manual_seed(2025)
    for case in range(60):
        E, S = r.randint(1, 40), r.randint(0, 4)
        k = r.randint(1, E)
        scale, gscale = r.choice([0.5, 1.0, 2.5]), r.choice([1.0, 0.7])
        zt = (torch.randn(6, E + S, generator=g) * r.choice([0.5, 2.0, 6.0])).numpy()
        bias = (torch.rand(E, generator=g) * 0.2 - 0.1).numpy() if r.random() < 0.7 else None
        idx, w, sw = oracle.route_sigmoid_sink(zt, E, S, k, bias, scale, gscale)
        sig = (1.0 / (1.0 + np.exp(-zt[:, :E].astype(np.float64)))).astype(np.float32)
        score = sig + (0 if bias is None else bias)
        for t in range(6):
            assert idx[t].tolist() == sorted(range(E), key=lambda e: (-float(score[t, e]), e))[:k], (case, t)
            ref = d_sink_weights_logspace([float(zt[t, e]) for e in idx[t]] + [float(v) for v in zt[t, E:]],
                                          scale * gscale)
            got = list(w[t]) + list(sw[t])
            assert all(close(a, b, 1e-12, 1e-300) for a, b in zip(got, ref)), (case, t, got, ref)
        # softmax top-k on logits with frequent ties (few distinct values):
        # descending, ties to the lowest index, softmax over the selected
        zt = torch.randint(-3, 4, (6, E), generator=g).float().numpy() * r.choice([0.5, 1.0])
        idx, w = oracle.route_softmax_topk(zt, E, k)
        for t in range(6):
            sel = sorted(range(E), key=lambda e: (-float(zt[t, e]), e))[:k]
            assert idx[t].tolist() == sel, (case, t)
            ex = np.exp(zt[t, sel].astype(np.float64) - zt[t, sel].max())
            assert np.allclose(w[t], ex / ex.sum(), rtol=1e-14, atol=0), (case, t)
        T = r.randint(1, 60)
        idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32).numpy()
        counts, offsets, perm, inv = oracle.create_indices(idx, E)
        flat = idx.reshape(-1)
        assert perm.tolist() == sorted(range(flat.size), key=lambda s: (flat[s], s))
        assert offsets.tolist() == [0] + np.cumsum(np.bincount(flat, minlength=E)).tolist()
        assert (inv[perm] == np.arange(flat.size)).all()


ALL_PINS = [pin_activation_closed_forms, pin_activation_library_routines, pin_softmax_router, pin_sink_router,
            pin_csr, pin_ffn_dense_reduction, pin_ffn_brute_force, pin_ffn_invariants, pin_ffn_empty_experts,
            pin_weight_first, pin_token_mask, pin_shared_experts, pin_random_brute_force]
