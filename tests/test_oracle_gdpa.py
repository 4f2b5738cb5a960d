"""Pins for the GDPA oracle (oracle/gdpa.py): generalized dot-product
attention, the softmax replaced by GELU or SiLU ("GEM (Meta)", section
"Custom kernels").

Each pin checks the oracle against something other than its own code:
- a literal second implementation (math.erf / math.exp, exactly rounded
  sums, keys listed per query) on tiny inputs;
- the identity act(x) - act(-x) = x, true of both activations, which turns
  the difference of two GDPA calls into plain linear attention;
- PyTorch autograd through torch's own GELU / SiLU (fp64);
- central finite differences;
- independence of the examples, and single-key closed forms.
"""
import math

import numpy as np
import pytest
import torch

from oracle import gdpa


def _case(rng, lengths, H, D, scale=1.0):
    offs = np.zeros(len(lengths) + 1, dtype=np.int64)
    offs[1:] = np.cumsum(lengths)
    T = int(offs[-1])
    mk = lambda s: rng.standard_normal((T, H, D)) * s
    return offs, mk(scale), mk(scale), mk(1.0), mk(1.0)


def _lit_act(x, kind):
    if kind == "gelu":
        return 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))
    return x / (1.0 + math.exp(-x))


def _literal_fwd(offs, q, k, v, keys_of, kind, lit_act=_lit_act):
    """keys_of(e, i, L) lists the keys query i of example e sees."""
    T, H, D = q.shape
    out = np.zeros((T, H, D))
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        for h in range(H):
            for i in range(s1 - s0):
                keys = keys_of(e, i, s1 - s0)
                w = [lit_act(math.fsum(q[s0 + i, h, d] * k[s0 + j, h, d] for d in range(D)) / math.sqrt(D), kind)
                     for j in keys]
                for d in range(D):
                    out[s0 + i, h, d] = math.fsum(a * v[s0 + j, h, d] for a, j in zip(w, keys))
    return out


def _block_keys(block, window):
    return lambda e, i, L: list(range(max(0, i // block - (window - 1)) * block, i + 1))


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
@pytest.mark.parametrize("block,window", [(1, 3), (4, 1), (5, 2), (3, 100)])
def test_matches_literal_implementation(kind, block, window):
    rng = np.random.default_rng(700 + 10 * block + window + (1000 if kind == "silu" else 0))
    offs, q, k, v, _ = _case(rng, [13, 0, 9, 1], 2, 3, scale=1.5)
    got = gdpa.fwd(offs, q, k, v, block, window, kind)
    ref = _literal_fwd(offs, q, k, v, _block_keys(block, window), kind)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_odd_part_is_linear_attention(kind):
    """act(x) - act(-x) = x for GELU and SiLU, so out(q) - out(-q) is the
    masked linear attention sum_j s_ij v_j (no activation at all)."""
    rng = np.random.default_rng(601)
    offs, q, k, v, _ = _case(rng, [30, 17], 2, 8, scale=2.0)
    diff = gdpa.fwd(offs, q, k, v, 4, 2, kind) - gdpa.fwd(offs, -q, k, v, 4, 2, kind)
    lin = _literal_fwd(offs, q, k, v, _block_keys(4, 2), kind, lit_act=lambda x, _: x)
    np.testing.assert_allclose(diff, lin, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_gradients_match_torch_autograd(kind):
    rng = np.random.default_rng(602)
    block, window, H, D = 4, 2, 2, 8
    offs, q, k, v, do = _case(rng, [15, 0, 22], H, D, scale=1.5)
    dq, dk, dv = gdpa.bwd(offs, q, k, v, do, block, window, kind)
    out = gdpa.fwd(offs, q, k, v, block, window, kind)
    f = torch.nn.functional.gelu if kind == "gelu" else torch.nn.functional.silu
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        L = s1 - s0
        if L == 0:
            continue
        i = torch.arange(L)[:, None]
        j = torch.arange(L)[None, :]
        mask = ((j <= i) & (j // block >= i // block - (window - 1))).double()
        tq, tk, tv = (torch.tensor(x[s0:s1].transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
                      for x in (q, k, v))
        o = (f(tq @ tk.transpose(1, 2) / math.sqrt(D)) * mask) @ tv
        o.backward(torch.tensor(do[s0:s1].transpose(1, 0, 2)))
        t = lambda x: x.detach().numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(out[s0:s1], t(o), rtol=0, atol=1e-12)
        for name, got, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
            np.testing.assert_allclose(got[s0:s1], t(ref), rtol=0, atol=1e-11, err_msg=f"{name} e{e}")


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_finite_differences(kind):
    rng = np.random.default_rng(603)
    offs, q, k, v, do = _case(rng, [7, 5], 1, 3, scale=1.2)
    dq, dk, dv = gdpa.bwd(offs, q, k, v, do, 2, 2, kind)
    loss = lambda q_, k_, v_: float(np.sum(gdpa.fwd(offs, q_, k_, v_, 2, 2, kind) * do))
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            sub = lambda y: tuple(y if n == name else a for n, a in zip("qkv", args))
            num[idx] = (loss(*sub(xp)) - loss(*sub(xm))) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_activation_derivative(kind):
    x = np.linspace(-12, 12, 2001)
    h = 1e-5
    num = (gdpa.act(x + h, kind) - gdpa.act(x - h, kind)) / (2 * h)
    np.testing.assert_allclose(gdpa.act_grad(x, kind), num, rtol=0, atol=1e-8)
    # known values: GELU(1) = Phi(1), SiLU(1) = 1 / (1 + e^-1)
    ref = 0.5 * (1 + math.erf(1 / math.sqrt(2))) if kind == "gelu" else 1 / (1 + math.exp(-1))
    assert abs(float(gdpa.act(1.0, kind)) - ref) < 1e-15


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_examples_are_independent(kind):
    rng = np.random.default_rng(604)
    offs, q, k, v, do = _case(rng, [11, 19], 2, 4)
    a = gdpa.fwd(offs, q, k, v, 3, 2, kind), *gdpa.bwd(offs, q, k, v, do, 3, 2, kind)
    s = slice(11, 30)
    one = np.array([0, 19])
    b = gdpa.fwd(one, q[s], k[s], v[s], 3, 2, kind), *gdpa.bwd(one, q[s], k[s], v[s], do[s], 3, 2, kind)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x[s], y, rtol=0, atol=1e-13)


# ------------------------------------------------- cross / pooled attention ---

@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_cross_matches_literal_and_single_key(kind):
    rng = np.random.default_rng(605)
    qo = np.array([0, 6, 6, 10])                 # 3 examples; the second has no queries
    ko = np.array([0, 3, 7, 8])                  # short jagged key/value sets; the third has one key
    H, D = 2, 4
    q = rng.standard_normal((10, H, D)) * 1.5
    k = rng.standard_normal((8, H, D))
    v = rng.standard_normal((8, H, D))
    got = gdpa.cross_fwd(qo, ko, q, k, v, kind)
    ref = np.zeros_like(q)
    for e in range(3):
        for h in range(H):
            for i in range(qo[e], qo[e + 1]):
                w = [_lit_act(math.fsum(q[i, h, d] * k[j, h, d] for d in range(D)) / math.sqrt(D), kind)
                     for j in range(ko[e], ko[e + 1])]
                for d in range(D):
                    ref[i, h, d] = math.fsum(a * v[j, h, d] for a, j in zip(w, range(ko[e], ko[e + 1])))
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # one key: out_i = act(s_i0) v_0 exactly
    s = np.einsum("ihd,hd->ih", q[6:10], k[7]) / math.sqrt(D)
    np.testing.assert_allclose(got[6:10], gdpa.act(s, kind)[..., None] * v[7][None], rtol=0, atol=1e-14)


@pytest.mark.parametrize("kind", gdpa.ACTIVATIONS)
def test_cross_gradients_match_torch_autograd(kind):
    rng = np.random.default_rng(606)
    qo = np.array([0, 9, 14])
    ko = np.array([0, 4, 12])
    H, D = 2, 8
    q = rng.standard_normal((14, H, D)) * 1.5
    k = rng.standard_normal((12, H, D))
    v = rng.standard_normal((12, H, D))
    do = rng.standard_normal((14, H, D))
    dq, dk, dv = gdpa.cross_bwd(qo, ko, q, k, v, do, kind)
    f = torch.nn.functional.gelu if kind == "gelu" else torch.nn.functional.silu
    for e in range(2):
        a, b = slice(qo[e], qo[e + 1]), slice(ko[e], ko[e + 1])
        tq = torch.tensor(q[a].transpose(1, 0, 2), requires_grad=True)
        tk = torch.tensor(k[b].transpose(1, 0, 2), requires_grad=True)
        tv = torch.tensor(v[b].transpose(1, 0, 2), requires_grad=True)
        o = f(tq @ tk.transpose(1, 2) / math.sqrt(D)) @ tv
        o.backward(torch.tensor(do[a].transpose(1, 0, 2)))
        t = lambda x: x.detach().numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(dq[a], t(tq.grad), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk[b], t(tk.grad), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[b], t(tv.grad), rtol=0, atol=1e-11)


def test_pooled_attention_is_cross_attention_with_shared_seeds():
    """Pooled multi-head attention: the same seed queries for every example.
    Each example's pooled rows equal cross-attention of the seeds alone
    against that example's sequence."""
    rng = np.random.default_rng(607)
    H, D, n_seeds = 2, 4, 3
    seeds = rng.standard_normal((n_seeds, H, D))
    ko = np.array([0, 5, 5, 17])
    k = rng.standard_normal((17, H, D))
    v = rng.standard_normal((17, H, D))
    qo = np.arange(4) * n_seeds
    q = np.concatenate([seeds] * 3)
    got = gdpa.cross_fwd(qo, ko, q, k, v, "silu")
    for e in range(3):
        one = gdpa.cross_fwd(np.array([0, n_seeds]), np.array([0, ko[e + 1] - ko[e]]), seeds,
                             k[ko[e]:ko[e + 1]], v[ko[e]:ko[e + 1]], "silu")
        np.testing.assert_allclose(got[qo[e]:qo[e + 1]], one, rtol=0, atol=1e-14)
    assert not got[n_seeds:2 * n_seeds].any()     # an empty sequence pools to zero
