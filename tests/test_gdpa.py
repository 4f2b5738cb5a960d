"""GPU parity of generalized dot-product attention (ba_gdpa_fwd / ba_gdpa_bwd,
called through the C ABI) against the fp64 oracle in oracle/gdpa.py.

GDPA replaces the softmax with an activation such as GELU or SiLU ("GEM
(Meta)", section "Custom kernels"); the reading implemented on both sides:
out_i = sum over visible j of act(q_i . k_j / sqrt(D)) v_j under the block
rule, no normalisation. The activation values fed to the P V product and
their derivatives fed to dS are rounded to bf16, like the softmax path's
probabilities, so the tolerances are the project's bf16 ones (parity_util):
max-abs 2e-2 and relative L2 1e-2 on out, dq, dk, dv, the max-abs bound
taken relative to max(1, max|ref|) on peaked inputs whose outputs run to
tens or hundreds (no normalisation keeps them small).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs
from oracle import gdpa as G
from parity_util import check_bf16, f64

pytestmark = pytest.mark.gpu

CASES = [
    # (head_dim, block, window, lengths)
    (128, 256, 2, [64, 4096, 1000, 257, 129]),      # the jagged long-history shapes, reduced batch
    (64, 128, 2, [1024, 1024, 0, 300]),
    (128, 64, 1, [0, 1, 127, 128, 129, 383]),       # independent 64-token blocks
    (64, 100, 3, [1, 99, 250, 640]),
]


def run_gpu(inp, block, window, act):
    q, k, v, dout = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].cuda()
    out = ba.gdpa_fwd(q, k, v, offs, block, window, act)
    dq, dk, dv = ba.gdpa_bwd(q, k, v, dout, offs, block, window, act)
    torch.cuda.synchronize()
    return {n: t.cpu() for n, t in dict(out=out, dq=dq, dk=dk, dv=dv).items()}


def run_oracle(inp, block, window, act):
    args = (inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    out = G.fwd(*args, block, window, act)
    dq, dk, dv = G.bwd(*args, f64(inp["dout"]), block, window, act)
    return dict(out=out, dq=dq, dk=dk, dv=dv)


@pytest.mark.parametrize("act", ["gelu", "silu"])
@pytest.mark.parametrize("head_dim,block,window,lengths", CASES)
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_gdpa_matches_oracle(act, head_dim, block, window, lengths, peaked):
    w = CONFIGS[3].replace(head_dim=head_dim, block=block, window=window, heads=2, batch=len(lengths))
    q_gain = 1.0
    if peaked:
        w = w.replace(qkv_scale=1.0)
        q_gain = 3.0
    inp = make_inputs(w, q_gain=q_gain, lengths=lengths, seed=300 + head_dim + block)
    got = run_gpu(inp, block, window, act)
    ref = run_oracle(inp, block, window, act)
    for n in ("out", "dq", "dk", "dv"):
        check_bf16(f"{act} {n}", got[n], ref[n], peaked=peaked)


def test_gdpa_examples_are_isolated_and_deterministic():
    """Examples do not see each other (a jagged batch equals its examples run
    one by one, bit for bit), and a second call gives the same bits."""
    w = CONFIGS[3].replace(heads=2, batch=3)
    lengths = [300, 129, 700]
    inp = make_inputs(w, lengths=lengths, seed=11)
    got = run_gpu(inp, w.block, w.window, "gelu")
    again = run_gpu(inp, w.block, w.window, "gelu")
    offs = inp["seq_offsets"].numpy()
    for n in got:
        assert torch.equal(got[n], again[n]), n
    for e in range(3):
        sl = slice(int(offs[e]), int(offs[e + 1]))
        one = {n: inp[n][sl].clone() for n in ("q", "k", "v", "dout")}
        one["seq_offsets"] = torch.tensor([0, lengths[e]], dtype=torch.int32)
        alone = run_gpu(one, w.block, w.window, "gelu")
        for n in got:
            assert torch.equal(got[n][sl], alone[n]), (e, n)


def _poison(t, s0, n):
    pattern = torch.tensor([float("inf"), float("nan"), float("-inf")], dtype=t.dtype)
    rows = t[s0:s0 + n]
    rows.copy_(pattern.repeat(rows.numel() // 3 + 1)[: rows.numel()].view_as(rows))


@pytest.mark.parametrize("act", ["gelu", "silu"])
def test_gdpa_examples_are_isolated_from_non_finite_neighbours(act):
    """Inf / NaN in the first rows of a neighbour's q, k, v and dout (or in all
    of a short example's rows) leave every other example's out, dq, dk and dv
    bit-equal to a clean run: the partial tiles at example ends never multiply
    a neighbour's rows by zero activations."""
    lengths = [300, 200, 1000, 129, 777, 90, 128, 5]
    w = CONFIGS[3].replace(heads=2, batch=len(lengths))
    inp = make_inputs(w, lengths=lengths, seed=4343)
    offs = inp["seq_offsets"].numpy()
    poisoned = {1: 40, 3: lengths[3], 5: lengths[5], 7: lengths[7]}
    dirty = dict(inp)
    for n in ("q", "k", "v", "dout"):
        dirty[n] = inp[n].clone()
        for e, rows in poisoned.items():
            _poison(dirty[n], int(offs[e]), rows)
    clean = run_gpu(inp, w.block, w.window, act)
    got = run_gpu(dirty, w.block, w.window, act)
    ref = run_oracle(inp, w.block, w.window, act)
    for e in range(len(lengths)):
        if e in poisoned:
            continue
        sl = slice(int(offs[e]), int(offs[e + 1]))
        for n in ("out", "dq", "dk", "dv"):
            assert torch.equal(got[n][sl], clean[n][sl]), f"example {e} {n} changed by a neighbour"
            check_bf16(f"{act} e{e} {n}", got[n][sl], ref[n][sl])


def test_gdpa_rejects_fp32_and_unknown_activations():
    q = torch.zeros((128, 2, 64), device="cuda")
    offs = torch.tensor([0, 128], dtype=torch.int32, device="cuda")
    prob = ba.make_problem(q, offs)
    ws = ba.workspace_for(ba.ba_gdpa_workspace_size(prob, 64, 1), q.device)
    assert ba.ba_gdpa_fwd(prob, "gelu", q, q, q, offs, 64, 1, q.clone(), ws) == ba.BA_ERR_UNSUPPORTED
    qb = q.to(torch.bfloat16)
    prob = ba.make_problem(qb, offs)
    assert ba.ba_gdpa_fwd(prob, 7, qb, qb, qb, offs, 64, 1, qb.clone(), ws) == ba.BA_ERR_INVALID_ARG


# ----------------------------------------------------- cross-attention ---
# Example b's queries against every key of its own key/value set
# (oracle/gdpa.py cross_fwd / cross_bwd): GEM's cross- and pooled attention,
# the short-key/value case. Query and key/value sets are jagged separately,
# with empty sets on either side.

CROSS = [
    # (head_dim, query lengths, key/value lengths)
    (128, [300, 1, 1000, 0, 129], [64, 200, 17, 50, 0]),
    (64, [256, 700, 33], [128, 1, 300]),
    (128, [64, 64, 64, 64], [500, 128, 129, 1]),   # pooled shape: few seeds per example, longer sequences
]


def _cross_inputs(head_dim, lq, lk, seed, scale):
    g = torch.Generator().manual_seed(seed)
    H = 2
    q = (torch.randn(sum(lq), H, head_dim, generator=g) * scale).to(torch.bfloat16)
    k = (torch.randn(sum(lk), H, head_dim, generator=g) * scale).to(torch.bfloat16)
    v = (torch.randn(sum(lk), H, head_dim, generator=g) * scale).to(torch.bfloat16)
    dout = torch.randn(sum(lq), H, head_dim, generator=g).to(torch.bfloat16)
    qo = torch.tensor([0, *np.cumsum(lq)], dtype=torch.int32)
    ko = torch.tensor([0, *np.cumsum(lk)], dtype=torch.int32)
    return q, k, v, dout, qo, ko


@pytest.mark.parametrize("act", ["gelu", "silu"])
@pytest.mark.parametrize("head_dim,lq,lk", CROSS)
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_gdpa_cross_matches_oracle(act, head_dim, lq, lk, peaked):
    q, k, v, dout, qo, ko = _cross_inputs(head_dim, lq, lk, 77 + head_dim, 1.0 if peaked else head_dim ** -0.5)
    dev = [t.cuda() for t in (q, k, v, dout, qo, ko)]
    out = ba.gdpa_cross_fwd(*dev[:3], dev[4], dev[5], act)
    dq, dk, dv = ba.gdpa_cross_bwd(*dev[:4], dev[4], dev[5], act)
    torch.cuda.synchronize()
    args = (qo.numpy(), ko.numpy(), f64(q), f64(k), f64(v))
    ref_out = G.cross_fwd(*args, act)
    ref_dq, ref_dk, ref_dv = G.cross_bwd(*args, f64(dout), act)
    for name, got, ref in (("out", out, ref_out), ("dq", dq, ref_dq), ("dk", dk, ref_dk), ("dv", dv, ref_dv)):
        check_bf16(f"cross {act} {name}", got.cpu(), ref, peaked=peaked)
    # empty sets: no keys -> out = dq = 0; no queries -> dk = dv = 0
    for e in range(len(lq)):
        qs, ks = slice(int(qo[e]), int(qo[e + 1])), slice(int(ko[e]), int(ko[e + 1]))
        if lk[e] == 0:
            assert not out[qs].any() and not dq[qs].any()
        if lq[e] == 0:
            assert not dk[ks].any() and not dv[ks].any()


def test_gdpa_cross_examples_are_isolated_from_non_finite_neighbours():
    """Cross-attention: Inf / NaN in one example's queries, keys, values and
    dout leave the other examples' results bit-equal to a clean run (each side's
    partial tiles end inside a neighbour's rows)."""
    lq, lk = [300, 100, 1000, 129], [64, 200, 17, 130]
    q, k, v, dout, qo, ko = _cross_inputs(128, lq, lk, 91, 128 ** -0.5)

    def run(q_, k_, v_, do_):
        dev = [t.cuda() for t in (q_, k_, v_, do_, qo, ko)]
        out = ba.gdpa_cross_fwd(*dev[:3], dev[4], dev[5], "silu")
        dq, dk, dv = ba.gdpa_cross_bwd(*dev[:4], dev[4], dev[5], "silu")
        torch.cuda.synchronize()
        return out.cpu(), dq.cpu(), dk.cpu(), dv.cpu()

    clean = run(q, k, v, dout)
    d = [t.clone() for t in (q, k, v, dout)]
    _poison(d[0], int(qo[1]), lq[1])
    _poison(d[3], int(qo[1]), lq[1])
    _poison(d[1], int(ko[1]), lk[1])
    _poison(d[2], int(ko[1]), lk[1])
    got = run(*d)
    for e in (0, 2, 3):
        qs, ks = slice(int(qo[e]), int(qo[e + 1])), slice(int(ko[e]), int(ko[e + 1]))
        for name, a, b, sl in (("out", got[0], clean[0], qs), ("dq", got[1], clean[1], qs),
                               ("dk", got[2], clean[2], ks), ("dv", got[3], clean[3], ks)):
            assert torch.equal(a[sl], b[sl]), f"example {e} {name} changed by a neighbour"
