"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Inputs come from the seeded generator (block_sparse_attention_kunlun_b200/
workloads.py); the oracle receives exactly the values the GPU sees (bf16
inputs upcast without rounding). Tolerances: see parity_util.py.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
import oracle
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, draw_lengths, make_inputs
from parity_util import check_abs, check_bf16, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_gpu(inp, block, window, bwd=True):
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    offs = inp["seq_offsets"].to(DEV)
    skip = inp["skip"].to(DEV) if inp["skip"] is not None else None
    out, lse = ba.block_attention_fwd(q, k, v, offs, block, window, skip=skip)
    res = dict(out=out, lse=lse)
    if bwd:
        dout = inp["dout"].to(DEV)
        dq, dk, dv = ba.block_attention_bwd(q, k, v, out, lse, dout, offs, block, window, skip=skip)
        res.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    return {n: t.cpu() for n, t in res.items()}


def run_oracle(inp, block, window, bwd=True):
    args = (inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    skip = inp["skip"].numpy() if inp["skip"] is not None else None
    out, lse = oracle.fwd(*args, block, window, skip=skip)
    res = dict(out=out, lse=lse)
    if bwd:
        dq, dk, dv = oracle.bwd(*args, f64(inp["dout"]), block, window, skip=skip)
        res.update(dq=dq, dk=dk, dv=dv)
    return res


def compare(got, ref, fp32=False, peaked=False, skip=None, offs=None):
    lse_ref, lse_got = f64(ref["lse"]).copy(), f64(got["lse"]).copy()
    if fp32:
        check_abs("out", got["out"], ref["out"], 1e-5)
        check_abs("lse", lse_got, lse_ref, 1e-5)
    else:
        for name in ("out", "dq", "dk", "dv"):
            if name in got:
                check_bf16(name, got[name], ref[name], peaked=peaked)
        check_abs("lse", lse_got, lse_ref, 2e-3)
    if fp32:
        for name in ("dq", "dk", "dv"):
            if name in got:
                check_abs(name, got[name], ref[name], 1e-5)


# ------------------------------------------------------- reduced configs ---

REDUCED = {
    "cfg2": (2, dict(lengths=[1024] * 3)),
    "cfg3": (3, dict(lengths=[64, 4096, 1000, 257, 129])),
    "cfg4": (4, dict(lengths=[4096])),
    "cfg5": (5, dict(lengths=[300, 2000, 64, 1500, 777, 90])),
}


@pytest.mark.parametrize("name", list(REDUCED))
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_reduced_configs(name, peaked):
    cfg, kw = REDUCED[name]
    w = CONFIGS[cfg]
    q_gain = 1.0
    if peaked:  # unscaled N(0,1) q/k, q x3: sharply peaked rows expose masking/max bugs
        w = w.replace(qkv_scale=1.0)
        q_gain = 3.0
    inp = make_inputs(w, q_gain=q_gain, **kw)
    got = run_gpu(inp, w.block, w.window)
    ref = run_oracle(inp, w.block, w.window)
    compare(got, ref, peaked=peaked)


def test_config1_fp32_forward_full():
    w = CONFIGS[1]
    inp = make_inputs(w)
    got = run_gpu(inp, w.block, w.window, bwd=False)
    ref = run_oracle(inp, w.block, w.window, bwd=False)
    compare(got, ref, fp32=True)


@pytest.mark.parametrize("head_dim", [32, 64])
def test_fp32_backward(head_dim):
    w = CONFIGS[1].replace(head_dim=head_dim, window=2, block=48, fwd_only=False)
    inp = make_inputs(w, lengths=[256, 77, 0, 130])
    got = run_gpu(inp, w.block, w.window)
    ref = run_oracle(inp, w.block, w.window)
    compare(got, ref, fp32=True)


# ------------------------------------------------- ragged and edge cases ---

EDGE = [
    # (head_dim, block, window, lengths)
    (128, 64, 1, [0, 1, 127, 128, 129, 0, 383, 2 * 64 + 17]),
    (64, 100, 3, [1, 99, 100, 101, 250, 640]),
    (128, 128, 5, [129, 1000, 33, 777]),
    (64, 512, 2, [1500, 512, 511, 513]),
    (128, 256, 2, [2 * 256 + 17, 5, 1200]),
    (128, 7, 9, [300, 61]),
    (64, 1000000, 1, [700, 300]),        # one block: full causal attention
    (128, 64, 1000000, [600, 190]),      # window covers everything: full causal
    (64, 128, 2, [0, 0, 0, 200]),        # leading empty examples
    # window 1 with blocks dividing 128: every query tile sees only its own key
    # tile, and the backward runs as one fused pass
    (64, 64, 1, [1, 127, 129, 640, 65, 300]),
    (128, 32, 1, [1000, 33, 128, 257]),
    (128, 128, 1, [129, 1, 500, 384]),
    (64, 16, 1, [77, 256, 3]),
]


@pytest.mark.parametrize("head_dim,block,window,lengths", EDGE)
def test_edge_shapes(head_dim, block, window, lengths):
    w = CONFIGS[3].replace(head_dim=head_dim, block=block, window=window, heads=2,
                           qkv_scale=1.0, batch=len(lengths))
    inp = make_inputs(w, q_gain=1.0, lengths=lengths, seed=77 + head_dim + block % 97)
    got = run_gpu(inp, block, window)
    ref = run_oracle(inp, block, window)
    compare(got, ref, peaked=True)


@pytest.mark.parametrize("head_dim", [64, 128])
def test_single_key_rows_pass_values_through(head_dim):
    """block = 1, window = 1: every query sees only itself, so out = v exactly."""
    w = CONFIGS[3].replace(head_dim=head_dim, block=1, window=1, heads=3, batch=3)
    inp = make_inputs(w, lengths=[130, 1, 257])
    got = run_gpu(inp, 1, 1)
    assert torch.equal(got["out"], inp["v"])
    ref = run_oracle(inp, 1, 1)
    compare(got, ref)


def test_all_examples_skipped_and_empty_batch():
    w = CONFIGS[5].replace(skip_p=1.0, batch=3)
    inp = make_inputs(w, lengths=[200, 0, 129])
    got = run_gpu(inp, w.block, w.window)
    assert torch.equal(got["out"], inp["v"])
    assert torch.equal(got["dv"], inp["dout"])
    assert not got["dq"].any() and not got["dk"].any() and not got["lse"].any()
    # empty batch: nothing to do, but every call still succeeds
    e = make_inputs(CONFIGS[3].replace(batch=2), lengths=[0, 0])
    got = run_gpu(e, 256, 2)
    assert got["out"].numel() == 0 and got["dq"].numel() == 0


def test_forward_is_deterministic_and_status_ok():
    w = CONFIGS[3]
    inp = make_inputs(w, lengths=[1000, 3000, 70])
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs = inp["seq_offsets"].cuda()
    prob = ba.make_problem(q, offs)
    ws = ba.workspace_for(ba.ba_fwd_workspace_size(prob, w.block, w.window), q.device)
    a = ba.block_attention_fwd(q, k, v, offs, w.block, w.window, workspace=ws)
    b = ba.block_attention_fwd(q, k, v, offs, w.block, w.window, workspace=ws)
    assert ba.ba_device_status(ws) == ba.BA_OK
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("block", [64, 128])
def test_repeated_steps_with_one_key_tile_per_item(block):
    """Items of one key tile (window 1) make the forward's softmax fast next to its
    epilogue, so a softmax group can finish its next item before the epilogue has
    taken this one. Thirty fwd + bwd steps on 32 jagged histories must all report
    a clean status and give bit-identical results (no item interferes with another)."""
    w = CONFIGS[3].replace(block=block, window=1, batch=32)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(CONFIGS[3].seed)
    lengths = draw_lengths(CONFIGS[3], gen)[:32].tolist()  # config 3's first 32 histories
    inp = make_inputs(w, lengths=lengths)
    q, k, v, dout = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].cuda()
    prob = ba.make_problem(q, offs)
    wf = ba.workspace_for(ba.ba_fwd_workspace_size(prob, block, 1), q.device)
    wb = ba.workspace_for(ba.ba_bwd_workspace_size(prob, block, 1), q.device)
    first = None
    for step in range(30):
        out, lse = ba.block_attention_fwd(q, k, v, offs, block, 1, workspace=wf)
        assert ba.ba_device_status(wf) == ba.BA_OK, f"forward, step {step}"
        dq, dk, dv = ba.block_attention_bwd(q, k, v, out, lse, dout, offs, block, 1, workspace=wb)
        assert ba.ba_device_status(wb) == ba.BA_OK, f"backward, step {step}"
        res = (out, lse, dq, dk, dv)
        if first is None:
            first = tuple(t.clone() for t in res)
        else:
            for name, a, b in zip(("out", "lse", "dq", "dk", "dv"), first, res):
                assert torch.equal(a, b), f"{name} differs at step {step}"


# ------------------------------------------------ full sizes, sampled rows ---

def sample_rows(L, block, rng, extra=6):
    cand = {0, 1, block - 1, block, block + 1, 127, 128, 129, L // 2, L - 2, L - 1}
    cand |= set(int(x) for x in rng.integers(0, L, size=extra))
    return sorted(r for r in cand if 0 <= r < L)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_sampled(cfg):
    w = CONFIGS[cfg]
    inp = make_inputs(w)
    got = run_gpu(inp, w.block, w.window)
    offs = inp["seq_offsets"].numpy()
    lens = np.diff(offs)
    skip = inp["skip"].numpy() if inp["skip"] is not None else np.zeros(w.batch, np.uint8)
    rng = np.random.default_rng(cfg)
    live = [e for e in range(w.batch) if not skip[e] and lens[e] > 0]
    picks = sorted({live[0], live[-1], *rng.choice(live, size=min(2, len(live)), replace=False)})
    if cfg == 4:
        picks = picks[:3]
    for e in picks:
        s0, L = int(offs[e]), int(lens[e])
        sl = slice(s0, s0 + L)
        qe, ke, ve, de = (f64(inp[n][sl]) for n in ("q", "k", "v", "dout"))
        heads = [0, w.heads - 1] if cfg != 4 else [0]
        for h in heads:
            rows = sample_rows(L, w.block, rng)
            ref = oracle.rows(qe, ke, ve, h, rows, w.block, w.window, dout_e=de,
                              want=("out", "lse", "dq", "dk", "dv"))
            g = {n: f64(got[n][sl][rows, h]) for n in ("out", "dq", "dk", "dv")}
            g["lse"] = f64(got["lse"][h, s0:s0 + L][rows])
            for n in ("out", "dq", "dk", "dv"):
                check_bf16(f"cfg{cfg} e{e} h{h} {n}", g[n], ref[n])
            check_abs(f"cfg{cfg} e{e} h{h} lse", g["lse"], ref["lse"], 2e-3)
    # skipped examples pass through exactly
    for e in [e for e in range(w.batch) if skip[e]][:4]:
        sl = slice(int(offs[e]), int(offs[e + 1]))
        assert torch.equal(got["out"][sl], inp["v"][sl])
        assert torch.equal(got["dv"][sl], inp["dout"][sl])
        assert not got["dq"][sl].any() and not got["dk"][sl].any()


# ------------------------------------------- sliding-window attention ---
# ba_swa_fwd / ba_swa_bwd (query i sees keys i - w < j <= i) against the
# oracle's block rule with block = 1 (pinned to the window rule on the CPU).

def run_gpu_swa(inp, wt):
    q, k, v, dout = (inp[n].to(DEV) for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].to(DEV)
    out, lse = ba.sliding_window_attention_fwd(q, k, v, offs, wt)
    dq, dk, dv = ba.sliding_window_attention_bwd(q, k, v, out, lse, dout, offs, wt)
    torch.cuda.synchronize()
    return {n: t.cpu() for n, t in dict(out=out, lse=lse, dq=dq, dk=dk, dv=dv).items()}


SWA_CASES = [
    # (head_dim, window in tokens, lengths)
    (128, 512, [1500, 513, 1, 128, 0, 900]),
    (64, 100, [250, 99, 101, 640]),
    (128, 64, [2000, 65, 63, 129]),
    (128, 1000000, [700, 300]),          # window covers everything: full causal
]


@pytest.mark.parametrize("head_dim,wt,lengths", SWA_CASES)
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_sliding_window(head_dim, wt, lengths, peaked):
    w = CONFIGS[3].replace(head_dim=head_dim, heads=2, batch=len(lengths))
    q_gain = 1.0
    if peaked:
        w = w.replace(qkv_scale=1.0)
        q_gain = 3.0
    inp = make_inputs(w, q_gain=q_gain, lengths=lengths, seed=500 + wt % 997 + head_dim)
    got = run_gpu_swa(inp, wt)
    ref = run_oracle(inp, 1, wt)
    compare(got, ref, peaked=peaked)


def test_sliding_window_full_size_sampled():
    """Config 3 shapes (256 jagged histories, H8 D128) with a 512-token window, sampled rows."""
    w = CONFIGS[3]
    wt = 512
    inp = make_inputs(w)
    got = run_gpu_swa(inp, wt)
    offs = inp["seq_offsets"].numpy()
    lens = np.diff(offs)
    rng = np.random.default_rng(512)
    picks = sorted({0, w.batch - 1, *rng.choice(w.batch, size=2, replace=False)})
    for e in picks:
        s0, L = int(offs[e]), int(lens[e])
        sl = slice(s0, s0 + L)
        qe, ke, ve, de = (f64(inp[n][sl]) for n in ("q", "k", "v", "dout"))
        for h in (0, w.heads - 1):
            rows = sample_rows(L, wt, rng)
            ref = oracle.rows(qe, ke, ve, h, rows, 1, wt, dout_e=de, want=("out", "lse", "dq", "dk", "dv"))
            for n in ("out", "dq", "dk", "dv"):
                check_bf16(f"swa e{e} h{h} {n}", f64(got[n][sl][rows, h]), ref[n])
            check_abs(f"swa e{e} h{h} lse", f64(got["lse"][h, s0:s0 + L][rows]), ref["lse"], 2e-3)


# ------------------------------------------------ isolation of examples ---
# The oracle's examples are independent (tests/test_oracle.py: a jagged batch
# equals separate runs). On the GPU a 128-row tile at an example's end also
# loads the next example's rows; these cases put Inf and NaN there (and in a
# skipped example) and require every other example's results to be bit-equal
# to a clean run and within tolerance of the oracle.

ISOLATION = [
    # (dtype, head_dim, block, window)
    (torch.bfloat16, 128, 256, 2),
    (torch.bfloat16, 64, 64, 1),
    (torch.bfloat16, 128, 100, 3),
    (torch.float32, 32, 48, 2),
]


def _poison(t, s0, n):
    pattern = torch.tensor([float("inf"), float("nan"), float("-inf")], dtype=t.dtype)
    rows = t[s0:s0 + n]
    rows.copy_(pattern.repeat(rows.numel() // 3 + 1)[: rows.numel()].view_as(rows))


@pytest.mark.parametrize("dtype,head_dim,block,window", ISOLATION)
def test_examples_are_isolated_from_non_finite_neighbours(dtype, head_dim, block, window):
    lengths = [300, 200, 1000, 129, 777, 90, 128, 5]
    skip = torch.tensor([0, 0, 0, 1, 0, 0, 0, 0], dtype=torch.uint8)
    base = CONFIGS[1] if dtype == torch.float32 else CONFIGS[3]
    w = base.replace(head_dim=head_dim, block=block, window=window, heads=2, batch=len(lengths),
                     fwd_only=False)
    inp = make_inputs(w, lengths=lengths, seed=4242 + head_dim)
    inp["skip"] = skip
    offs = inp["seq_offsets"].numpy()
    poisoned = {1: 40, 3: lengths[3], 5: lengths[5], 7: lengths[7]}  # example -> rows poisoned from its start
    dirty = dict(inp)
    for n in ("q", "k", "v", "dout"):
        dirty[n] = inp[n].clone()
        for e, rows in poisoned.items():
            _poison(dirty[n], int(offs[e]), rows)
    clean_got = run_gpu(inp, block, window)
    dirty_got = run_gpu(dirty, block, window)
    ref = run_oracle(inp, block, window)
    for e in range(len(lengths)):
        if e in poisoned or lengths[e] == 0:
            continue
        sl = slice(int(offs[e]), int(offs[e + 1]))
        for n in ("out", "dq", "dk", "dv"):
            assert torch.equal(dirty_got[n][sl], clean_got[n][sl]), f"example {e} {n} changed by a neighbour"
            if dtype == torch.float32:
                check_abs(f"e{e} {n}", dirty_got[n][sl], ref[n][sl], 1e-5)
            else:
                check_bf16(f"e{e} {n}", dirty_got[n][sl], ref[n][sl])
        assert torch.equal(dirty_got["lse"][:, sl], clean_got["lse"][:, sl]), f"example {e} lse changed"
        check_abs(f"e{e} lse", dirty_got["lse"][:, sl], ref["lse"][:, sl], 1e-5 if dtype == torch.float32 else 2e-3)


@pytest.mark.parametrize("head_dim", [128, 64])
def test_gradients_into_16_byte_aligned_outputs(head_dim):
    """dq, dk and dv at addresses that are 16-byte but not 32-byte aligned (the
    dQ epilogue then takes 16-byte stores instead of 32-byte ones) get the same
    bits as into freshly allocated (256-byte aligned) tensors."""
    w = CONFIGS[3].replace(head_dim=head_dim, heads=2, batch=3)
    inp = make_inputs(w, lengths=[300, 129, 64], seed=77 + head_dim)
    q, k, v, dout = (inp[n].to(DEV) for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].to(DEV)
    out, lse = ba.block_attention_fwd(q, k, v, offs, w.block, w.window)
    ref = ba.block_attention_bwd(q, k, v, out, lse, dout, offs, w.block, w.window)
    shifted = []
    for _ in range(3):
        buf = torch.empty(q.numel() + 8, dtype=q.dtype, device=DEV)
        t = buf[8:].view(q.shape)                  # 16 bytes past a 256-byte boundary
        assert t.data_ptr() % 32 == 16
        shifted.append(t)
    got = ba.block_attention_bwd(q, k, v, out, lse, dout, offs, w.block, w.window,
                                 dq=shifted[0], dk=shifted[1], dv=shifted[2])
    torch.cuda.synchronize()
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        assert torch.equal(a, b), name
