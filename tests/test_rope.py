"""GPU parity of the rotary entry points (ba_rope_fwd / ba_rope_bwd, called
through the C ABI) against the oracle's rope_fwd / rope_bwd.

The rotary embedding is RoFormer's rotation of adjacent pairs of q and k at
each row's position within its example ("GEM (Meta)", section "Custom
kernels": the block-attention kernel fuses the rotary embedding's backward
pass). The library holds the rotated q and k in the input dtype, the type
its tensor-core products take, so for bf16 the oracle rotates exactly in
fp64 and rounds that exact value to the nearest bf16 (operand_dtype); for
fp32 it does not round. Tables come from the seeded input module (RoFormer's
frequencies, float32).

Tolerances: out, dq, dk, dv and the fp32 path as in parity_util. lse gets
parity_util's 2e-3 plus a bound derived from the kernel's arithmetic: the
kernel forms each rotated value in float32 (two products and a sum or
difference, each rounded once), which lies within
    eps = 2^-23 (1 + 2^-23) (|x0 c| + |x1 s|)
of the exact value (|fl(a op b) - (a op b)| <= 2^-24 |a op b| per
operation). The kernel's bf16 operand is then some bf16 value between
round(y - eps) and round(y + eps), and so is the oracle's round(y): the two
differ by at most the width of that interval (one bf16 step where a
rounding midpoint lies inside [y - eps, y + eps]; more only where the sum
cancels, |y| far below |x0 c| + |x1 s|; 0 almost everywhere). With dq, dk
those widths, every score of row i moves by at most
    B_i = (1/sqrt(D)) max_j sum_d (dq_id |k_jd| + |q_id| dk_jd + dq_id dk_jd),
and lse, a smooth maximum of the scores, moves by at most max_j of that
(its gradient with respect to the scores is a probability vector). B_i is
0 for every row without such an operand.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
import oracle
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs, rope_tables
from parity_util import check_abs, check_bf16, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_gpu_rope(inp, block, window, cos, sin, bwd=True):
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    offs = inp["seq_offsets"].to(DEV)
    skip = inp["skip"].to(DEV) if inp["skip"] is not None else None
    c, s = cos.to(DEV), sin.to(DEV)
    prob = ba.make_problem(q, offs)
    ws = ba.workspace_for(ba.ba_rope_bwd_workspace_size(prob, block, window), q.device)
    out, lse = ba.rope_block_attention_fwd(q, k, v, offs, block, window, c, s, skip=skip, workspace=ws)
    res = dict(out=out, lse=lse)
    status = [ba.ba_device_status(ws)]
    if bwd:
        dout = inp["dout"].to(DEV)
        dq, dk, dv = ba.rope_block_attention_bwd(q, k, v, out, lse, dout, offs, block, window, c, s, skip=skip,
                                                 workspace=ws)
        res.update(dq=dq, dk=dk, dv=dv)
        status.append(ba.ba_device_status(ws))
    torch.cuda.synchronize()
    # q and k are read, never rotated in place
    assert torch.equal(q.cpu(), inp["q"]) and torch.equal(k.cpu(), inp["k"])
    res = {n: t.cpu() for n, t in res.items()}
    res["status"] = status
    return res


def run_oracle_rope(inp, block, window, cos, sin, bwd=True):
    operand = torch.bfloat16 if inp["q"].dtype == torch.bfloat16 else None
    args = (inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]))
    c, s = f64(cos), f64(sin)
    skip = inp["skip"].numpy() if inp["skip"] is not None else None
    out, lse = oracle.rope_fwd(*args, c, s, block, window, skip=skip, operand_dtype=operand)
    res = dict(out=out, lse=lse)
    if bwd:
        dq, dk, dv = oracle.rope_bwd(*args, f64(inp["dout"]), c, s, block, window, skip=skip, operand_dtype=operand)
        res.update(dq=dq, dk=dk, dv=dv)
    return res


def flip_step(x, seq_offsets, cos, sin, rows_pos=None):
    """Per element of the rotated operand: how far the kernel's bf16 value may
    sit from the oracle's, the width round(y + eps) - round(y - eps) of the
    interval both lie in (0 where the float32 evaluation cannot change the
    rounding)."""
    x = f64(x)
    pos = oracle.positions(seq_offsets) if rows_pos is None else np.asarray(rows_pos)
    c = f64(cos)[pos][:, None, :]
    s = f64(sin)[pos][:, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    mag = np.empty_like(x)
    mag[..., 0::2] = np.abs(x0 * c) + np.abs(x1 * s)
    mag[..., 1::2] = np.abs(x0 * s) + np.abs(x1 * c)
    y = oracle._rotate_at(x, pos, cos, sin, False)
    eps = 2.0 ** -23 * (1 + 2.0 ** -23) * mag
    return np.abs(oracle.round_bf16(y + eps) - oracle.round_bf16(y - eps))


def _visible_range(i, L, block, window):
    """Keys [lo, i] that local query i sees (the block rule)."""
    b = i // block
    return (b - window + 1) * block if b >= window else 0


def lse_flip_bound(q_e, k_e, cos, sin, head, rows, block, window):
    """B_i (module docstring) for the given local rows of one example's head,
    the maximum taken over the keys each row sees: how far the kernel's lse
    may sit from the oracle's because of bf16 rounding decisions its float32
    evaluation may take the other way. Split as
    max_j (A_ij + C_ij) <= max_j A_ij + max_j C_ij with
    A_ij = sum_d dq_id (|k_jd| + dk_jd) (rows with a q change) and
    C_ij = sum_d |q_id| dk_jd (keys with a k change)."""
    L, _, D = q_e.shape
    offs = np.array([0, L], dtype=np.int32)
    qr = np.abs(oracle._rotated_operand(q_e, offs, f64(cos), f64(sin), torch.bfloat16)[:, head])
    kr = np.abs(oracle._rotated_operand(k_e, offs, f64(cos), f64(sin), torch.bfloat16)[:, head])
    dq = flip_step(q_e, offs, cos, sin)[:, head]
    dk = flip_step(k_e, offs, cos, sin)[:, head]
    rows = np.asarray(rows, dtype=np.int64)
    b = np.zeros(len(rows))
    kk = kr + dk
    for n, i in enumerate(rows):
        lo = _visible_range(int(i), L, block, window)
        if dq[i].any():
            b[n] += float(np.max(kk[lo:i + 1] @ dq[i]))
        js = lo + np.flatnonzero(dk[lo:i + 1].any(axis=1))
        if js.size:
            b[n] += float(np.max(dk[js] @ qr[i]))
    return b / np.sqrt(D)


def lse_bounds(inp, cos, sin, block, window):
    """B for every row of a batch, [heads, total_tokens]."""
    offs = inp["seq_offsets"].numpy()
    T, H, _ = inp["q"].shape
    out = np.zeros((H, T))
    for e in range(len(offs) - 1):
        s0, s1 = int(offs[e]), int(offs[e + 1])
        if s1 == s0:
            continue
        qe, ke = f64(inp["q"][s0:s1]), f64(inp["k"][s0:s1])
        for h in range(H):
            out[h, s0:s1] = lse_flip_bound(qe, ke, cos, sin, h, np.arange(s1 - s0), block, window)
    return out


def compare_rope(got, ref, fp32=False, peaked=False, lse_extra=None):
    assert all(st == ba.BA_OK for st in got["status"]), got["status"]
    for name in ("out", "dq", "dk", "dv"):
        if name in got:
            if fp32:
                check_abs(name, got[name], ref[name], 1e-5)
            else:
                check_bf16(name, got[name], ref[name], peaked=peaked)
    if fp32:
        check_abs("lse", got["lse"], ref["lse"], 1e-5)
        return
    diff = np.abs(f64(got["lse"]) - f64(ref["lse"]))
    tol = 2e-3 + (lse_extra if lse_extra is not None else 0.0)
    bad = diff > tol
    assert not bad.any(), (f"lse: {int(bad.sum())} rows beyond 2e-3 + flip bound; worst excess "
                           f"{float(np.max(diff - tol)):.3e}, max diff {float(diff.max()):.3e}")


BF16_CASES = [
    # (head_dim, block, window, lengths): several tiles, ragged tails, empty examples
    (128, 256, 2, [64, 4096, 1000, 257, 129]),      # config 3 shapes, reduced batch
    (64, 128, 2, [1024, 1024, 0, 300]),             # config 2 shapes
    (128, 64, 1, [0, 1, 127, 128, 129, 383]),       # the pages' independent 64-token blocks
    (64, 100, 3, [1, 99, 250, 640]),
]


@pytest.mark.parametrize("head_dim,block,window,lengths", BF16_CASES)
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_rope_bf16(head_dim, block, window, lengths, peaked):
    w = CONFIGS[3].replace(head_dim=head_dim, block=block, window=window, heads=2, batch=len(lengths))
    q_gain = 1.0
    if peaked:
        w = w.replace(qkv_scale=1.0)
        q_gain = 3.0
    inp = make_inputs(w, q_gain=q_gain, lengths=lengths, seed=900 + head_dim + block)
    cos, sin = rope_tables(max(lengths) + 5, head_dim)
    got = run_gpu_rope(inp, block, window, cos, sin)
    ref = run_oracle_rope(inp, block, window, cos, sin)
    compare_rope(got, ref, peaked=peaked, lse_extra=lse_bounds(inp, cos, sin, block, window))


@pytest.mark.parametrize("head_dim", [32, 64])
def test_rope_fp32(head_dim):
    w = CONFIGS[1].replace(head_dim=head_dim, window=2, block=48, fwd_only=False)
    lengths = [256, 77, 0, 130]
    inp = make_inputs(w, lengths=lengths)
    cos, sin = rope_tables(256, head_dim)
    got = run_gpu_rope(inp, w.block, w.window, cos, sin)
    ref = run_oracle_rope(inp, w.block, w.window, cos, sin)
    compare_rope(got, ref, fp32=True)


def test_rope_with_skipped_examples():
    w = CONFIGS[5]
    lengths = [300, 2000, 64, 1500, 777, 90]
    inp = make_inputs(w, lengths=lengths)
    assert inp["skip"].any() and not inp["skip"].all()
    cos, sin = rope_tables(2048, w.head_dim)
    got = run_gpu_rope(inp, w.block, w.window, cos, sin)
    ref = run_oracle_rope(inp, w.block, w.window, cos, sin)
    compare_rope(got, ref, lse_extra=lse_bounds(inp, cos, sin, w.block, w.window))
    offs = inp["seq_offsets"].numpy()
    for e in np.flatnonzero(inp["skip"].numpy()):
        sl = slice(int(offs[e]), int(offs[e + 1]))
        assert torch.equal(got["out"][sl], inp["v"][sl])
        assert not got["dq"][sl].any() and not got["dk"][sl].any()


@pytest.mark.parametrize("head_dim", [64, 128])
def test_identity_tables_match_plain_attention_bitwise(head_dim):
    """cos = 1, sin = 0: the rotation pass copies q and k exactly and the
    epilogues' transposed rotation is exact, so every output equals ba_fwd /
    ba_bwd bit for bit."""
    w = CONFIGS[3].replace(head_dim=head_dim, heads=2, batch=3)
    inp = make_inputs(w, lengths=[700, 129, 1000], seed=31)
    cos, sin = torch.ones(1000, head_dim // 2), torch.zeros(1000, head_dim // 2)
    got = run_gpu_rope(inp, w.block, w.window, cos, sin)
    q, k, v, dout = (inp[n].to(DEV) for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].to(DEV)
    out, lse = ba.block_attention_fwd(q, k, v, offs, w.block, w.window)
    dq, dk, dv = ba.block_attention_bwd(q, k, v, out, lse, dout, offs, w.block, w.window)
    for name, t in (("out", out), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.equal(got[name], t.cpu()), name


def test_tables_shorter_than_an_example_are_reported():
    """Rows past the tables are left unrotated (no read outside the tables)
    and the status word reports it; a call with long enough tables on the
    same workspace size is clean."""
    w = CONFIGS[3].replace(heads=2, batch=2)
    inp = make_inputs(w, lengths=[300, 129], seed=5)
    cos, sin = rope_tables(200, w.head_dim)
    got = run_gpu_rope(inp, w.block, w.window, cos, sin)
    assert got["status"] == [ba.BA_ERR_INVALID_ARG, ba.BA_ERR_INVALID_ARG]
    cos, sin = rope_tables(300, w.head_dim)
    got = run_gpu_rope(inp, w.block, w.window, cos, sin)
    assert got["status"] == [ba.BA_OK, ba.BA_OK]


def test_rope_full_size_sampled():
    """Config 3 (256 jagged histories of 64-4096 tokens, H8 D128, block 256,
    window 2) with rotary tables of 4096 rows; sampled rows of four examples."""
    w = CONFIGS[3]
    inp = make_inputs(w)
    cos, sin = rope_tables(4096, w.head_dim)
    got = run_gpu_rope(inp, w.block, w.window, cos, sin)
    assert got["status"] == [ba.BA_OK, ba.BA_OK]
    offs = inp["seq_offsets"].numpy()
    lens = np.diff(offs)
    rng = np.random.default_rng(4096)
    picks = sorted({0, w.batch - 1, *rng.choice(w.batch, size=2, replace=False)})
    c, s = f64(cos), f64(sin)
    for e in picks:
        s0, L = int(offs[e]), int(lens[e])
        sl = slice(s0, s0 + L)
        qe, ke, ve, de = (f64(inp[n][sl]) for n in ("q", "k", "v", "dout"))
        for h in (0, w.heads - 1):
            cand = {0, 1, 127, 128, 255, 256, 257, L // 2, L - 1} | set(int(x) for x in rng.integers(0, L, 6))
            rows = sorted(r for r in cand if r < L)
            ref = oracle.rope_rows(qe, ke, ve, c, s, h, rows, w.block, w.window, dout_e=de,
                                   want=("out", "lse", "dq", "dk", "dv"), operand_dtype=torch.bfloat16)
            for n in ("out", "dq", "dk", "dv"):
                check_bf16(f"rope e{e} h{h} {n}", f64(got[n][sl][rows, h]), ref[n])
            tol = 2e-3 + lse_flip_bound(qe, ke, cos, sin, h, rows, w.block, w.window)
            diff = np.abs(f64(got["lse"][h, s0:s0 + L][rows]) - ref["lse"])
            assert np.all(diff <= tol), f"rope e{e} h{h} lse: max excess {float(np.max(diff - tol)):.3e}"


def test_rotated_copies_round_within_their_float32_error_and_are_reused():
    """A property of the kernel, not an oracle comparison: the rotation pass's
    bf16 copies equal the exact rotation rounded to nearest even except where
    the float32 evaluation's error interval (module docstring) holds more than
    one rounding result, and there they stay inside that interval; a backward
    reading the forward's kept copies gives the same bits as one that
    recomputes them."""
    w = CONFIGS[3].replace(heads=2, batch=3, qkv_scale=1.0)
    inp = make_inputs(w, q_gain=3.0, lengths=[1000, 129, 700], seed=41)
    cos, sin = rope_tables(1000, w.head_dim)
    q, k, v, dout = (inp[n].to(DEV) for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].to(DEV)
    c, s = cos.to(DEV), sin.to(DEV)
    q_rot, k_rot = torch.empty_like(q), torch.empty_like(k)
    out, lse = ba.rope_block_attention_fwd(q, k, v, offs, w.block, w.window, c, s, q_rot=q_rot, k_rot=k_rot)
    saved = ba.rope_block_attention_bwd(q, k, v, out, lse, dout, offs, w.block, w.window, c, s,
                                        q_rot=q_rot, k_rot=k_rot)
    fresh = ba.rope_block_attention_bwd(q, k, v, out, lse, dout, offs, w.block, w.window, c, s)
    out2, lse2 = ba.rope_block_attention_fwd(q, k, v, offs, w.block, w.window, c, s)
    torch.cuda.synchronize()
    offs_np = inp["seq_offsets"].numpy()
    for name, got, x in (("q_rot", q_rot, inp["q"]), ("k_rot", k_rot, inp["k"])):
        ref = oracle._rotated_operand(f64(x), offs_np, f64(cos), f64(sin), torch.bfloat16)
        step = flip_step(x, offs_np, cos, sin)
        g = f64(got.cpu())
        same = g == ref
        assert np.all(np.abs(g - ref) <= step), name
        assert same.mean() > 0.999, name
    for a, b, name in zip(saved, fresh, ("dq", "dk", "dv")):
        assert torch.equal(a, b), name
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
