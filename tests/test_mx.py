"""GPU parity of the MXFP8 path against oracle/mx.py: the quantisation pass
(ba_mx_quantize) byte for byte, block attention with MXFP8 Q and K in the
score product (ba_mx_fwd, the block-scaled tensor-core MMA) and its
straight-through backward (ba_mx_bwd) at the bf16 tolerances.

MX quantisation is integer/byte work (an exponent per block and a rounded
code per element), so its codes must match the oracle's exactly. The
attention's result is block attention of the dequantised Q and K (the oracle
dequantises and runs its fp64 attention); the MMA takes the E4M3 codes and
E8M0 scales themselves, so the comparison is at the project's bf16
tolerances (parity_util)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs
from oracle import mx as MX
import oracle
from parity_util import check_abs, check_bf16, f64

pytestmark = pytest.mark.gpu


def _codes_to_values(codes):
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_mx_quantize_matches_the_oracle_byte_for_byte():
    g = torch.Generator().manual_seed(5)
    rows, heads, D = 1000, 3, 128
    x = torch.randn(rows, heads, D, generator=g) * torch.exp2(torch.randint(-20, 20, (rows, heads, 1), generator=g))
    x[5] = 0.0                                # all-zero blocks
    x[7, 0, :32] = 1e-30                      # tiny values
    x[9, 1, 3] = 3.0e38                       # near the top of the bf16 range
    x[11, 2, :] = torch.tensor([448.0, 464.0, 480.0, -500.0] * 32)  # the block maximum itself clamps
    x = x.to(torch.bfloat16)
    el, sc = ba.mx_quantize(x.cuda())
    torch.cuda.synchronize()
    ref_el, ref_sc = MX.quantize(f64(x), "e4m3")         # [rows, heads, D/32, 32], [rows, heads, D/32, 1]
    got_el = _codes_to_values(el.cpu()).reshape(ref_el.shape)
    assert np.array_equal(got_el, ref_el)
    got_e = sc.cpu().numpy()[:, :heads].astype(np.int64) - 127
    assert np.array_equal(got_e, np.log2(ref_sc[..., 0]).astype(np.int64))


MX_CASES = [
    # (block, window, lengths)
    (256, 2, [64, 4096, 1000, 257, 129]),     # the jagged long-history shapes, reduced batch
    (64, 1, [0, 1, 127, 128, 129, 383]),      # independent 64-token blocks
    (512, 4, [2048]),
]


@pytest.mark.parametrize("block,window,lengths", MX_CASES)
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_mx_forward_matches_oracle(block, window, lengths, peaked):
    w = CONFIGS[3].replace(block=block, window=window, heads=2, batch=len(lengths))
    q_gain = 1.0
    if peaked:
        w = w.replace(qkv_scale=1.0)
        q_gain = 3.0
    inp = make_inputs(w, q_gain=q_gain, lengths=lengths, seed=640 + block)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs = inp["seq_offsets"].cuda()
    out, lse = ba.mx_block_attention_fwd(q, k, v, offs, block, window)
    torch.cuda.synchronize()
    ref_out, ref_lse = MX.fwd(inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), block,
                              window)
    check_bf16("mx out", out.cpu(), ref_out, peaked=peaked)
    check_abs("mx lse", lse.cpu(), ref_lse, 2e-3)
    # the quantisation is visible: plain attention on the unquantised q, k differs somewhat
    plain_out, _ = oracle.fwd(inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), block, window)
    assert np.abs(ref_out - plain_out).max() > 0


def test_mx_forward_with_skip_and_isolation():
    """Skipped examples pass v through; Inf/NaN in a neighbour's rows leave the
    other examples' outputs bit-equal to a clean run."""
    w = CONFIGS[5].replace(heads=2, batch=5)
    lengths = [300, 200, 1000, 129, 777]
    inp = make_inputs(w, lengths=lengths, seed=9)
    skip = torch.tensor([0, 1, 0, 0, 0], dtype=torch.uint8)
    offs_np = inp["seq_offsets"].numpy()
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs, sk = inp["seq_offsets"].cuda(), skip.cuda()
    out, lse = ba.mx_block_attention_fwd(q, k, v, offs, w.block, w.window, skip=sk)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    s3 = int(offs_np[3])
    for t in (q2, k2, v2):
        t[s3:s3 + 40] = float("nan")
    out2, lse2 = ba.mx_block_attention_fwd(q2, k2, v2, offs, w.block, w.window, skip=sk)
    torch.cuda.synchronize()
    ref_out, ref_lse = MX.fwd(offs_np, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), w.block, w.window,
                              skip=skip.numpy())
    for e in range(5):
        sl = slice(int(offs_np[e]), int(offs_np[e + 1]))
        if e == 1:
            assert torch.equal(out[sl].cpu(), inp["v"][sl])
            continue
        check_bf16(f"mx e{e} out", out[sl].cpu(), ref_out[sl])
        if e != 3:
            assert torch.equal(out[sl], out2[sl]) and torch.equal(lse[:, sl], lse2[:, sl]), e


@pytest.mark.parametrize("block,window,lengths", MX_CASES)
@pytest.mark.parametrize("peaked", [False, True], ids=["config", "peaked"])
def test_mx_backward_matches_oracle(block, window, lengths, peaked):
    """ba_mx_bwd (after ba_mx_fwd) against the oracle's straight-through
    gradients of block attention on the dequantised Q and K."""
    w = CONFIGS[3].replace(block=block, window=window, heads=2, batch=len(lengths))
    q_gain = 1.0
    if peaked:
        w = w.replace(qkv_scale=1.0)
        q_gain = 3.0
    inp = make_inputs(w, q_gain=q_gain, lengths=lengths, seed=660 + block)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].cuda()
    out, lse = ba.mx_block_attention_fwd(q, k, v, offs, block, window)
    dq, dk, dv = ba.mx_block_attention_bwd(q, k, v, out, lse, do, offs, block, window)
    torch.cuda.synchronize()
    ref = MX.bwd(inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["dout"]),
                 block, window)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        check_bf16(f"mx {name}", got.cpu(), r, peaked=peaked)
    # the quantisation is visible in the gradients too
    plain = oracle.bwd(inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["dout"]),
                       block, window)
    assert np.abs(ref[0] - plain[0]).max() > 0


def test_mx_backward_with_skip_and_isolation():
    """Skipped examples get dq = dk = 0 and dv = dout; Inf/NaN in a neighbour's
    rows of q, k, v and dout leave the other examples' gradients bit-equal."""
    w = CONFIGS[5].replace(heads=2, batch=5)
    lengths = [300, 200, 1000, 129, 777]
    inp = make_inputs(w, lengths=lengths, seed=19)
    skip = torch.tensor([0, 1, 0, 0, 0], dtype=torch.uint8)
    offs_np = inp["seq_offsets"].numpy()
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    offs, sk = inp["seq_offsets"].cuda(), skip.cuda()
    out, lse = ba.mx_block_attention_fwd(q, k, v, offs, w.block, w.window, skip=sk)
    g = ba.mx_block_attention_bwd(q, k, v, out, lse, do, offs, w.block, w.window, skip=sk)
    q2, k2, v2, do2 = q.clone(), k.clone(), v.clone(), do.clone()
    s3 = int(offs_np[3])
    for t in (q2, k2, v2, do2):
        t[s3:s3 + 40] = float("nan")
    out2, lse2 = ba.mx_block_attention_fwd(q2, k2, v2, offs, w.block, w.window, skip=sk)
    g2 = ba.mx_block_attention_bwd(q2, k2, v2, out2, lse2, do2, offs, w.block, w.window, skip=sk)
    torch.cuda.synchronize()
    ref = MX.bwd(offs_np, f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["dout"]), w.block, w.window,
                 skip=skip.numpy())
    for e in range(5):
        sl = slice(int(offs_np[e]), int(offs_np[e + 1]))
        if e == 1:
            assert not g[0][sl].any() and not g[1][sl].any() and torch.equal(g[2][sl].cpu(), inp["dout"][sl])
            continue
        for name, got, r in zip(("dq", "dk", "dv"), g, ref):
            check_bf16(f"mx e{e} {name}", got[sl].cpu(), r[sl])
        if e != 3:
            for a, b2 in zip(g, g2):
                assert torch.equal(a[sl], b2[sl]), e


def test_mx_backward_direct_call_and_status_word():
    """ba_mx_bwd through the C entry point with a caller-sized workspace; the
    status word ba_device_status reads sits at the workspace's start."""
    w = CONFIGS[3].replace(heads=2, batch=3)
    inp = make_inputs(w, lengths=[300, 129, 64], seed=21)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    offs = inp["seq_offsets"].cuda()
    out, lse = ba.mx_block_attention_fwd(q, k, v, offs, w.block, w.window)
    prob = ba.make_problem(q, offs)
    ws = ba.workspace_for(ba.ba_mx_bwd_workspace_size(prob, w.block, w.window), q.device)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    assert ba.ba_mx_bwd(prob, q, k, v, out, lse, do, offs, w.block, w.window, None, dq, dk, dv, ws) == ba.BA_OK
    assert ba.ba_device_status(ws) == ba.BA_OK
    ref = ba.mx_block_attention_bwd(q, k, v, out, lse, do, offs, w.block, w.window)
    torch.cuda.synchronize()
    for a, b in zip((dq, dk, dv), ref):
        assert torch.equal(a, b)


def test_mx_backward_rejects_head_dim_64_and_small_workspace():
    q = torch.zeros((128, 2, 64), dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor([0, 128], dtype=torch.int32, device="cuda")
    prob = ba.make_problem(q, offs)
    lse = torch.zeros((2, 128), device="cuda")
    ws = ba.workspace_for(ba.ba_mx_bwd_workspace_size(prob, 64, 1), q.device)
    assert ba.ba_mx_bwd(prob, q, q, q, q, lse, q, offs, 64, 1, None, q.clone(), q.clone(), q.clone(),
                        ws) == ba.BA_ERR_UNSUPPORTED
    q = torch.zeros((128, 2, 128), dtype=torch.bfloat16, device="cuda")
    prob = ba.make_problem(q, offs)
    need = ba.ba_mx_bwd_workspace_size(prob, 64, 1)
    assert need > ba.ba_bwd_workspace_size(prob, 64, 1)
    ws = ba.workspace_for(need, q.device)
    assert ba.ba_mx_bwd(prob, q, q, q, q, lse, q, offs, 64, 1, None, q.clone(), q.clone(), q.clone(), ws,
                        workspace_bytes=need - 256) == ba.BA_ERR_INVALID_ARG


def test_mx_forward_rejects_head_dim_64():
    q = torch.zeros((128, 2, 64), dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor([0, 128], dtype=torch.int32, device="cuda")
    prob = ba.make_problem(q, offs)
    ws = ba.workspace_for(ba.ba_mx_fwd_workspace_size(prob, 64, 1), q.device)
    lse = torch.empty((2, 128), device="cuda")
    assert ba.ba_mx_fwd(prob, q, q, q, offs, 64, 1, None, q.clone(), lse, ws) == ba.BA_ERR_UNSUPPORTED
