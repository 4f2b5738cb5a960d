"""Failure detection: every wait in the attention kernels is bounded and a
timeout comes back as BA_ERR_TIMEOUT through ba_device_status, without
faulting the GPU. The self-test entry point makes one such wait run out (a
barrier nothing completes) and the device must stay usable afterwards."""
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba
import oracle
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs
from parity_util import check_bf16, f64


def test_selftest_rejects_bad_arguments_before_launching():
    assert ba.ba_selftest_wait_timeout(0, 1000, workspace_bytes=256, stream=0) == ba.BA_ERR_INVALID_ARG      # null
    assert ba.ba_selftest_wait_timeout(256, 0, workspace_bytes=256, stream=0) == ba.BA_ERR_INVALID_ARG       # limit
    assert ba.ba_selftest_wait_timeout(256, 2_000_000, workspace_bytes=256, stream=0) == ba.BA_ERR_INVALID_ARG
    assert ba.ba_selftest_wait_timeout(256, 1000, workspace_bytes=128, stream=0) == ba.BA_ERR_INVALID_ARG    # size
    assert ba.ba_selftest_wait_timeout(260, 1000, workspace_bytes=256, stream=0) == ba.BA_ERR_INVALID_ARG    # alignment


@pytest.mark.gpu
def test_wait_times_out_and_device_stays_usable():
    ws = ba.workspace_for(256, torch.device("cuda"))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    assert ba.ba_selftest_wait_timeout(ws, 3000) == ba.BA_OK
    t1.record()
    assert ba.ba_device_status(ws) == ba.BA_ERR_TIMEOUT
    assert 2.9 <= t0.elapsed_time(t1) < 1000  # it waited about its limit, then returned
    # the same context still runs the attention path correctly, with a clean status
    w = CONFIGS[3].replace(heads=2, batch=2)
    inp = make_inputs(w, lengths=[300, 129])
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs = inp["seq_offsets"].cuda()
    prob = ba.make_problem(q, offs)
    wsf = ba.workspace_for(ba.ba_fwd_workspace_size(prob, w.block, w.window), q.device)
    out, lse = ba.block_attention_fwd(q, k, v, offs, w.block, w.window, workspace=wsf)
    assert ba.ba_device_status(wsf) == ba.BA_OK
    ref_out, _ = oracle.fwd(inp["seq_offsets"].numpy(), f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                            w.block, w.window)
    check_bf16("out after timeout", out.cpu(), ref_out)
