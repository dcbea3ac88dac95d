"""Failure detection on a B200 without a GPU fault.

Every pipelined kernel waits on mbarriers through one bounded wait: after its
budget it records MOE_ERR_TIMEOUT and the waiting site in the workspace status
word and returns, and any wait that finds a failure already recorded gives up
at once. Here a wait that nothing satisfies (an mbarrier no one arrives at)
is made to run out; the host reads the status, and the context stays usable
for a correct forward afterwards."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import BF16_TOL, check_close, dev, dev_bf16, host_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402

SITE_SELFTEST = 7


def _tiny_forward_ok():
    cfg = mi.CONFIGS["tiny"]
    L = mi.make_layer(cfg)
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = torch.zeros(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), dev_bf16(L["w13"]),
                    dev_bf16(L["w2"]), d, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k)
    check_close(mi.bf16_to_f32(host_bf16(out)), ref["out"], BF16_TOL)


def test_wait_runs_out_records_timeout_and_context_survives():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    moe.moe_check_wait_timeout(ws, 4_000_000)  # about 2 ms of SM clocks
    e1.record()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == (moe.MOE_ERR_TIMEOUT << 8) | SITE_SELFTEST
    assert e0.elapsed_time(e1) < 500.0
    moe.moe_clear_device_status(ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    _tiny_forward_ok()


def test_wait_gives_up_at_once_when_a_failure_is_recorded():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    earlier = (moe.MOE_ERR_TIMEOUT << 8) | 3
    ws[:4].view(torch.int32).fill_(earlier)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    moe.moe_check_wait_timeout(ws, 2_000_000_000)  # would be about a second
    e1.record()
    torch.cuda.synchronize()
    assert e0.elapsed_time(e1) < 100.0
    assert moe.moe_get_device_status(ws) == earlier  # the first failure is kept
    _tiny_forward_ok()


def test_wait_budget_is_validated():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for bad in (0, 999, 3_000_000_000):
        with pytest.raises(moe.MoeError):
            moe.moe_check_wait_timeout(ws, bad)
