"""The failure path of the bounded waits, without a GPU fault: a wait on an mbarrier that nothing completes
gives up after its limit, records its code in the device status word and returns; the host reads and clears
the word, and the context keeps working."""
import time

import pytest
import torch

from mixture_experts_layer_aux_b200.synthetic import Workload, make_inputs

pytestmark = pytest.mark.gpu

SELFTEST_CODE = 0x1F0


def test_bounded_wait_gives_up_and_reports(moe):
    assert moe.moe_get_device_status() == 0                     # clean start (and cleared)
    torch.cuda.synchronize()
    t0 = time.monotonic()
    moe.moe_selftest_wait_timeout()
    word = moe.moe_get_device_status(clear=True)                # synchronises
    dt = time.monotonic() - t0
    assert word == SELFTEST_CODE
    assert 1.9 < dt < 60.0, dt                                  # the 2 s limit, not an early or endless wait
    assert moe.moe_get_device_status() == 0                     # cleared
    # the context is still usable: a small layer forward runs and reports no failure
    wl = Workload("after-timeout", T=128, H=256, E=8, k=2, F=256)
    d = make_inputs(wl, device="cuda", seed=1)
    cfg = moe.make_config(wl)
    y = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    aux = torch.empty(1, dtype=torch.float32, device="cuda") if cfg.compute_aux else None
    moe.moe_layer_fwd(cfg, d["x"], d["W_r"], None, d["W_g"], d["W_u"], d["W_d"], None, None, None, None, None, None,
                      None, None, None, y, aux, idx, None, None, None, None,
                      moe.workspace(moe.moe_layer_workspace_size(cfg)))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    assert bool(torch.isfinite(y.float()).all())
