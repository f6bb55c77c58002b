"""Failure detection on the GPU without a fault.

A bounded wait is made to run out by planting the failure on the host: the
workspace header's ticket counter is set so that the scan starts at its
second chunk, i.e. the first chunk of every chain is never scanned.  Tiles of
the second chunk then wait for a carry nothing will publish; the wait gives
up after its iteration cap, records a timeout in the workspace status and
raises the abort flag, every other waiter stops, and the kernel exits
normally.  ``esa_check`` must report ESA_ERR_TIMEOUT, and the context and the
same workspace must keep working for the next call (the kernel's last CTA
resets the ticket and abort words and advances the epoch).

Nothing here faults, traps or hangs: every wait involved is bounded.
"""
import time

import pytest
import torch

from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, compare, oracle_fwd_bwd

pytestmark = pytest.mark.gpu

B, T, H, D, MODE, DTYPE = 2, 1024, 4, 32, 1, "f16"   # 16-bit, 64-channel tiles: 128-row tiles, 8 per chain
NCHAINS = B * (H * D // 64)
TICKET_WORD = {"fwd": 4, "bwd": 5}   # int32 index of ticket[0] / ticket[1] in the workspace header


def _inputs(dev):
    x = inputs.make_scan_inputs(B, T, H, D, DTYPE, 2.0, 55)
    return {k: x[k].to(dev) for k in ("a", "v", "q", "dy")}


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_lookback_wait_times_out_and_the_context_survives(cuda_device, which):
    xd = _inputs(cuda_device)
    ws = esa.new_workspace(B, T, H, D, DT[DTYPE], cuda_device)
    if which == "bwd":   # a good forward first: the backward needs its chunk states
        esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=MODE, workspace=ws)
        esa.esa_check(ws)
    torch.cuda.synchronize()
    ws.view(torch.int32)[TICKET_WORD[which]] = NCHAINS   # skip the first chunk in processing order
    t0 = time.time()
    if which == "fwd":
        esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=MODE, workspace=ws)
    else:
        esa.esa_scan_bwd(xd["a"], xd["v"], xd["q"], xd["dy"], ws, mode=MODE)
    with pytest.raises(esa.EsaError) as err:
        esa.esa_check(ws)
    assert err.value.code == esa.ESA_ERR_TIMEOUT
    assert time.time() - t0 < 60
    assert int(ws.view(torch.int32)[TICKET_WORD[which]]) == 0      # the kernel reset its ticket counter

    # the same workspace, the next call: correct results, no stale status
    y, Ef, _ = esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=MODE, workspace=ws)
    da, dv, dq, dE0 = esa.esa_scan_bwd(xd["a"], xd["v"], xd["q"], xd["dy"], ws, mode=MODE)
    esa.esa_check(ws)
    gpu = {"y": y, "E_final": Ef, "da": da, "dv": dv, "dq": dq, "dE_init": dE0}
    compare(gpu, oracle_fwd_bwd(xd, MODE), TOL[DT[DTYPE]], tuple(gpu))


def test_uninitialised_workspace_is_reported(cuda_device):
    xd = _inputs(cuda_device)
    n = esa.esa_workspace_size(B, T, H, D, DT[DTYPE])
    ws = torch.zeros(n, dtype=torch.uint8, device=cuda_device)      # never passed to esa_workspace_init
    esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=MODE, workspace=ws)
    with pytest.raises(esa.EsaError) as err:
        esa.esa_check(ws)
    assert err.value.code == esa.ESA_ERR_WORKSPACE
    esa.esa_workspace_init(ws)
    y, Ef, _ = esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=MODE, workspace=ws)
    esa.esa_check(ws)
    ref = oracle_fwd_bwd(xd, MODE, with_bwd=False)
    compare({"y": y, "E_final": Ef}, ref, TOL[DT[DTYPE]], ("y", "E_final"))
