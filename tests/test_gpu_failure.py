"""The failure path of the kernels' bounded waits, made to run out on purpose without a fault:
tt_probe_bounded_wait waits on a shared-memory barrier that nothing arrives on, gives up after
the given limit and records TT_ERR_DEVICE_TIMEOUT in the workspace; the context stays usable."""
import time

import pytest
import torch

from denoiser_attention_b200 import api
from denoiser_attention_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_us", [100, 2000])
def test_bounded_wait_gives_up_and_reports(cuda_lib, limit_us):
    ws = B.new_workspace(256)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.tt_probe_bounded_wait(ws, limit_us)
    st, detail = B.tt_get_device_error(ws)
    elapsed = time.perf_counter() - t0
    assert st == B.TT_ERR_DEVICE_TIMEOUT and detail == B.TT_DETAIL_WAIT_PROBE
    assert elapsed >= limit_us * 1e-6
    assert B.tt_get_device_error(ws) == (B.TT_OK, 0)   # the read cleared the word
    # the context is still usable: a library kernel runs and gives the right answer afterwards
    masked = torch.tensor([[1, 0, 1, 1], [0, 0, 0, 1]], dtype=torch.uint8, device="cuda")
    tau = api.block_tau(masked)
    torch.cuda.synchronize()
    assert tau.cpu().tolist() == [0.75, 0.25]


def test_step_check_errors_raises_on_a_recorded_error(cuda_lib):
    # a device error recorded in a cached workspace surfaces through check_device_errors()
    ws = api.workspace(256, torch.device("cuda"), "probe")
    B.tt_probe_bounded_wait(ws, 50)
    with pytest.raises(B.TTError) as e:
        api.check_device_errors("cuda")
    assert e.value.status == B.TT_ERR_DEVICE_TIMEOUT
    api.check_device_errors("cuda")    # cleared by the read
