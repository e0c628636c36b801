"""The bounded waits' error path on the GPU, run on purpose.

ss2d_diag_bounded_wait runs the tensor-core kernels' wait on an mbarrier that nothing arrives
at, with a short poll limit: the kernel records the timeout in a projection-form workspace's
error word, frees its tensor memory and returns.  ss2d_device_status must then report
SS2D_ERR_DEVICE, and the context must stay usable: the next projection-form call clears the
word, runs, and matches the oracle.  No fault, trap or hang is involved: every wait ends."""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from oracle import oracle as orc
from selective_scan_02_b200.inputs import Workload, bf16_bits, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _dev(a, dtype="f32"):
    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def test_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    wl = Workload("diag", 1, 32, 8, 16, 16, 4, "bf16", "bf16", 950)
    inp = make_inputs(wl)
    t = dict(x=_dev(inp["x"], "bf16"), A_logs=_dev(inp["A_logs"]), Ds=_dev(inp["Ds"]), dt_bias=_dev(inp["dt_bias"]),
             x_proj_weight=_dev(inp["x_proj_weight"], "bf16"), dt_projs_weight=_dev(inp["dt_projs_weight"]))
    ws = torch.zeros(ss.forward_core_workspace_size(**t), dtype=torch.uint8, device="cuda")
    ss.check_device_status(**t, workspace=ws)  # a clear word passes
    word = ws[:4].view(torch.int32)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ss.diag_bounded_wait(word, 4096)
    e1.record()
    torch.cuda.synchronize()
    assert int(word.item()) == 1
    print(f"4096 polls of an mbarrier that never completes: {e0.elapsed_time(e1):.3f} ms")
    with pytest.raises(ss.Ss2dError) as e:
        ss.check_device_status(**t, workspace=ws)
    assert e.value.name == "SS2D_ERR_DEVICE"
    # the context still works: the next call clears the word, runs and is right
    y = ss.forward_core(**t, workspace=ws)
    torch.cuda.synchronize()
    ss.check_device_status(**t, workspace=ws)
    ref = orc.forward_core(inp["x"], inp["A_logs"], inp["Ds"], inp["dt_bias"], x_proj_weight=inp["x_proj_weight"],
                           dt_projs_weight=inp["dt_projs_weight"])
    got = y.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref * ref)))
    assert float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms))) <= 5e-3


def test_diag_rejects_bad_arguments():
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ss.Ss2dError):
        ss.diag_bounded_wait(word, 0)
    with pytest.raises(ss.Ss2dError):
        ss.diag_bounded_wait(word, (1 << 20) + 1)
    torch.cuda.synchronize()
    assert int(word.item()) == 0
