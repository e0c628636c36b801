"""CUDA-graph capture of the library's calls.

No entry point allocates, synchronises or reads back from the device inside a call (the
status readers excepted), so a call can be captured into a CUDA graph on a side stream and
replayed.  The first call on a device raises kernels' shared-memory limits
(cudaFuncSetAttribute), so each call runs once eagerly before the capture.  Each replay must
give the eager result: bit for bit where the result is deterministic (the page-order merge,
the backward's ddts), within the last bits of the four-way atomic merge elsewhere."""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from selective_scan_02_b200.inputs import BlockWorkload, Workload, bf16_bits, make_block_inputs, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _dev(a, dtype="f32"):
    if dtype == "bf16":
        return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn(s)
    torch.cuda.current_stream().wait_stream(s)
    return g


def _close(a, b, tol):
    a, b = a.double(), b.double()
    return float((a - b).abs().max()) <= tol * float(b.abs().max())


@pytest.mark.parametrize("page_order", [False, True])
def test_forward_core_replays_in_a_graph(page_order):
    wl = Workload("graph", 2, 64, 24, 32, 16, 0, "bf16", "bf16", 900)
    inp = make_inputs(wl)
    t = dict(x=_dev(inp["x"], "bf16"), dts=_dev(inp["dts"], "bf16"), Bs=_dev(inp["Bs"]), Cs=_dev(inp["Cs"]),
             A_logs=_dev(inp["A_logs"]), Ds=_dev(inp["Ds"]), dt_bias=_dev(inp["dt_bias"]))
    y = torch.empty((wl.B, wl.D, wl.H, wl.W), device="cuda")
    ws = torch.empty(max(ss.forward_core_workspace_size(**t, page_order=page_order), 1), dtype=torch.uint8,
                     device="cuda")
    eager = ss.forward_core(**t, page_order=page_order).clone()
    g = _capture(lambda s: ss.forward_core(**t, y=y, workspace=ws, stream=s, page_order=page_order))
    for _ in range(3):
        y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        if page_order:
            assert torch.equal(y.view(torch.int32), eager.view(torch.int32))
        else:
            assert _close(y, eager, 1e-6)


def test_projection_form_and_backward_replay_in_a_graph():
    wl = Workload("graph_p", 2, 32, 8, 16, 16, 4, "bf16", "bf16", 901)
    inp = make_inputs(wl)
    t = dict(x=_dev(inp["x"], "bf16"), A_logs=_dev(inp["A_logs"]), Ds=_dev(inp["Ds"]), dt_bias=_dev(inp["dt_bias"]),
             x_proj_weight=_dev(inp["x_proj_weight"], "bf16"), dt_projs_weight=_dev(inp["dt_projs_weight"]))
    dy = torch.from_numpy(np.random.default_rng(5).standard_normal((2, 32, 8, 16)).astype(np.float32)).cuda()
    y = torch.empty((2, 32, 8, 16), device="cuda")
    ws = torch.empty(ss.forward_core_workspace_size(**t), dtype=torch.uint8, device="cuda")
    y_eager = ss.forward_core(**t).clone()
    g_eager = {k: v.clone() for k, v in ss.forward_core_backward(**t, dy=dy).items()}
    grads = ss.forward_core_backward(**t, dy=dy)
    bws = torch.empty(ss.forward_core_backward_workspace_size(**t), dtype=torch.uint8, device="cuda")

    def step(s):
        ss.forward_core(**t, y=y, workspace=ws, stream=s)
        ss.forward_core_backward(**t, dy=dy, grads=grads, workspace=bws, stream=s)

    g = _capture(step)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert _close(y, y_eager, 1e-6)
        for k, v in g_eager.items():
            assert _close(grads[k], v, 1e-5), k


def test_block_replays_in_a_graph():
    wl = BlockWorkload("graph_b", 2, 12, 16, 32, 64, 16, 4, 3, 902)
    inp = make_block_inputs(wl)
    bf = ("x", "in_proj_weight", "x_proj_weight", "out_proj_weight")
    t = {k: _dev(v, "bf16" if k in bf else "f32") for k, v in inp.items()}
    keys = ("x", "in_proj_weight", "conv_weight", "conv_bias", "x_proj_weight", "dt_projs_weight", "dt_projs_bias",
            "A_logs", "Ds", "out_norm_weight", "out_norm_bias", "out_proj_weight")
    args = [t[k] for k in keys]
    out = torch.empty((2, 12, 16, 32), device="cuda")
    ws = torch.empty(ss.block_forward_workspace_size(*args), dtype=torch.uint8, device="cuda")
    eager = ss.block_forward(*args).clone()
    g = _capture(lambda s: ss.block_forward(*args, out=out, workspace=ws, stream=s))
    for _ in range(3):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert _close(out, eager, 1e-5)
