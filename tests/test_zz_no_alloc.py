"""ss2d_forward_core_static: the projection form of the core for callers that cannot
allocate device memory at call time (it takes no workspace and uses the library's
static scratch).  Checked through the C ABI against ss2d_forward_core, which takes a
caller-provided workspace, on two calls in a row (the static scratch keeps the previous
call's contents, so the second call shows nothing stale leaks into the result).

This file is collected last so that, if it fails, a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import selective_scan_02_b200 as ss
from selective_scan_02_b200.inputs import Workload, bf16_bits, make_inputs

pytestmark = pytest.mark.gpu

TOL = 5e-3  # the bf16-input tolerance the parity tests use


def _dev(a, bf16=False):
    if bf16:
        return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _rel_err(got, ref):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms)))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# (B, D, H, W, N, R, channels_last): a small case; one whose batch does not fit the
# 16 MiB scratch at once (1.9 MiB per image), so the entry point runs several slices;
# one whose slices are scanned in segments (few images, long sequences), so each slice
# also holds segment states, which grow with the slice's image count; and the last
# two in channels-last layout.
CASES = [(2, 32, 9, 16, 16, 6, False), (11, 64, 56, 56, 16, 6, False), (9, 208, 60, 64, 16, 6, False),
         (11, 64, 56, 56, 16, 6, True), (9, 208, 60, 64, 16, 6, True)]


def _inputs(B, D, H, W, N, R, channels_last):
    inp = make_inputs(Workload("noalloc", B, D, H, W, N, R, "bf16", "bf16", 900 + B + D))
    x = _dev(inp["x"], True)
    if channels_last:
        x = x.permute(0, 2, 3, 1).contiguous()
    t = dict(x=x, A_logs=_dev(inp["A_logs"]), Ds=_dev(inp["Ds"]), dt_bias=_dev(inp["dt_bias"]),
             x_proj_weight=_dev(inp["x_proj_weight"], True), dt_projs_weight=_dev(inp["dt_projs_weight"]))
    return inp, t


@pytest.mark.parametrize("case", CASES)
def test_static_scratch_matches_workspace_entry(case):
    B, D, H, W, N, R, cl = case
    _, t = _inputs(B, D, H, W, N, R, cl)
    ref = ss.forward_core(**t, channels_last=cl)
    for _ in range(2):
        y = ss.forward_core_static(**t, channels_last=cl)
        torch.cuda.synchronize()
        assert torch.isfinite(y).all().item()
        assert _rel_err(y, ref) <= TOL


def test_static_scratch_segmented_slices_match_the_oracle():
    # The oracle computes the first and the last image; the slice plan puts them in
    # different slices, each scanned in segments.
    from oracle import oracle as orc

    B, D, H, W, N, R, _ = CASES[2]
    inp, t = _inputs(B, D, H, W, N, R, False)
    y = ss.forward_core_static(**t).cpu().numpy()
    for b in (0, B - 1):
        ref = orc.forward_core(inp["x"][b:b + 1], inp["A_logs"], inp["Ds"], inp["dt_bias"],
                               x_proj_weight=inp["x_proj_weight"], dt_projs_weight=inp["dt_projs_weight"])
        assert _rel_err(torch.from_numpy(y[b:b + 1]), torch.from_numpy(ref)) <= TOL


def test_static_scratch_rejects_images_larger_than_the_scratch():
    # One 192x192 image needs 4*(R+2N)*H*W*4 = 22.4 MB of scratch, more than the 16 MiB array.
    B, D, H, W, N, R = 1, 16, 192, 192, 16, 6
    x = torch.zeros((B, D, H, W), dtype=torch.bfloat16, device="cuda")
    args = dict(x=x, A_logs=torch.zeros((4 * D, N), device="cuda"), Ds=torch.zeros(4 * D, device="cuda"),
                dt_bias=torch.zeros(4 * D, device="cuda"),
                x_proj_weight=torch.zeros((4, R + 2 * N, D), dtype=torch.bfloat16, device="cuda"),
                dt_projs_weight=torch.zeros((4, D, R), device="cuda"))
    with pytest.raises(ss.Ss2dError) as ei:
        ss.forward_core_static(**args)
    assert ei.value.name == "SS2D_ERR_UNSUPPORTED"
    assert "static" in str(ei.value)
