"""GPU parity: every kernel against the fp64 oracle through the C-ABI.

Small and medium cases are compared element by element over the whole
output (Y is poisoned with NaN first, so unwritten outputs fail); the five
workloads at full size are compared on sampled outputs the oracle computes
one by one, plus properties that hold at any size.
"""

import numpy as np
import pytest
import torch

from cases import random_case
from parity import (check_close, draw_case, full_parity, gpu_run, sampled_parity, to_oracle,
                    attrs_from)
from oracle import conv_transpose_ref
from transposed_convolution_02_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _wl_case(wl):
    return dict(x_shape=wl.x_shape, w_shape=wl.w_shape, strides=wl.strides,
                dilations=wl.dilations, pads=wl.pads, output_padding=wl.output_padding,
                auto_pad=wl.auto_pad, group=wl.group, bias=wl.bias)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    major, _ = torch.cuda.get_device_capability()
    assert major == 10, "these kernels are built for sm_100a"


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
@pytest.mark.parametrize("layout", ["nchw", "nhwc"])
def test_generic_random_sweep(dtype, layout):
    rng = np.random.default_rng(100 + (dtype == torch.float16) + 2 * (layout == "nhwc"))
    for i in range(60):
        case = random_case(rng, pads=(-1, 3))
        full_parity(case, dtype, 5000 + i, layout, algo="generic", expect_kernel="generic")


def test_generic_empty_and_degenerate():
    # C = 0 (no term reaches any output: Y = bias), a 1x1 kernel, N = 0.
    case = dict(x_shape=[2, 0, 5], w_shape=[0, 3, 2], strides=[2], bias=True)
    x = torch.zeros([2, 0, 5], dtype=torch.float32)
    w = torch.zeros([0, 3, 2], dtype=torch.float32)
    b = torch.tensor([1.0, -2.0, 0.5])
    op, y = gpu_run(case, x, w, b, "nchw", "generic")
    assert torch.all(y.cpu() == b.view(1, 3, 1))
    full_parity(dict(x_shape=[2, 6, 9, 7], w_shape=[6, 5, 1, 1], strides=[1, 1], bias=True),
                torch.float16, 77, "nchw", algo="generic")
    op, y = gpu_run(dict(x_shape=[0, 4, 5], w_shape=[4, 2, 3], strides=[2]),
                    torch.zeros([0, 4, 5]), torch.zeros([4, 2, 3]), None, "nchw", "generic",
                    poison=False)
    assert y.shape == (0, 2, 11)


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_workload_reduced(wid):
    """Each workload's attributes on reduced sizes, whole output compared."""
    wl = WORKLOADS[wid]
    case = _wl_case(wl)
    x_shape = list(wl.x_shape)
    w_shape = list(wl.w_shape)
    if wid == 2:
        x_shape, w_shape = [2, 96, 13, 21], [96, 40, 4, 4]
    elif wid == 3:
        x_shape, w_shape = [1, 24, 5, 6, 7], [24, 20, 3, 3, 3]
    elif wid == 4:
        x_shape, w_shape = [2, 72, 45], [72, 52, 16]
    elif wid == 5:
        x_shape, w_shape = [2, 64, 9, 11], [64, 16, 3, 3]
        case["group"] = 4
    case["x_shape"], case["w_shape"] = x_shape, w_shape
    for layout in ("nchw", "nhwc"):
        full_parity(case, wl.dtype, 900 + wid, layout)


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_workload_full_size(wid):
    """The workload at full size, auto-chosen kernel (the launch the benchmark
    times): sampled outputs against the oracle, plus whole-output properties."""
    wl = WORKLOADS[wid]
    case = _wl_case(wl)
    x, w, b = make_inputs(wl)
    op, y = gpu_run(case, x, w, b, "nchw", "auto")
    assert not torch.isnan(y).any()
    rng = np.random.default_rng(wid)
    sampled_parity(op, y, x, w, b, case, wl.dtype, "nchw", rng,
                   n_random=400 if wid in (2, 4) else 1500)
    if wid == 1:
        xa, wa, ba = to_oracle(x, w, b, "nchw")
        ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
        check_close(y, ref, absacc, wl.dtype, "workload 1 whole")
    if wid == 5:
        # only odd rows and odd columns receive taps: the rest is the bias, exactly
        bb = b.cuda().view(1, -1, 1, 1).expand(y.shape[0], -1, y.shape[2], y.shape[3])
        assert torch.equal(y[:, :, 0::2, :], bb[:, :, 0::2, :])
        assert torch.equal(y[:, :, :, 0::2], bb[:, :, :, 0::2])
