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
from parity import (check_close, check_points, draw_case, full_parity, gpu_run, sampled_parity,
                    stratified_points, to_oracle, attrs_from)
from oracle import conv_transpose_ref
from transposed_convolution_02_b200 import ct
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


# Kernel that automatic selection must pick for each reduced workload, per
# layout (sizes above the 1e7-FLOP threshold under which the gather kernel is
# chosen, so each reduced case runs on the kernel family of its workload).
REDUCED = {
    1: ([1, 8, 8, 8], [8, 4, 3, 3], None, ("generic", "generic")),
    2: ([2, 96, 13, 21], [96, 40, 4, 4], None, ("dense_tc_pair", "dense_tc")),
    3: ([1, 64, 6, 8, 10], [64, 32, 3, 3, 3], None, ("dense_tc", "dense_tc")),
    4: ([2, 72, 45], [72, 52, 16], None, ("dense_tc_pair", "dense_tc_pair")),
    5: ([2, 128, 12, 14], [128, 16, 3, 3], 8, ("grouped", "generic")),
}


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_workload_reduced(wid):
    """Each workload's attributes on reduced sizes, whole output compared, on
    the kernel automatic selection picks for the workload's family."""
    wl = WORKLOADS[wid]
    case = _wl_case(wl)
    x_shape, w_shape, group, kernels = REDUCED[wid]
    case["x_shape"], case["w_shape"] = list(x_shape), list(w_shape)
    if group is not None:
        case["group"] = group
    for layout, kernel in zip(("nchw", "nhwc"), kernels):
        full_parity(case, wl.dtype, 900 + wid, layout, expect_kernel=kernel)


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_workload_full_size(wid):
    """The workload at full size, auto-chosen kernel (the launch the benchmark
    times): stratified and random outputs against the oracle evaluated point
    by point, plus whole-output properties.  The stratified set holds a point
    for every (image, stride phase, 32-channel block, run of 16 consecutive
    positions of the phase) and both ends of every phase row, so every unit,
    CTA, epilogue warp and channel piece of the kernel is checked."""
    wl = WORKLOADS[wid]
    case = _wl_case(wl)
    x, w, b = make_inputs(wl)
    op, y = gpu_run(case, x, w, b, "nchw", "auto")
    assert not torch.isnan(y).any()
    rng = np.random.default_rng(wid)
    sampled_parity(op, y, x, w, b, case, wl.dtype, "nchw", rng,
                   n_random=400 if wid in (2, 4) else 1500)
    pts = stratified_points(list(y.shape), wl.strides, rng,
                            mblock=16 if wl.group > 1 else 32)
    check_points(op, y, x, w, b, case, wl.dtype, "nchw", pts, "stratified workload %d" % wid)
    if wid == 1:
        xa, wa, ba = to_oracle(x, w, b, "nchw")
        ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
        check_close(y, ref, absacc, wl.dtype, "workload 1 whole")
    if wid == 5:
        # only odd rows and odd columns receive taps: the rest is the bias, exactly
        bb = b.cuda().view(1, -1, 1, 1).expand(y.shape[0], -1, y.shape[2], y.shape[3])
        assert torch.equal(y[:, :, 0::2, :], bb[:, :, 0::2, :])
        assert torch.equal(y[:, :, :, 0::2], bb[:, :, :, 0::2])


# Attribute paths of the ai.onnx.ConvTranspose README ("Attributes") that the
# workloads do not exercise, each through the tensor-core and grouped kernels:
# output_shape (its pads split at the end under NOTSET, like SAME_LOWER under
# SAME_LOWER), VALID, an explicit kernel_shape, and SAME totals that are
# negative (kernel 1, stride 2) under both SAME rules.
ATTR_CASES = [
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 4, 4], strides=[2, 2], output_shape=[17, 19],
         bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 4, 4], strides=[2, 2], output_shape=[17, 19],
         auto_pad="SAME_LOWER", bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 3, 3], strides=[2, 2], auto_pad="VALID",
         bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 4, 4], strides=[2, 2], kernel_shape=[4, 4],
         pads=[1, 2, 0, 1], bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 1, 1], strides=[2, 2], auto_pad="SAME_LOWER",
         bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 1, 1], strides=[2, 2], auto_pad="SAME_UPPER",
         bias=True),
    dict(x_shape=[1, 32, 5, 6, 7], w_shape=[32, 24, 3, 3, 3], strides=[2, 2, 2],
         output_shape=[9, 12, 13], auto_pad="SAME_LOWER", bias=True),
]


@pytest.mark.parametrize("idx", range(len(ATTR_CASES)))
@pytest.mark.parametrize("algo,dtype,layout", [
    ("dense_tc_pair", torch.float16, "nchw"),
    ("dense_tc", torch.float16, "nchw"),
    ("dense_tc", torch.float16, "nhwc"),
    ("dense_tc_pair", torch.float32, "nchw"),
    ("dense_tc_pair", torch.float16, "nhwc"),
])
def test_attribute_paths_on_tensor_cores(idx, algo, dtype, layout):
    case = ATTR_CASES[idx]
    try:
        full_parity(case, dtype, 1200 + idx, layout, algo=algo, expect_kernel=algo)
    except ct.CtError as e:
        # only a kernel-capability refusal at plan time is acceptable
        assert e.status == 9, e
        assert algo == "dense_tc" and len(case["x_shape"]) == 5, (algo, case)


@pytest.mark.parametrize("case", [
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 16, 3, 3], strides=[2, 2], output_shape=[17, 19],
         group=4, bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
         output_shape=[19, 21], auto_pad="SAME_LOWER", group=4, bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 16, 3, 3], strides=[2, 2], auto_pad="VALID",
         group=4, bias=True),
    dict(x_shape=[2, 64, 9, 16], w_shape=[64, 16, 1, 1], strides=[2, 2], auto_pad="SAME_LOWER",
         group=2, bias=True),
    dict(x_shape=[2, 64, 9, 10], w_shape=[64, 16, 3, 3], strides=[2, 2], kernel_shape=[3, 3],
         pads=[0, 2, 1, 1], group=4, bias=True),
])
def test_attribute_paths_grouped(case):
    full_parity(case, torch.float16, 1300, "nchw", algo="grouped", expect_kernel="grouped")


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
def test_channels_last_wrapper(dtype):
    """conv_transpose_nhwc in the ClikaRT::ops::conv_transpose form: input
    [N, D.., C_in], weight [C_in, K.., O/groups], padding as interleaved
    (lo, hi) pairs per spatial dim, activation; checked against the oracle
    with the pads split into the README's begins and ends."""
    rng = np.random.default_rng(17)
    for i, (xs, ws, st, pad_lohi, op_, g, act) in enumerate([
        ([2, 64, 9, 10], [64, 48, 4, 4], [2, 2], [1, 2, 0, 1], [0, 0], 1, "identity"),
        ([2, 64, 9, 10], [64, 48, 3, 3], [2, 2], [2, 0, 1, 1], [1, 1], 1, "relu"),
        ([2, 32, 300], [32, 24, 16], [8], [3, 5], [0], 1, "identity"),
        ([1, 32, 5, 6, 7], [32, 16, 3, 3, 3], [2, 2, 2], [1, 1, 0, 2, 1, 0], [1, 0, 1], 1, "relu"),
        ([2, 64, 7, 9], [64, 8, 3, 3], [2, 2], [1, 0, 0, 1], [0, 0], 4, "identity"),
    ]):
        r = len(xs) - 2
        begins = [pad_lohi[2 * a] for a in range(r)]
        ends = [pad_lohi[2 * a + 1] for a in range(r)]
        case = dict(x_shape=xs, w_shape=ws, strides=st, pads=begins + ends, output_padding=op_,
                    group=g, bias=True, activation=act)
        x, w, b = draw_case(case, dtype, 1400 + i, "nhwc")
        y = ct.conv_transpose_nhwc(x.cuda(), w.cuda(), b.cuda(), stride=st, padding=pad_lohi,
                                   output_padding=op_, groups=g, dilation=[1] * r,
                                   activation=act)
        torch.cuda.synchronize()
        xa, wa, ba = to_oracle(x, w, b, "nhwc")
        ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case), activation=act)
        check_close(y, np.moveaxis(ref, 1, -1), np.moveaxis(absacc, 1, -1), dtype,
                    "conv_transpose_nhwc %d" % i)


def test_channels_first_wrapper():
    """conv_transpose, the one-call channels-first form, on the attribute
    paths of the README table (output_shape, SAME_LOWER, dilations, group)."""
    for i, case in enumerate([
        dict(x_shape=[2, 64, 9, 10], w_shape=[64, 48, 4, 4], strides=[2, 2], output_shape=[17, 19],
             auto_pad="SAME_LOWER", bias=True),
        dict(x_shape=[2, 64, 9, 10], w_shape=[64, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
             auto_pad="SAME_UPPER", group=4, bias=True),
        dict(x_shape=[2, 36, 200], w_shape=[36, 20, 16], strides=[8], pads=[4, 4], bias=False),
    ]):
        dtype = torch.float32 if len(case["x_shape"]) == 3 else torch.float16
        x, w, b = draw_case(case, dtype, 1500 + i)
        y = ct.conv_transpose(x.cuda(), w.cuda(), b.cuda() if b is not None else None,
                              strides=case["strides"], dilations=case.get("dilations"),
                              pads=case.get("pads"), auto_pad=case.get("auto_pad", "NOTSET"),
                              group=case.get("group", 1), output_shape=case.get("output_shape"))
        torch.cuda.synchronize()
        xa, wa, ba = to_oracle(x, w, b, "nchw")
        ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
        check_close(y, ref, absacc, dtype, "conv_transpose %d" % i)


def _dense_case(rng, lim_in):
    case = random_case(rng, groups=(1,), max_cg=1, max_mg=1, lim_in=lim_in,
                       lim_k={1: 9, 2: 5, 3: 3})
    c = int(rng.choice([8, 16, 24, 64, 72, 136]))
    m = int(rng.choice([1, 7, 16, 33, 64, 100, 128, 200]))
    case["x_shape"][1] = c
    case["w_shape"][0] = c
    case["w_shape"][1] = m
    return case


@pytest.mark.parametrize("layout", ["nchw", "nhwc"])
def test_dense_tc_random_sweep(layout):
    """fp16 group-1 shapes on the tcgen05 halo phase-GEMM kernel (falling back
    to the per-tap kernel for rows narrower than 8 J positions): ranks 1-3,
    strides/dilations up to 3-4, negative and asymmetric pads, M not a
    multiple of 16, C spanning partial 64-channel blocks, phases without
    taps (filled with the bias)."""
    rng = np.random.default_rng(300 + (layout == "nhwc"))
    kernels = []
    for i in range(40):
        case = _dense_case(rng, {1: 400, 2: 40, 3: 12})
        op, _ = full_parity(case, torch.float16, 7000 + i, layout, algo="dense_tc")
        assert op.kernel in ("dense_tc", "dense_tc_pertap")
        kernels.append(op.kernel)
    assert kernels.count("dense_tc") >= 20, kernels


@pytest.mark.parametrize("layout", ["nchw", "nhwc"])
def test_dense_tc_pertap_random_sweep(layout):
    """The general per-tap tcgen05 kernel on the same kind of shapes."""
    rng = np.random.default_rng(400 + (layout == "nhwc"))
    for i in range(30):
        case = _dense_case(rng, {1: 300, 2: 20, 3: 7})
        full_parity(case, torch.float16, 8000 + i, layout, algo="dense_tc_pertap",
                    expect_kernel="dense_tc_pertap")


def test_dense_tc_dead_phases_and_degenerate():
    # stride 2, dilation 2: taps land only on odd outputs; the rest is bias
    case = dict(x_shape=[2, 32, 9, 10], w_shape=[32, 24, 3, 3], strides=[2, 2],
                dilations=[2, 2], auto_pad="SAME_UPPER", bias=True)
    for algo in ("dense_tc", "dense_tc_pertap"):
        full_parity(case, torch.float16, 41, "nchw", algo=algo, expect_kernel=algo)
    # 1x1 kernel, stride 1 (the plain GEMM case), and a rank-1 long signal
    for algo in ("dense_tc", "dense_tc_pertap"):
        full_parity(dict(x_shape=[3, 64, 17, 9], w_shape=[64, 48, 1, 1], strides=[1, 1],
                         bias=True), torch.float16, 42, "nchw", algo=algo, expect_kernel=algo)
        full_parity(dict(x_shape=[2, 16, 1000], w_shape=[16, 8, 16], strides=[8], pads=[4, 4],
                         bias=True), torch.float16, 43, "nhwc", algo=algo, expect_kernel=algo)
    # many M-tiles in y with a ragged tail, several channel blocks, both layouts
    for layout in ("nchw", "nhwc"):
        full_parity(dict(x_shape=[2, 136, 23, 70], w_shape=[136, 96, 4, 4], strides=[2, 2],
                         pads=[1, 1, 1, 1], bias=True), torch.float16, 44, layout,
                    algo="dense_tc", expect_kernel="dense_tc")


@pytest.mark.parametrize("algo,dtype,layout,case", [
    ("generic", torch.float32, "nchw", dict(x_shape=[2, 6, 7], w_shape=[6, 4, 3], strides=[2],
                                            pads=[1, 0], group=2, bias=True)),
    ("generic", torch.float16, "nhwc", dict(x_shape=[2, 4, 5, 6], w_shape=[4, 3, 3, 3], strides=[2, 1],
                                            bias=True)),
    ("generic", torch.float32, "nchw", dict(x_shape=[1, 3, 4], w_shape=[3, 2, 3], strides=[90], bias=True)),
    ("dense_tc", torch.float16, "nchw", dict(x_shape=[2, 64, 9, 20], w_shape=[64, 48, 4, 4], strides=[2, 2],
                                             pads=[1, 1, 1, 1], bias=True)),
    ("dense_tc", torch.float16, "nchw", dict(x_shape=[2, 32, 5, 6, 12], w_shape=[32, 32, 3, 3, 3],
                                             strides=[2, 2, 2], dilations=[2, 2, 2], auto_pad="SAME_UPPER",
                                             bias=True)),
    ("dense_tc_pertap", torch.float16, "nhwc", dict(x_shape=[2, 32, 6, 5], w_shape=[32, 16, 3, 3],
                                                    strides=[2, 2], pads=[1, 1, 1, 1], bias=True)),
    ("fp32_gemm", torch.float32, "nchw", dict(x_shape=[2, 24, 40], w_shape=[24, 40, 4], strides=[4],
                                              dilations=[2], pads=[1, 2], bias=True)),
    ("grouped", torch.float16, "nchw", dict(x_shape=[2, 32, 9, 16], w_shape=[32, 16, 3, 3], strides=[2, 2],
                                            dilations=[2, 2], auto_pad="SAME_UPPER", group=2, bias=True)),
    ("grouped", torch.float16, "nchw", dict(x_shape=[2, 64, 7, 9], w_shape=[64, 24, 2, 2], strides=[3, 3],
                                            group=2, bias=True)),
])
def test_relu_activation(algo, dtype, layout, case):
    """The ReLU activation after the bias, in every kernel family and in the
    bias-only outputs of tap-less phases."""
    case = dict(case, activation="relu")
    full_parity(case, dtype, 90, layout, algo=algo, expect_kernel=algo)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_generic_untabled_stride(dtype):
    """Stride 80 (more phases than the phase tables hold): the generic
    kernel's 64-bit form, which tests every tap."""
    full_parity(dict(x_shape=[2, 4, 5], w_shape=[4, 3, 3], strides=[80], bias=True), dtype, 80,
                "nchw", algo="generic", expect_kernel="generic")
    full_parity(dict(x_shape=[1, 6, 3, 2], w_shape=[6, 2, 2, 3], strides=[70, 3], dilations=[2, 1],
                     pads=[3, 1, 0, 2], group=2, bias=True), dtype, 81, "nhwc", algo="generic",
                expect_kernel="generic")


def test_grouped_random_sweep():
    """fp16 grouped channels-first shapes on the mma.sync grouped phase kernel:
    ranks 1-2, 16-64 channels per group, strides/dilations up to 3, pads,
    output_padding, phases without taps (bias only)."""
    rng = np.random.default_rng(500)
    for i in range(40):
        case = random_case(rng, max_rank=2, groups=(2, 4, 8), max_cg=1, max_mg=1,
                           lim_in={1: 60, 2: 14}, lim_k={1: 5, 2: 4}, strides=(1, 4),
                           dils=(1, 4))
        g = case["group"]
        cg = int(rng.choice([16, 32, 48, 64]))
        mg = int(rng.choice([8, 16, 24, 40, 64]))
        case["x_shape"][1] = cg * g
        case["w_shape"][0] = cg * g
        case["w_shape"][1] = mg
        full_parity(case, torch.float16, 9000 + i, "nchw", algo="grouped", expect_kernel="grouped")


def test_grouped_bias_only_phases_exact():
    # the grouped workload's geometry (stride 2, dilation 2, SAME_UPPER) at a
    # smaller size: 3/4 of the outputs are exactly the bias
    case = dict(x_shape=[2, 64, 13, 11], w_shape=[64, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
                auto_pad="SAME_UPPER", group=4, bias=True)
    x, w, b = draw_case(case, torch.float16, 61)
    op, y = gpu_run(case, x, w, b, "nchw", "grouped")
    assert op.kernel == "grouped"
    bb = b.cuda().view(1, -1, 1, 1)
    assert torch.equal(y[:, :, 0::2, :], bb.expand_as(y[:, :, 0::2, :]))
    assert torch.equal(y[:, :, :, 0::2], bb.expand_as(y[:, :, :, 0::2]))
    full_parity(case, torch.float16, 61, "nchw", algo="grouped", expect_kernel="grouped")


@pytest.mark.parametrize("case", [
    # one stride phase with taps in each axis (stride 2, dilation 2, kernel 3):
    # 16-byte stores (out_x % 8 == 0), a ragged segment and row-block tail
    dict(x_shape=[2, 32, 13, 12], w_shape=[32, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_UPPER", group=2, bias=True),
    # 8-byte stores (out_x % 8 == 4), half an output-channel tile (M/group = 8)
    dict(x_shape=[3, 64, 7, 10], w_shape=[64, 8, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_UPPER", group=4, bias=True),
    # the even column phase carries the taps (SAME_LOWER), no bias
    dict(x_shape=[2, 32, 9, 16], w_shape=[32, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_LOWER", group=2, bias=False),
    # rank 1
    dict(x_shape=[2, 48, 40], w_shape=[48, 16, 3], strides=[2], dilations=[2],
         auto_pad="SAME_UPPER", group=3, bias=True),
    # one tap (kernel 1, output_padding 1) and two k-steps per tap (32 channels per group)
    dict(x_shape=[2, 64, 8, 8], w_shape=[64, 16, 1, 1], strides=[2, 2], output_padding=[1, 1],
         group=2, bias=True),
    # four taps (kernel 2, dilation 2, output_padding 1 so that out_x % 4 == 0)
    dict(x_shape=[2, 32, 11, 11], w_shape=[32, 8, 2, 2], strides=[2, 2], dilations=[2, 2],
         output_padding=[1, 1], group=2, bias=True),
])
def test_grouped_one_phase_path(case):
    """Grouped shapes whose outputs get taps in one stride phase only (the
    path that keeps the weights in registers and stores (bias, value) pairs)."""
    full_parity(case, torch.float16, 70, "nchw", algo="grouped", expect_kernel="grouped")


@pytest.mark.parametrize("case", [
    # many row blocks per CTA (16 images x 32 groups): the persistent CTAs
    # walk several blocks each, with the tile of the next one in flight
    dict(x_shape=[16, 512, 16, 16], w_shape=[512, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_UPPER", group=32, bias=True),
    # ragged last row block, the taps in the even phases (SAME_LOWER), ReLU
    dict(x_shape=[3, 64, 21, 24], w_shape=[64, 16, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_LOWER", group=4, bias=True, activation="relu"),
    # 64 channels per group (eight 8-channel pieces per pixel), 8 output channels
    dict(x_shape=[2, 128, 10, 16], w_shape=[128, 8, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_UPPER", group=2, bias=True),
    # rank 1 with a 256-wide output row, no bias
    dict(x_shape=[4, 96, 128], w_shape=[96, 16, 3], strides=[2], dilations=[2],
         auto_pad="SAME_UPPER", group=6, bias=False),
    # stride 3 in y (two tap-less row phases), a 1x1 kernel (one tap),
    # output_padding on both axes
    dict(x_shape=[2, 32, 12, 16], w_shape=[32, 16, 1, 1], strides=[3, 2], pads=[0, 0, 0, 0],
         output_padding=[2, 1], group=2, bias=True),
    # dilation 2 with kernels of 2 and 3 taps, 16 and 32 channels per group:
    # 2, 4, 6, 8 and 12 (tap, 16-channel step) MMA steps per output tile
    dict(x_shape=[2, 32, 12, 16], w_shape=[32, 16, 1, 2], strides=[2, 2], dilations=[2, 2], pads=[0, 0, 0, 1],
         group=2, bias=True),
    dict(x_shape=[2, 32, 12, 16], w_shape=[32, 16, 2, 2], strides=[2, 2], dilations=[2, 2], pads=[0, 0, 0, 1],
         group=2, bias=True, activation="relu"),
    dict(x_shape=[2, 32, 12, 16], w_shape=[32, 16, 2, 3], strides=[2, 2], dilations=[2, 2], pads=[0, 1, 0, 2],
         group=2, bias=True),
    dict(x_shape=[2, 64, 12, 16], w_shape=[64, 16, 2, 2], strides=[2, 2], dilations=[2, 2], pads=[0, 0, 0, 1],
         group=2, bias=True),
    dict(x_shape=[2, 64, 12, 16], w_shape=[64, 16, 2, 3], strides=[2, 2], dilations=[2, 2], pads=[0, 1, 0, 2],
         group=2, bias=False),
    # rank 1, four taps
    dict(x_shape=[4, 96, 64], w_shape=[96, 16, 4], strides=[2], dilations=[2], pads=[0, 5], group=6, bias=True),
])
def test_grouped_stream_path(case):
    """One-phase grouped shapes with 16-byte output rows (out_x % 8 == 0, at
    most 256): the persistent form of the grouped kernel, whose tap-less rows
    leave by TMA tensor stores of a bias tile.  Outputs that no tap reaches
    must be exactly the activated bias; the rest within the fp16 tolerance."""
    x, w, b = draw_case(case, torch.float16, 83)
    op, y = gpu_run(case, x, w, b, "nchw", "grouped")
    assert op.kernel == "grouped"
    xa, wa, ba = to_oracle(x, w, b, "nchw")
    act = case.get("activation", "identity")
    ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case), activation=act)
    check_close(y, ref, absacc, torch.float16, "%s grouped" % (case,))
    bias_only = torch.from_numpy(absacc == 0)
    assert bias_only.any()
    bb = (b.float() if b is not None else torch.zeros(case["w_shape"][1] * case["group"]))
    bb = (bb.clamp_min(0) if act == "relu" else bb).half()
    want = bb.view([1, -1] + [1] * (y.dim() - 2)).expand(y.shape)
    got = y.cpu()
    assert torch.equal(got[bias_only], want[bias_only])


@pytest.mark.parametrize("layout", ["nchw", "nhwc"])
def test_fp32_gemm_random_sweep(layout):
    """fp32 group-1 shapes on the register-tiled FFMA phase GEMM: ranks 1-3,
    strides/dilations up to 3-4, pads, output_padding, C not a multiple of 8,
    M not a multiple of 128, phases without taps."""
    rng = np.random.default_rng(600 + (layout == "nhwc"))
    for i in range(40):
        case = random_case(rng, groups=(1,), max_cg=1, max_mg=1,
                           lim_in={1: 300, 2: 24, 3: 8}, lim_k={1: 9, 2: 5, 3: 3})
        c = int(rng.choice([1, 3, 8, 20, 64, 72]))
        m = int(rng.choice([1, 5, 33, 128, 130, 200]))
        case["x_shape"][1] = c
        case["w_shape"][0] = c
        case["w_shape"][1] = m
        full_parity(case, torch.float32, 11000 + i, layout, algo="fp32_gemm",
                    expect_kernel="fp32_gemm")


@pytest.mark.parametrize("algo,dtype,layout,case", [
    ("dense_tc", torch.float16, "nchw", dict(x_shape=[2, 64, 9, 20], w_shape=[64, 72, 4, 4], strides=[2, 2],
                                             pads=[1, 1, 1, 1], bias=True)),
    ("dense_tc", torch.float16, "nhwc", dict(x_shape=[2, 64, 9, 20], w_shape=[64, 72, 4, 4], strides=[2, 2],
                                             pads=[1, 1, 1, 1], bias=True)),
    ("dense_tc_pertap", torch.float16, "nchw", dict(x_shape=[2, 32, 6, 5], w_shape=[32, 40, 3, 3],
                                                    strides=[2, 2], pads=[1, 1, 1, 1], bias=True)),
    ("grouped", torch.float16, "nchw", dict(x_shape=[2, 64, 7, 9], w_shape=[64, 24, 2, 2], strides=[2, 2],
                                            group=2, bias=True)),
    ("fp32_gemm", torch.float32, "nchw", dict(x_shape=[2, 24, 40], w_shape=[24, 40, 4], strides=[4],
                                              pads=[1, 2], bias=True)),
    ("generic", torch.float16, "nchw", dict(x_shape=[2, 6, 7], w_shape=[6, 4, 3], strides=[2], bias=True)),
    ("dense_tc_pair", torch.float16, "nchw", dict(x_shape=[2, 64, 9, 20], w_shape=[64, 72, 4, 4],
                                                  strides=[2, 2], pads=[1, 1, 1, 1], bias=True)),
])
def test_bias_off_16_byte_boundary(algo, dtype, layout, case):
    """A bias that starts one element past a 16-byte boundary (a view into a
    larger tensor): the kernels that read the bias in 16-byte pieces take
    their element-wise path instead."""
    x, w, b = draw_case(case, dtype, 95, layout)
    store = torch.zeros(b.numel() + 1, dtype=dtype, device="cuda")
    store[1:] = b.cuda()
    bview = store[1:]
    assert bview.data_ptr() % 16 != 0
    op = ct.ConvTranspose(w.cuda(), list(x.shape), bview, layout=layout, strides=case["strides"],
                          dilations=case.get("dilations"), pads=case.get("pads"),
                          group=case.get("group", 1), algo=algo)
    assert op.kernel == algo, op.kernel
    y = torch.full(op.y_shape, float("nan"), dtype=dtype, device="cuda")
    op(x.cuda(), out=y)
    torch.cuda.synchronize()
    xa, wa, ba = to_oracle(x, w, b, layout)
    ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
    if layout == "nhwc":
        ref = np.moveaxis(ref, 1, -1)
        absacc = np.moveaxis(absacc, 1, -1)
    check_close(y, ref, absacc, dtype, "unaligned bias %s %s" % (algo, layout))


def _pair_case(rng):
    case = random_case(rng, max_rank=3, groups=(1,), max_cg=1, max_mg=1,
                       lim_in={1: 700, 2: 40, 3: 12}, lim_k={1: 9, 2: 5, 3: 3})
    c = int(rng.choice([8, 16, 24, 64, 72, 136, 256]))
    m = int(rng.choice([1, 7, 16, 33, 64, 100, 128, 200, 256]))
    case["x_shape"][1] = c
    case["w_shape"][0] = c
    case["w_shape"][1] = m
    return case


def test_dense_tc_pair_random_sweep():
    """fp16 group-1 channels-first shapes with one to three spatial axes on
    the CTA-pair tcgen05 kernel: strides/dilations up to 4, negative and
    asymmetric pads, output_padding, M not a multiple of 16 (up to 256), C
    spanning partial 64-channel blocks, phases without taps.  Shapes whose
    padded input runs exceed the kernel's tile are refused at plan time."""
    rng = np.random.default_rng(600)
    ran = 0
    for i in range(70):
        case = _pair_case(rng)
        try:
            full_parity(case, torch.float16, 9000 + i, "nchw", algo="dense_tc_pair",
                        expect_kernel="dense_tc_pair")
        except ct.CtError as e:
            assert e.status == 9, e   # CT_ERR_UNSUPPORTED from ct_plan
            continue
        ran += 1
    assert ran >= 30, ran


@pytest.mark.parametrize("case", [
    # the 2-D decoder's attributes on a smaller image: several units per image, ragged tail
    dict(x_shape=[3, 256, 21, 23], w_shape=[256, 128, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1], bias=True),
    # M = 256 (one phase per accumulator buffer) and M = 200 (Np 208)
    dict(x_shape=[2, 64, 11, 13], w_shape=[64, 256, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1], bias=True),
    dict(x_shape=[2, 72, 9, 17], w_shape=[72, 200, 3, 3], strides=[2, 2], pads=[1, 1, 1, 1],
         output_padding=[1, 1], bias=True),
    # stride 1 (a plain 3x3 convolution with tap-reversed weights), no bias
    dict(x_shape=[2, 64, 30, 30], w_shape=[64, 64, 3, 3], strides=[1, 1], pads=[1, 1, 1, 1]),
    # taps only on odd outputs: the rest is the bias
    dict(x_shape=[2, 32, 9, 10], w_shape=[32, 48, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_UPPER", bias=True),
    # one spatial axis: a long fp16 vocoder-style upsample
    dict(x_shape=[2, 64, 3000], w_shape=[64, 32, 16], strides=[8], pads=[4, 4], bias=True),
    # stride 3, odd output width (no paired x phases), C = 8
    dict(x_shape=[1, 8, 15, 19], w_shape=[8, 24, 5, 5], strides=[3, 3], pads=[2, 1, 0, 2], bias=True),
    # the 3-D upsample's attributes on a smaller volume (two input slices per unit)
    dict(x_shape=[2, 64, 6, 9, 11], w_shape=[64, 32, 3, 3, 3], strides=[2, 2, 2], pads=[1, 1, 1, 1, 1, 1],
         output_padding=[1, 1, 1]),
    # 3-D, stride 1 along z (three input slices), M = 40
    dict(x_shape=[1, 16, 5, 7, 6], w_shape=[16, 40, 3, 2, 2], strides=[1, 2, 2], pads=[1, 0, 0, 1, 1, 0],
         bias=True),
])
def test_dense_tc_pair_cases(case):
    full_parity(case, torch.float16, 77, "nchw", algo="dense_tc_pair", expect_kernel="dense_tc_pair")
    full_parity(dict(case, activation="relu"), torch.float16, 78, "nchw", algo="dense_tc_pair",
                expect_kernel="dense_tc_pair")


@pytest.mark.parametrize("case", [
    # the 1-D vocoder's attributes on a shorter signal
    dict(x_shape=[2, 64, 300], w_shape=[64, 48, 16], strides=[8], pads=[4, 4], bias=True),
    # 2-D stride 2 with M = 40 and C = 36 (a partial 32-channel block)
    dict(x_shape=[2, 36, 9, 13], w_shape=[36, 40, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1], bias=True),
    # 3-D, odd output width, no bias
    dict(x_shape=[1, 32, 4, 5, 7], w_shape=[32, 24, 3, 3, 3], strides=[2, 2, 2], pads=[1, 1, 1, 1, 1, 1]),
    # taps only on odd outputs
    dict(x_shape=[2, 16, 7, 8], w_shape=[16, 32, 3, 3], strides=[2, 2], dilations=[2, 2],
         auto_pad="SAME_UPPER", bias=True),
])
def test_dense_tc_pair_fp32(case):
    """The CTA-pair kernel on fp32 operands (3xTF32: high and low TF32 parts,
    three MMAs per step) within the fp32 tolerance."""
    full_parity(case, torch.float32, 79, "nchw", algo="dense_tc_pair", expect_kernel="dense_tc_pair")
    full_parity(dict(case, activation="relu"), torch.float32, 80, "nchw", algo="dense_tc_pair",
                expect_kernel="dense_tc_pair")


def test_dense_tc_pair_fp32_random_sweep():
    """fp32 group-1 channels-first shapes with one to three spatial axes on the
    3xTF32 CTA-pair kernel, compared with the fp64 oracle at the fp32
    tolerance."""
    rng = np.random.default_rng(610)
    ran = 0
    for i in range(40):
        case = _pair_case(rng)
        case["x_shape"][1] = case["w_shape"][0] = int(rng.choice([4, 12, 32, 36, 64, 100]))
        try:
            full_parity(case, torch.float32, 9500 + i, "nchw", algo="dense_tc_pair",
                        expect_kernel="dense_tc_pair")
        except ct.CtError as e:
            assert e.status == 9, e
            continue
        ran += 1
    assert ran >= 15, ran


@pytest.mark.parametrize("case", [
    # 128-position tiles of two input rows (W = 64), padded origin (1, 1)
    dict(x_shape=[2, 64, 8, 64], w_shape=[64, 32, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1], bias=True),
    # W = 32 (four rows per tile), 72 channels (a partial 64-channel block), stride 1
    dict(x_shape=[1, 72, 4, 32], w_shape=[72, 16, 3, 3], strides=[1, 1], pads=[1, 1, 1, 1], bias=True),
    # W = 128 (one row per tile), a 1x1 kernel: no halo, padded origin 0
    dict(x_shape=[2, 128, 4, 128], w_shape=[128, 32, 1, 1], strides=[1, 1], bias=False),
    # 3-D on the pair kernel, k = s (no halo), 16 x 16 slices
    dict(x_shape=[1, 64, 2, 8, 16], w_shape=[64, 16, 2, 2, 2], strides=[2, 2, 2], bias=True),
])
def test_dense_tc_pair_whole_row_tiles(case):
    """fp16 channels-first shapes whose 128-position re-layout tiles are whole
    input rows (W of 32, 64 or 128), with and without a halo, a partial
    64-channel block and a 3-D volume: the whole output against the oracle."""
    full_parity(case, torch.float16, 91, "nchw", algo="dense_tc_pair", expect_kernel="dense_tc_pair")


@pytest.mark.parametrize("dtype,case", [
    (torch.float16, dict(x_shape=[2, 64, 11, 13], w_shape=[64, 72, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1],
                         bias=True)),
    (torch.float16, dict(x_shape=[2, 24, 300], w_shape=[24, 40, 16], strides=[8], pads=[4, 4], bias=True)),
    (torch.float16, dict(x_shape=[1, 16, 4, 5, 6], w_shape=[16, 24, 3, 3, 3], strides=[2, 2, 2],
                         pads=[1, 1, 1, 1, 1, 1], output_padding=[1, 1, 1], bias=True)),
    (torch.float32, dict(x_shape=[2, 32, 9, 10], w_shape=[32, 48, 3, 3], strides=[2, 2], dilations=[2, 2],
                         auto_pad="SAME_UPPER", bias=True)),
    (torch.float32, dict(x_shape=[2, 36, 200], w_shape=[36, 20, 16], strides=[8], pads=[4, 4])),
])
def test_dense_tc_pair_channels_last(dtype, case):
    """Channels-last X, W ([C, k.., M]) and Y on the CTA-pair kernel: the
    padding copy instead of the transpose, channel rows stored as 16-byte
    pieces."""
    full_parity(case, dtype, 83, "nhwc", algo="dense_tc_pair", expect_kernel="dense_tc_pair")
    full_parity(dict(case, activation="relu"), dtype, 84, "nhwc", algo="dense_tc_pair",
                expect_kernel="dense_tc_pair")


@pytest.mark.parametrize("dtype,layout,case", [
    # 300 output channels: two tiles of 160, the second partly beyond M
    (torch.float16, "nchw", dict(x_shape=[2, 64, 9, 11], w_shape=[64, 300, 4, 4], strides=[2, 2],
                                 pads=[1, 1, 1, 1], bias=True)),
    # 3-D with 320 output channels (no tuned fp16 kernel takes more than 256)
    (torch.float16, "nchw", dict(x_shape=[1, 32, 4, 5, 6], w_shape=[32, 320, 3, 3, 3], strides=[2, 2, 2],
                                 pads=[1, 1, 1, 1, 1, 1], output_padding=[1, 1, 1], bias=True)),
    (torch.float16, "nhwc", dict(x_shape=[2, 32, 7, 9], w_shape=[32, 272, 3, 3], strides=[2, 2],
                                 pads=[1, 1, 1, 1], bias=True)),
    (torch.float32, "nchw", dict(x_shape=[2, 36, 100], w_shape=[36, 512, 16], strides=[8], pads=[4, 4],
                                 bias=True)),
])
def test_dense_tc_pair_channel_tiles(dtype, layout, case):
    """More than 256 output channels: the pair kernel walks output-channel
    tiles of at most 256 (one MMA's N); automatic selection takes it."""
    full_parity(case, dtype, 85, layout, expect_kernel="dense_tc_pair")
    full_parity(dict(case, activation="relu"), dtype, 86, layout, algo="dense_tc_pair",
                expect_kernel="dense_tc_pair")


@pytest.mark.parametrize("dtype,case", [
    # (sizes above the 10 MFLOP below which the generic kernel is chosen)
    (torch.float16, dict(x_shape=[4, 3, 40, 48], w_shape=[3, 64, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1],
                         bias=True)),
    (torch.float16, dict(x_shape=[2, 12, 8, 10, 12], w_shape=[12, 16, 3, 3, 3], strides=[2, 2, 2],
                         pads=[1, 1, 1, 1, 1, 1], bias=True)),
    (torch.float32, dict(x_shape=[4, 5, 2000], w_shape=[5, 24, 8], strides=[4], pads=[2, 2], bias=True)),
])
def test_dense_tc_pair_channels_padded(dtype, case):
    """Input channels that do not fill a 16-byte row (C = 3, 12, 5): the
    channels-first re-layout pads them with zeros; automatic selection takes
    the pair kernel instead of the generic one."""
    full_parity(case, dtype, 87, "nchw", expect_kernel="dense_tc_pair")


@pytest.mark.parametrize("idx", range(6))
def test_general_shapes_sampled(idx):
    """The shapes ``bench.py --general`` times (stride-1 3x3, 1x1, channels-last,
    512 output channels, 3 input channels, fp32 2-D), at the timed size and
    with the automatically chosen kernel: sampled outputs against the oracle."""
    import bench

    name, xs, ws, dt, layout, kw = bench.GENERAL_SHAPES[idx]
    case = dict(x_shape=list(xs), w_shape=list(ws), strides=kw["strides"], pads=kw.get("pads"),
                bias=True)
    x, w, b = draw_case(case, dt, 900 + 10 * idx, layout)
    op, y = gpu_run(case, x, w, b, layout, "auto")
    assert op.kernel in ("dense_tc_pair", "dense_tc"), (name, op.kernel)
    assert not torch.isnan(y).any(), name
    sampled_parity(op, y, x, w, b, case, dt, layout, np.random.default_rng(idx), n_random=600)


def test_multi_device_batch_split():
    """MultiDeviceConvTranspose: one caller's batch split into slices, one
    plan and packed weight per device, Y gathered on the first device.  With
    one GPU the slices share cuda:0, which still runs the split, the per-slice
    plans and the gather through the library's kernels."""
    from transposed_convolution_02_b200.shard import MultiDeviceConvTranspose
    # (every slice above the 1e7 FLOP under which the gather kernel is chosen)
    case = dict(x_shape=[5, 64, 16, 20], w_shape=[64, 48, 4, 4], strides=[2, 2],
                pads=[1, 1, 1, 1], bias=True)
    x, w, b = draw_case(case, torch.float16, 1600)
    md = MultiDeviceConvTranspose(w.cuda(), case["x_shape"], b.cuda(), devices=["cuda:0"] * 3,
                                  strides=case["strides"], pads=case["pads"])
    assert [op.x_shape[0] for op in md.ops] == [2, 2, 1]
    assert all(op.kernel == "dense_tc_pair" for op in md.ops)
    y = md.gather(md(x.cuda()))
    torch.cuda.synchronize()
    xa, wa, ba = to_oracle(x, w, b, "nchw")
    ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
    check_close(y, ref, absacc, torch.float16, "multi-device batch split")


@pytest.mark.parametrize("case", [
    # the 3-D upsample's attributes: J_x 12 of a 32-wide row segment, ragged y and z
    dict(x_shape=[2, 64, 6, 7, 12], w_shape=[64, 32, 3, 3, 3], strides=[2, 2, 2],
         pads=[1, 1, 1, 1, 1, 1], output_padding=[1, 1, 1]),
    # odd out_y (the last row's second y phase lies outside Y), bias
    dict(x_shape=[1, 32, 4, 5, 8], w_shape=[32, 16, 3, 3, 3], strides=[2, 2, 2],
         pads=[1, 1, 1, 1, 1, 1], output_padding=[1, 0, 1], bias=True),
    # 2-D decoder-like: 64-wide rows (two warps per row), M = 72 (a one-chunk channel block)
    dict(x_shape=[2, 32, 5, 64], w_shape=[32, 72, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1], bias=True),
    # J_x = 200: two x tiles of 128 (kernel 2, stride 2: one tap per phase)
    dict(x_shape=[1, 16, 3, 200], w_shape=[16, 24, 2, 2], strides=[2, 2], bias=True),
    # stride 1 along x (one x phase per store), M = 40
    dict(x_shape=[2, 32, 10, 24], w_shape=[32, 40, 3, 3], strides=[1, 1], pads=[1, 1, 1, 1], bias=True),
    # 1-D, 100 positions per row
    dict(x_shape=[2, 64, 100], w_shape=[64, 32, 4], strides=[2], pads=[1, 1], bias=True),
    # 20 positions per row, C = 136 (three channel blocks)
    dict(x_shape=[2, 136, 9, 20], w_shape=[136, 48, 4, 4], strides=[2, 2], pads=[1, 1, 1, 1], bias=True),
])
def test_dense_tc_row_mode(case):
    """The halo kernel's row mode (whole output rows per unit, one TMA box per
    x offset, epilogue tiles written by TMA tensor stores with the parts
    outside Y clipped): channels-first fp16 shapes with every phase live and
    out_x a multiple of 8, identity and ReLU."""
    full_parity(case, torch.float16, 97, "nchw", algo="dense_tc", expect_kernel="dense_tc")
    full_parity(dict(case, activation="relu"), torch.float16, 98, "nchw", algo="dense_tc",
                expect_kernel="dense_tc")
