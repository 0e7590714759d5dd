"""Host-side checks of libct.so that need no GPU: the library loads, exports
every entry point include/ct.h declares, and its resolver agrees with the
oracle's independent resolver on random attribute sets."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from cases import attrs_of, random_case
from oracle import Attrs, ResolveError, resolve_full
from transposed_convolution_02_b200 import ct
from transposed_convolution_02_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"CT_API\s+[\w\s\*]*?\b(ct_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    L = ct.lib()
    declared = _declared_symbols()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(L, name), name
    assert declared == set(ct.EXPORTED)


def test_status_strings():
    for code in range(0, 11):
        assert ct.ct_status_string(code)
    assert ct.ct_status_string(0) == "ok"


def _desc_from_case(case, layout="nchw", dtype=torch.float32):
    x_shape, w_shape = list(case["x_shape"]), list(case["w_shape"])
    if layout == "nhwc":
        x_shape = [x_shape[0]] + x_shape[2:] + [x_shape[1]]
        w_shape = [w_shape[0]] + w_shape[2:] + [w_shape[1]]
    m = case["w_shape"][1] * case["group"]
    return ct.make_desc(x_shape, w_shape, dtype=dtype, layout=layout,
                        strides=case["strides"], dilations=case.get("dilations"),
                        pads=case.get("pads"), output_padding=case.get("output_padding"),
                        auto_pad=case.get("auto_pad", "NOTSET"), group=case["group"],
                        bias_len=m if case.get("bias") else 0,
                        kernel_shape=case.get("kernel_shape"),
                        output_shape=case.get("output_shape"))


@pytest.mark.parametrize("layout", ["nchw", "nhwc"])
def test_resolver_agrees_with_oracle(layout):
    rng = np.random.default_rng(99)
    modes = ["NOTSET", "NOTSET", "SAME_UPPER", "SAME_LOWER", "VALID"]
    n_ok = n_err = 0
    for _ in range(3000):
        case = random_case(rng, pads=(-2, 4))
        r = len(case["strides"])
        case["auto_pad"] = str(rng.choice(modes))
        if case["auto_pad"] != "NOTSET" and rng.random() < 0.8:
            case["pads"] = [0] * (2 * r)
        # perturb to reach the error paths too
        u = rng.random()
        if u < 0.05:
            case["output_padding"][0] = max(case["strides"][0], case["dilations"][0])
        elif u < 0.10:
            case["kernel_shape"] = [k + 1 for k in case["w_shape"][2:]]
        elif u < 0.25:
            case["output_shape"] = [int(v) for v in rng.integers(1, 30, size=r)]
        elif u < 0.28:
            case["strides"][0] = 0
        try:
            yshape, res = resolve_full(case["x_shape"], case["w_shape"], attrs_of(case))
            want = ("ok", yshape, res.pad_begin, res.pad_end)
        except ResolveError:
            want = ("err",)
        d = _desc_from_case(case, layout)
        try:
            ys, pb, pe = ct.ct_output_shape(d)
            if layout == "nhwc":
                ys = [ys[0], ys[-1]] + ys[1:-1]
            got = ("ok", ys, pb, pe)
        except ct.CtError:
            got = ("err",)
        assert got == want, (case, got, want)
        n_ok += want[0] == "ok"
        n_err += want[0] == "err"
    assert n_ok > 1000 and n_err > 100


def test_error_classes():
    base = dict(x_shape=[1, 4, 5], w_shape=[4, 3, 3], strides=[2], pads=[1, 1], group=2)

    def status(**over):
        c = dict(base)
        c.update(over)
        d = _desc_from_case(c)
        for k in ("bias_len",):
            if k in over:
                setattr(d, k, over[k])
        try:
            ct.ct_output_shape(d)
            return 0
        except ct.CtError as e:
            return e.status

    assert status() == 0
    assert status(group=3) == 1                       # C % group
    assert status(w_shape=[3, 3, 3]) == 1             # W[0] != C
    assert status(bias_len=5) == 1                    # bias length != M = 6
    assert status(output_padding=[2]) == 4            # op >= max(s, d)
    assert status(strides=[0]) == 4
    assert status(kernel_shape=[2]) == 4
    assert status(auto_pad="SAME_UPPER") == 4         # pads with auto_pad
    d = _desc_from_case(base)
    d.rank = 4
    with pytest.raises(ct.CtError) as e:
        ct.ct_output_shape(d)
    assert e.value.status == 2
    d = _desc_from_case(base)
    d.dtype = 7
    with pytest.raises(ct.CtError) as e:
        ct.ct_output_shape(d)
    assert e.value.status == 3
    d = _desc_from_case(base)
    d.activation = 2                                  # only identity (0) and relu (1)
    with pytest.raises(ct.CtError) as e:
        ct.ct_output_shape(d)
    assert e.value.status == 4
    d.activation = 1
    ct.ct_output_shape(d)


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_workload_shapes_and_plan(wid):
    wl = WORKLOADS[wid]
    case = dict(x_shape=wl.x_shape, w_shape=wl.w_shape, strides=wl.strides,
                dilations=wl.dilations, pads=wl.pads, output_padding=wl.output_padding,
                auto_pad=wl.auto_pad, group=wl.group, bias=wl.bias)
    d = _desc_from_case(case, dtype=wl.dtype)
    ys, pb, pe = ct.ct_output_shape(d)
    assert ys == list(wl.y_shape)
    plan = ct.ct_plan(d)
    try:
        assert ct.ct_plan_kernel(plan) in ("generic", "dense_tc", "dense_tc_pair", "fp32_gemm", "grouped")
        assert ct.ct_prepacked_weight_bytes(plan) > 0
        assert ct.ct_workspace_bytes(plan) >= 0
    finally:
        ct.ct_plan_destroy(plan)


def test_forced_generic_and_unsupported():
    case = dict(x_shape=[1, 4, 5], w_shape=[4, 3, 3], strides=[2], pads=[1, 1], group=2)
    d = _desc_from_case(case)
    d.algo = ct.ALGO["generic"]
    plan = ct.ct_plan(d)
    assert ct.ct_plan_kernel(plan) == "generic"
    ct.ct_plan_destroy(plan)
    d.algo = ct.ALGO["dense_tc"]    # fp32 grouped: the tensor-core kernel cannot serve it
    with pytest.raises(ct.CtError) as e:
        ct.ct_plan(d)
    assert e.value.status == 9


def test_run_argument_checks_without_device():
    case = dict(x_shape=[1, 4, 5], w_shape=[4, 3, 3], strides=[2], pads=[1, 1], group=2,
                bias=True)
    plan = ct.ct_plan(_desc_from_case(case))
    try:
        P = ctypes.c_void_p
        # NULL y, NULL bias while a bias is declared: rejected before any device call
        with pytest.raises(ct.CtError) as e:
            ct.ct_run(plan, P(4096), P(4096), P(4096), P(0), P(0), P(0))
        assert e.value.status == 6
        with pytest.raises(ct.CtError) as e:
            ct.ct_run(plan, P(4096), P(4096), P(0), P(4096), P(0), P(0))
        assert e.value.status == 6
        with pytest.raises(ct.CtError) as e:   # fp32 y at an odd address
            ct.ct_run(plan, P(4096), P(4096), P(4096), P(4097), P(0), P(0))
        assert e.value.status == 5
        # ct_run_parts: the same checks; an unknown part bit is an attribute
        # error, an empty mask launches nothing
        with pytest.raises(ct.CtError) as e:
            ct.ct_run_parts(plan, P(4096), P(4096), P(4096), P(0), P(0), P(0), ct.PART_MAIN)
        assert e.value.status == 6
        with pytest.raises(ct.CtError) as e:
            ct.ct_run_parts(plan, P(4096), P(4096), P(4096), P(4096), P(0), P(0), 4)
        assert e.value.status == 4
        ct.ct_run_parts(plan, P(4096), P(4096), P(4096), P(4096), P(0), P(0), 0)
    finally:
        ct.ct_plan_destroy(plan)


def test_selftest_argument_checks_without_device():
    """The bounded-wait self-test refuses a limit outside 1 .. 2^31 before
    touching a device, and reports CT_ERR_DEVICE when there is none."""
    L = ct.lib()
    assert L.ct_selftest_wait_timeout(None, 0) == 4
    assert L.ct_selftest_wait_timeout(None, (1 << 31) + 1) == 4
    if not torch.cuda.is_available():
        assert L.ct_selftest_wait_timeout(None, 1000) == 7


def _kernel_for(x_shape, w_shape, dtype, layout="nchw", strides=None, pads=None, group=1):
    case = dict(x_shape=x_shape, w_shape=w_shape, strides=strides or [2] * (len(x_shape) - 2),
                pads=pads, group=group, bias=True)
    plan = ct.ct_plan(_desc_from_case(case, layout=layout, dtype=dtype))
    try:
        return (ct.ct_plan_kernel(plan), ct.ct_workspace_bytes(plan),
                ct.ct_prepacked_weight_bytes(plan))
    finally:
        ct.ct_plan_destroy(plan)


@pytest.mark.parametrize("x_shape,w_shape,dtype,layout,kernel", [
    # tiny problems: one gather launch
    ([1, 8, 8, 8], [8, 4, 3, 3], torch.float32, "nchw", "generic"),
    # fp16 dense, channels-first, one or two axes: the CTA-pair kernel
    ([8, 256, 64, 64], [256, 128, 4, 4], torch.float16, "nchw", "dense_tc_pair"),
    ([4, 64, 3000], [64, 32, 16], torch.float16, "nchw", "dense_tc_pair"),
    # fp16 dense, 3-D or channels-last: the single-SM halo kernel
    ([2, 64, 32, 32, 32], [64, 32, 3, 3, 3], torch.float16, "nchw", "dense_tc"),
    ([8, 256, 64, 64], [256, 128, 4, 4], torch.float16, "nhwc", "dense_tc"),
    # more than 256 output channels, or channels that do not fill a 16-byte
    # row: only the pair kernel takes them
    ([2, 64, 8, 8, 8], [64, 320, 3, 3, 3], torch.float16, "nchw", "dense_tc_pair"),
    ([8, 256, 32, 32], [256, 512, 4, 4], torch.float16, "nchw", "dense_tc_pair"),
    ([4, 3, 40, 48], [3, 64, 4, 4], torch.float16, "nchw", "dense_tc_pair"),
    # fp32: 3xTF32 on the pair kernel, both layouts
    ([16, 512, 2048], [512, 256, 16], torch.float32, "nchw", "dense_tc_pair"),
    ([16, 512, 2048], [512, 256, 16], torch.float32, "nhwc", "dense_tc_pair"),
])
def test_kernel_selection(x_shape, w_shape, dtype, layout, kernel):
    """Automatic kernel choice for the shape classes each kernel was measured
    fastest on (pure host code: no device touched)."""
    got, ws, wb = _kernel_for(x_shape, w_shape, dtype, layout)
    assert got == kernel, (x_shape, w_shape, dtype, layout, got)
    assert wb > 0 and ws >= 0


def test_kernel_selection_workloads_and_one_by_one():
    """The kernel each workload is measured on (host planning only), and the
    1x1 rule: 1x1 stride-1 fp16 channels-first shapes whose output rows are a
    multiple of 8 wide plan to the halo kernel (row mode), other widths to the
    pair kernel."""
    want = {1: "generic", 2: "dense_tc_pair", 3: "dense_tc", 4: "dense_tc_pair", 5: "grouped"}
    for wid, kernel in want.items():
        wl = WORKLOADS[wid]
        case = dict(x_shape=wl.x_shape, w_shape=wl.w_shape, strides=wl.strides,
                    dilations=wl.dilations, pads=wl.pads, output_padding=wl.output_padding,
                    auto_pad=wl.auto_pad, group=wl.group, bias=wl.bias)
        plan = ct.ct_plan(_desc_from_case(case, dtype=wl.dtype))
        try:
            assert ct.ct_plan_kernel(plan) == kernel, (wid, ct.ct_plan_kernel(plan))
        finally:
            ct.ct_plan_destroy(plan)
    k, _, _ = _kernel_for([8, 512, 64, 64], [512, 256, 1, 1], torch.float16, strides=[1, 1])
    assert k == "dense_tc"
    k, _, _ = _kernel_for([4, 128, 20, 20], [128, 64, 1, 1], torch.float16, strides=[1, 1])
    assert k == "dense_tc_pair"
    # a 1x1 kernel with stride 2 is not a plain GEMM: the pair kernel
    k, _, _ = _kernel_for([8, 256, 32, 32], [256, 128, 1, 1], torch.float16, strides=[2, 2])
    assert k == "dense_tc_pair"


def test_pair_kernel_sizes():
    """Workspace and packed-weight sizes of the pair kernel: the padded
    channels-last copy (two planes for fp32) and one packed tile per
    256 output channels."""
    # 2-D decoder: 8 images x (64+2) x (64+2) padded positions x 256 channels x 2 bytes
    kern, ws, wb = _kernel_for([8, 256, 64, 64], [256, 128, 4, 4], torch.float16)
    assert kern == "dense_tc_pair" and ws == 8 * 66 * 66 * 256 * 2
    # the same with 512 output channels: two channel tiles of packed weights
    kern2, ws2, wb2 = _kernel_for([8, 256, 64, 64], [256, 256, 4, 4], torch.float16)
    kern3, ws3, wb3 = _kernel_for([8, 256, 64, 64], [256, 512, 4, 4], torch.float16)
    assert kern3 == "dense_tc_pair" and ws3 == ws2 and wb3 == 2 * wb2
    # fp32: high parts and remainders of X (2 planes of 4-byte elements) and of W
    kf, wsf, wbf = _kernel_for([8, 256, 64, 64], [256, 128, 4, 4], torch.float32)
    assert kf == "dense_tc_pair" and wsf == 2 * 2 * ws and wbf == 2 * 2 * wb
    # C = 3 is padded to an 8-channel (16-byte) row in the workspace
    kc, wsc, _ = _kernel_for([4, 3, 40, 48], [3, 64, 4, 4], torch.float16)
    assert kc == "dense_tc_pair" and wsc == 4 * 42 * 50 * 8 * 2


def test_general_shapes_plan_to_tensor_core_kernels():
    """Every shape ``bench.py --general`` times plans (host code only) to a
    tensor-core kernel: stride 1 with a 3x3 window and 1x1 (the tap-reversed
    stride-1 form and the plain GEMM), channels-last, more than 256 output
    channels, a 3-channel input and fp32."""
    import bench

    assert len(bench.GENERAL_SHAPES) >= 6
    for name, xs, ws, dt, layout, kw in bench.GENERAL_SHAPES:
        xsl = xs if layout == "nchw" else [xs[0]] + xs[2:] + [xs[1]]
        wsl = ws if layout == "nchw" else [ws[0]] + ws[2:] + [ws[1]]
        desc = ct.make_desc(xsl, wsl, dtype=dt, layout=layout, bias_len=ws[1], **kw)
        plan = ct.ct_plan(desc)
        try:
            kern = ct.ct_plan_kernel(plan)
            y_shape, _, _ = ct.ct_output_shape(desc)
        finally:
            ct.ct_plan_destroy(plan)
        assert kern in ("dense_tc_pair", "dense_tc"), (name, kern)
        # spatial sizes: stride 1 keeps them (3x3 with pad 1, 1x1), stride 2
        # with k = 4, p = 1 doubles them
        sp = y_shape[2:] if layout == "nchw" else y_shape[1:-1]
        mult = kw["strides"][0]
        assert list(sp) == [mult * v for v in xs[2:]], (name, y_shape)


def test_size_limits_reject_overflowing_descriptors():
    """Sizes whose arithmetic would overflow int64 are refused at resolve
    time (CT_ERR_ATTR = 4); sizes just inside the limits resolve."""
    big = 1 << 30

    def status(x_shape, w_shape, **kw):
        d = ct.make_desc(x_shape, w_shape, dtype=torch.float16, **kw)
        try:
            ct.ct_output_shape(d)
            return 0
        except ct.CtError as e:
            return e.status

    assert status([1, 1, big], [1, 1, 1], strides=[1]) == 0
    assert status([1, 1, big + 1], [1, 1, 1], strides=[1]) == 4
    assert status([1, 1, 4], [1, 1, 1], strides=[big + 1]) == 4
    assert status([1, 1, 4], [1, 1, 3], strides=[1], dilations=[1 << 40]) == 4
    assert status([1, 1, 4], [1, 1, 3], strides=[1], pads=[-(1 << 40), 0]) == 4
    assert status([1 << 31, 1, 4], [1, 1, 3], strides=[1]) == 4
    assert status([1, 1, 4], [1, 1 << 31, 3], strides=[1]) == 4
    # each size in range, but X has 2^30 * 2^30 * 2^30 elements
    assert status([big, big, big], [big, 1, 1], strides=[1]) == 4
    # Y too large: 2^20 images x 2^20 channels x 2^30 outputs
    assert status([1 << 20, 1, 1 << 29], [1, 1 << 20, 1], strides=[2], output_padding=[1]) == 4
    # the old overflow: s * (in - 1) near 2^62 now refused instead of wrapping
    assert status([1, 1, 1 << 31], [1, 1, 1], strides=[1 << 31]) == 4


def test_ignored_pads_are_not_range_checked():
    """With output_shape the explicit pads are ignored, whatever their size."""
    d = ct.make_desc([1, 1, 4], [1, 1, 3], dtype=torch.float16, strides=[2],
                     pads=[1 << 40, 0], output_shape=[9])
    y, pb, pe = ct.ct_output_shape(d)
    assert list(y) == [1, 1, 9] and (pb[0], pe[0]) == (0, 0)


def test_call_checks_refuse_mismatched_tensors():
    """The binding refuses X or Y that do not match the plan before any launch
    (host logic only; CPU tensors stand in for device ones)."""
    dev = torch.device("cpu")
    x = torch.zeros(2, 4, 5, dtype=torch.float16)
    y = torch.zeros(2, 6, 9, dtype=torch.float16)
    ct.check_io(x, None, [2, 4, 5], [2, 6, 9], torch.float16, dev)
    ct.check_io(x, y, [2, 4, 5], [2, 6, 9], torch.float16, dev)
    with pytest.raises(ValueError):
        ct.check_io(torch.zeros(2, 4, 6, dtype=torch.float16), None, [2, 4, 5], [2, 6, 9],
                    torch.float16, dev)
    with pytest.raises(ValueError):
        ct.check_io(x.float(), None, [2, 4, 5], [2, 6, 9], torch.float16, dev)
    with pytest.raises(ValueError):
        ct.check_io(x, torch.zeros(2, 6, 8, dtype=torch.float16), [2, 4, 5], [2, 6, 9],
                    torch.float16, dev)
    with pytest.raises(ValueError):
        ct.check_io(x, y.float(), [2, 4, 5], [2, 6, 9], torch.float16, dev)
    with pytest.raises(ValueError):
        ct.check_io(x, torch.zeros(2, 9, 6, dtype=torch.float16).transpose(1, 2), [2, 4, 5],
                    [2, 6, 9], torch.float16, dev)
    with pytest.raises(ValueError):
        ct.check_io(x, None, [2, 4, 5], [2, 6, 9], torch.float16, torch.device("meta"))


def test_take_device_error_without_device():
    """ct_take_device_error needs the device: without one it reports
    CT_ERR_DEVICE (7) with no wait code."""
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(ct.CtError) as e:
        ct.ct_take_device_error()
    assert e.value.status == 7
    code = ctypes.c_int32(-5)
    assert ct.lib().ct_take_device_error(None, ctypes.byref(code)) == 7 and code.value == 0
    assert ct.lib().ct_take_device_error(None, None) == 6          # CT_ERR_NULL


def test_binding_argument_counts_match_header():
    """Every function include/ct.h declares is bound with as many ctypes
    arguments as the declaration has parameters (guards binding drift)."""
    L = ct.lib()
    src = open(os.path.join(ROOT, "include", "ct.h")).read()
    decls = re.findall(r"CT_API\s+[\w\s\*]*?\b(ct_\w+)\s*\(([^)]*)\)", src)
    assert decls
    for name, params in decls:
        params = " ".join(params.split())
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert getattr(L, name).argtypes is not None, name
        assert len(getattr(L, name).argtypes) == n, (name, n, getattr(L, name).argtypes)
