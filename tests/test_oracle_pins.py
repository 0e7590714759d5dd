"""CPU pins of the fp64 oracle: each check ties it to something other than
itself (hand-worked values, closed-form shapes, identities, a library special
case, invariants), so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import golden_io
from cases import attrs_of, random_case
from oracle import (Attrs, ResolveError, conv_transpose_points, conv_transpose_ref,
                    forward_conv_ref, resolve, resolve_full, to_channels_first)
from transposed_convolution_02_b200.workloads import WORKLOADS


def _attrs_from_fixture(rec):
    return Attrs(strides=rec.get("strides"), dilations=rec.get("dilations"),
                 pads=rec.get("pads"), output_padding=rec.get("output_padding"),
                 auto_pad=rec["auto_pad"], group=rec["group"],
                 kernel_shape=rec.get("kernel_shape"), output_shape=rec.get("output_shape"))


@pytest.mark.parametrize("path", golden_io.all_fixtures(),
                         ids=lambda p: p.rsplit("/", 1)[-1][:-4])
def test_golden_fixture(path):
    rec = golden_io.load(path)
    attrs = _attrs_from_fixture(rec)
    x, w = rec["x"], rec["w"]
    if rec["layout"] == "nhwc":
        x, w = to_channels_first(x, w)
    y, a = conv_transpose_ref(x, w, rec["bias"], attrs)
    if rec["layout"] == "nhwc":
        y = np.moveaxis(y, 1, -1)
    assert list(y.shape) == rec["y_shape"]
    np.testing.assert_allclose(y, rec["y"], rtol=0, atol=1e-12)


def test_readme_usage_example_shape():
    # ai.onnx.ConvTranspose README, JavaScript usage: x [1,1,3], w [1,2,2],
    # attributes at their defaults -> y has rank 3, M = 2, length 3 + 2 - 1.
    yshape, res = resolve_full([1, 1, 3], [1, 2, 2], Attrs(strides=None))
    assert yshape == [1, 2, 4]
    assert res.pad_begin == [0] and res.pad_end == [0]


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_workload_output_shapes(wid):
    wl = WORKLOADS[wid]
    attrs = Attrs(strides=wl.strides, dilations=wl.dilations, pads=wl.pads,
                  output_padding=wl.output_padding, auto_pad=wl.auto_pad, group=wl.group)
    yshape, _ = resolve_full(wl.x_shape, wl.w_shape, attrs,
                             wl.w_shape[1] * wl.group if wl.bias else None)
    assert yshape == list(wl.y_shape)


def test_same_upper_split_of_grouped_dilated_workload():
    # SAME_UPPER: out = in*stride; total = 2*55 + 0 + 4 + 1 - 112 = 3, the odd
    # unit at the end.
    res = resolve([56, 56], [3, 3], Attrs(strides=[2, 2], dilations=[2, 2],
                                          auto_pad="SAME_UPPER", group=32))
    assert res.out == [112, 112]
    assert res.pad_begin == [1, 1] and res.pad_end == [2, 2]


@pytest.mark.parametrize("mode", ["SAME_UPPER", "SAME_LOWER"])
def test_same_gives_in_times_stride(mode):
    rng = np.random.default_rng(7)
    for _ in range(300):
        r = int(rng.integers(1, 4))
        ins = [int(rng.integers(1, 30)) for _ in range(r)]
        ks = [int(rng.integers(1, 7)) for _ in range(r)]
        ss = [int(rng.integers(1, 5)) for _ in range(r)]
        ds = [int(rng.integers(1, 4)) for _ in range(r)]
        ops = [int(rng.integers(0, max(ss[a], ds[a]))) for a in range(r)]
        res = resolve(ins, ks, Attrs(strides=ss, dilations=ds, output_padding=ops,
                                     auto_pad=mode))
        assert res.out == [ins[a] * ss[a] for a in range(r)]
        for a in range(r):
            diff = res.pad_end[a] - res.pad_begin[a]
            assert diff in (0, 1, -1)
            total = res.pad_begin[a] + res.pad_end[a]
            if total % 2:
                # the odd unit (with its sign) at the stated end
                odd_end = (res.pad_end[a] - res.pad_begin[a]) == (1 if total > 0 else -1)
                assert odd_end == (mode == "SAME_UPPER")


def test_resolver_error_classes():
    ok = Attrs(strides=[2], pads=[1, 1], output_padding=[1])
    resolve([4], [3], ok)
    with pytest.raises(ResolveError):   # output_padding must be below max(stride, dilation)
        resolve([4], [3], Attrs(strides=[2], output_padding=[2]))
    resolve([4], [3], Attrs(strides=[1], dilations=[3], output_padding=[2]))
    with pytest.raises(ResolveError):   # kernel_shape must match W
        resolve([4], [3], Attrs(strides=[1], kernel_shape=[2]))
    with pytest.raises(ResolveError):   # pads with auto_pad
        resolve([4], [3], Attrs(strides=[1], pads=[1, 0], auto_pad="SAME_UPPER"))
    with pytest.raises(ResolveError):   # span length
        resolve([4, 4], [3, 3], Attrs(strides=[1]))
    with pytest.raises(ResolveError):   # non-positive stride
        resolve([4], [3], Attrs(strides=[0]))
    with pytest.raises(ResolveError):   # empty output
        resolve([1], [1], Attrs(strides=[1], pads=[1, 0]))
    with pytest.raises(ResolveError):   # channels
        resolve_full([1, 3, 4], [3, 2, 3], Attrs(strides=[1], group=2))
    with pytest.raises(ResolveError):   # bias length
        resolve_full([1, 4, 4], [4, 2, 3], Attrs(strides=[1], group=2), bias_len=3)
    with pytest.raises(ResolveError):   # W[0] must equal C
        resolve_full([1, 4, 4], [2, 2, 3], Attrs(strides=[1]))


def _torch_special_case(x, w, bias, attrs):
    """Library special case: PyTorch's CPU fp64 conv_transpose with no pads
    and no output_padding is the full scatter; slicing it by the begin pad
    and zero-extending to the resolved size gives the padded result."""
    rank = x.ndim - 2
    yshape, res = resolve_full(list(x.shape), list(w.shape), attrs,
                               None if bias is None else len(bias))
    fn = {1: F.conv_transpose1d, 2: F.conv_transpose2d, 3: F.conv_transpose3d}[rank]
    s = attrs.strides or [1] * rank
    d = attrs.dilations or [1] * rank
    full = fn(torch.from_numpy(x), torch.from_numpy(w), None, stride=tuple(s), padding=0,
              output_padding=0, groups=attrs.group, dilation=tuple(d)).numpy()
    y = np.zeros(yshape)
    dst, src = [slice(None), slice(None)], [slice(None), slice(None)]
    for a in range(rank):
        pb = res.pad_begin[a]
        lo = max(0, -pb)
        hi = min(res.out[a], full.shape[2 + a] - pb)
        if hi <= lo:
            dst.append(slice(0, 0))
            src.append(slice(0, 0))
        else:
            dst.append(slice(lo, hi))
            src.append(slice(lo + pb, hi + pb))
    y[tuple(dst)] = full[tuple(src)]
    if bias is not None:
        y += bias.reshape([1, -1] + [1] * rank)
    return y


def test_against_torch_library_sweep():
    rng = np.random.default_rng(1234)
    for _ in range(120):
        case = random_case(rng)
        attrs = attrs_of(case)
        x = rng.standard_normal(case["x_shape"])
        w = rng.standard_normal(case["w_shape"])
        b = rng.standard_normal(case["w_shape"][1] * case["group"]) if case["bias"] else None
        y, a = conv_transpose_ref(x, w, b, attrs)
        ref = _torch_special_case(x, w, b, attrs)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12, err_msg=str(case))


def test_relu_activation_against_torch_library():
    # ClikaRT::ops::conv_transpose, parameter `activation`: ReLU after the
    # bias.  Pinned to torch.relu applied to the library special case, and to
    # the bias-only positions of a stride-2 dilation-2 shape (ReLU of the bias).
    rng = np.random.default_rng(77)
    for _ in range(30):
        case = random_case(rng)
        attrs = attrs_of(case)
        x = rng.standard_normal(case["x_shape"])
        w = rng.standard_normal(case["w_shape"])
        b = rng.standard_normal(case["w_shape"][1] * case["group"]) if case["bias"] else None
        y, a = conv_transpose_ref(x, w, b, attrs, activation="relu")
        ref = torch.relu(torch.from_numpy(_torch_special_case(x, w, b, attrs))).numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12, err_msg=str(case))
        _, a_id = conv_transpose_ref(x, w, b, attrs)
        np.testing.assert_array_equal(a, a_id)     # the accumulator is the identity's
    x = rng.standard_normal([1, 2, 5, 5])
    w = rng.standard_normal([2, 3, 3, 3])
    b = np.array([-0.5, 0.0, 0.75])
    attrs = Attrs(strides=[2, 2], dilations=[2, 2], auto_pad="SAME_UPPER")
    y, _ = conv_transpose_ref(x, w, b, attrs, activation="relu")
    assert np.all(y[:, :, 0::2, :] == np.maximum(b, 0).reshape(1, 3, 1, 1))
    with pytest.raises(ValueError):
        conv_transpose_ref(x, w, b, attrs, activation="gelu")


def test_against_torch_library_workload_1():
    from transposed_convolution_02_b200.workloads import make_inputs
    wl = WORKLOADS[1]
    x, w, b = [t.double().numpy() for t in make_inputs(wl)]
    attrs = Attrs(strides=wl.strides, pads=wl.pads, output_padding=wl.output_padding)
    y, _ = conv_transpose_ref(x, w, b, attrs)
    np.testing.assert_allclose(y, _torch_special_case(x, w, b, attrs), rtol=1e-12, atol=1e-12)


def test_stride1_identity_with_tap_reversed_forward_conv():
    # ai.onnx.ConvTranspose README, ncdhw3d_implicit_sgmat: at stride 1 the
    # transposed convolution is a forward convolution of the unchanged input
    # with tap-reversed weights and begin pads of (k-1)*d - pad.
    rng = np.random.default_rng(5)
    for _ in range(25):
        case = random_case(rng, strides=(1, 2), max_cg=2, max_mg=2)
        case["output_padding"] = [0] * len(case["strides"])
        attrs = attrs_of(case)
        try:
            resolve_full(case["x_shape"], case["w_shape"], attrs)
        except ResolveError:
            continue
        x = rng.standard_normal(case["x_shape"])
        w = rng.standard_normal(case["w_shape"])
        y, _ = conv_transpose_ref(x, w, None, attrs)
        rank = x.ndim - 2
        g = case["group"]
        C, Mg = w.shape[0], w.shape[1]
        Cg = C // g
        flip = tuple(slice(None, None, -1) for _ in range(rank))
        wf = np.zeros([Mg * g, Cg] + list(w.shape[2:]))
        for gi in range(g):
            for ml in range(Mg):
                for cl in range(Cg):
                    wf[(gi * Mg + ml, cl)] = w[(gi * Cg + cl, ml) + flip]
        res = resolve(list(x.shape[2:]), list(w.shape[2:]), attrs)
        fpb = [(w.shape[2 + a] - 1) * case["dilations"][a] - res.pad_begin[a]
               for a in range(rank)]
        yf = forward_conv_ref(x, wf, [1] * rank, case["dilations"], fpb, res.out, g)
        np.testing.assert_allclose(y, yf, rtol=1e-12, atol=1e-12, err_msg=str(case))


def test_adjoint_identity():
    # <conv(u, W), x> = <u, convT(x, W)> with the forward conv using the same
    # W as its [C_out = C, C_in/group = M/group, k..] weight, the same stride,
    # dilation, group and begin pad, and output size = the input size.
    rng = np.random.default_rng(11)
    for _ in range(25):
        case = random_case(rng, max_cg=2, max_mg=2)
        rank = len(case["strides"])
        case["output_padding"] = [int(rng.integers(0, case["strides"][a])) for a in range(rank)]
        attrs = attrs_of(case)
        try:
            resolve_full(case["x_shape"], case["w_shape"], attrs)
        except ResolveError:
            continue
        x = rng.standard_normal(case["x_shape"])
        w = rng.standard_normal(case["w_shape"])
        y, _ = conv_transpose_ref(x, w, None, attrs)
        u = rng.standard_normal(y.shape)
        res = resolve(list(x.shape[2:]), list(w.shape[2:]), attrs)
        cu = forward_conv_ref(u, w, case["strides"], case["dilations"], res.pad_begin,
                              list(x.shape[2:]), case["group"])
        lhs = float(np.sum(cu * x))
        rhs = float(np.sum(u * y))
        assert abs(lhs - rhs) <= 1e-10 * (1 + abs(lhs)), (case, lhs, rhs)


def test_1x1_stride1_is_a_matmul():
    # the 1x1 kernels of the README (conv-1x1-gemm-*): per group,
    # Y[n, g*Mg + ml, p] = sum_c W[g*Cg + c, ml] * X[n, g*Cg + c, p].
    rng = np.random.default_rng(3)
    for g, Cg, Mg, sp in [(1, 5, 3, [7]), (2, 3, 4, [4, 5]), (4, 2, 2, [2, 3, 3])]:
        x = rng.standard_normal([2, g * Cg] + sp)
        w = rng.standard_normal([g * Cg, Mg] + [1] * len(sp))
        y, _ = conv_transpose_ref(x, w, None, Attrs(strides=[1] * len(sp), group=g))
        for gi in range(g):
            xg = x[:, gi * Cg:(gi + 1) * Cg].reshape(2, Cg, -1)
            wg = w[gi * Cg:(gi + 1) * Cg].reshape(Cg, Mg)
            ref = np.einsum("cm,ncp->nmp", wg, xg)
            np.testing.assert_allclose(y[:, gi * Mg:(gi + 1) * Mg].reshape(2, Mg, -1), ref,
                                       rtol=1e-12, atol=1e-12)


def test_linearity_and_group_independence():
    rng = np.random.default_rng(17)
    case = dict(x_shape=[2, 8, 5, 4], w_shape=[8, 3, 3, 2], strides=[2, 3], dilations=[1, 2],
                pads=[1, 0, 0, 2], output_padding=[1, 0], group=4)
    attrs = attrs_of(case)
    x1 = rng.standard_normal(case["x_shape"])
    x2 = rng.standard_normal(case["x_shape"])
    w1 = rng.standard_normal(case["w_shape"])
    w2 = rng.standard_normal(case["w_shape"])
    ya, _ = conv_transpose_ref(2 * x1 - 3 * x2, w1, None, attrs)
    yb = 2 * conv_transpose_ref(x1, w1, None, attrs)[0] - 3 * conv_transpose_ref(x2, w1, None, attrs)[0]
    np.testing.assert_allclose(ya, yb, rtol=1e-11, atol=1e-11)
    yc, _ = conv_transpose_ref(x1, w1 + w2, None, attrs)
    yd = conv_transpose_ref(x1, w1, None, attrs)[0] + conv_transpose_ref(x1, w2, None, attrs)[0]
    np.testing.assert_allclose(yc, yd, rtol=1e-11, atol=1e-11)
    # zeroing group 1's input channels changes only group 1's outputs
    x3 = x1.copy()
    x3[:, 2:4] = 0
    y1, _ = conv_transpose_ref(x1, w1, None, attrs)
    y3, _ = conv_transpose_ref(x3, w1, None, attrs)
    changed = np.any(np.abs(y1 - y3) > 0, axis=(0, 2, 3))
    assert list(np.nonzero(changed)[0]) == [3, 4, 5]


def test_bias_only_positions_are_exact():
    # stride 2, dilation 2, SAME_UPPER (the grouped workload's geometry): only
    # odd output positions on each axis receive taps; every other output is
    # exactly the bias.
    rng = np.random.default_rng(2)
    x = rng.standard_normal([1, 4, 5, 6])
    w = rng.standard_normal([4, 2, 3, 3])
    b = rng.standard_normal(4)
    y, a = conv_transpose_ref(x, w, b, Attrs(strides=[2, 2], dilations=[2, 2],
                                              auto_pad="SAME_UPPER", group=2))
    assert y.shape == (1, 4, 10, 12)
    for m in range(4):
        plane = y[0, m]
        assert np.all(plane[0::2, :] == b[m])
        assert np.all(plane[:, 0::2] == b[m])
        assert np.all(a[0, m][0::2, :] == 0)
        assert np.all(np.abs(plane[1::2, 1::2] - b[m]) > 0)


def test_abs_accumulator():
    rng = np.random.default_rng(23)
    case = random_case(rng)
    attrs = attrs_of(case)
    x = np.abs(rng.standard_normal(case["x_shape"]))
    w = np.abs(rng.standard_normal(case["w_shape"]))
    y, a = conv_transpose_ref(x, w, None, attrs)
    np.testing.assert_allclose(a, y, rtol=1e-12, atol=1e-12)
    y2, a2 = conv_transpose_ref(-x, w, None, attrs)
    np.testing.assert_allclose(a2, a, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y2, -y, rtol=1e-12, atol=1e-12)


def test_points_agree_with_full_scatter():
    rng = np.random.default_rng(29)
    for _ in range(20):
        case = random_case(rng)
        attrs = attrs_of(case)
        x = rng.standard_normal(case["x_shape"])
        w = rng.standard_normal(case["w_shape"])
        b = rng.standard_normal(case["w_shape"][1] * case["group"]) if case["bias"] else None
        y, a = conv_transpose_ref(x, w, b, attrs)
        idx = np.array(list(np.ndindex(*y.shape)))
        pick = idx[rng.choice(len(idx), size=min(40, len(idx)), replace=False)]
        yv, av = conv_transpose_points(x, w, b, attrs, pick)
        np.testing.assert_allclose(yv, y[tuple(pick.T)], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(av, a[tuple(pick.T)], rtol=1e-12, atol=1e-12)


def test_empty_channels_give_bias():
    # C = 0: no term reaches any output, so Y is the bias.
    x = np.zeros([2, 0, 3])
    w = np.zeros([0, 3, 2])
    b = np.array([1.0, -2.0, 0.5])
    y, a = conv_transpose_ref(x, w, b, Attrs(strides=[2]))
    assert y.shape == (2, 3, 6)
    assert np.all(y == b.reshape(1, 3, 1)) and np.all(a == 0)
