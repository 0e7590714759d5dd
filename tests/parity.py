"""Shared helpers of the GPU parity tests: run a case through the C-ABI (via
the thin binding) and compare with the fp64 oracle element by element."""

import numpy as np
import torch

from oracle import Attrs, conv_transpose_points, conv_transpose_ref, to_channels_first
from transposed_convolution_02_b200 import ct
from transposed_convolution_02_b200.workloads import draw

# Acceptance: |y - ref| <= REL * sum|x*w| + ABS, elementwise.
TOL = {torch.float32: (1e-5, 1e-6), torch.float16: (4e-3, 1e-3)}


def attrs_from(case):
    return Attrs(strides=case["strides"], dilations=case.get("dilations"),
                 pads=case.get("pads"), output_padding=case.get("output_padding"),
                 auto_pad=case.get("auto_pad", "NOTSET"), group=case.get("group", 1),
                 kernel_shape=case.get("kernel_shape"), output_shape=case.get("output_shape"))


def draw_case(case, dtype, seed, layout="nchw"):
    """Seeded X, W, bias for a channels-first case; permuted when channels-last."""
    x = draw(case["x_shape"], ("normal", 1.0), seed, dtype)
    w = draw(case["w_shape"], ("normal", 0.5), seed + 1, dtype)
    m = case["w_shape"][1] * case.get("group", 1)
    b = draw([m], ("normal", 0.5), seed + 2, dtype) if case.get("bias") else None
    if layout == "nhwc":
        x = x.movedim(1, -1).contiguous()
        w = w.movedim(1, -1).contiguous()
    return x, w, b


def to_oracle(x, w, b, layout):
    xa = x.double().numpy()
    wa = w.double().numpy()
    if layout == "nhwc":
        xa, wa = to_channels_first(xa, wa)
    ba = b.double().numpy() if b is not None else None
    return xa, wa, ba


def gpu_run(case, x, w, b, layout, algo="auto", poison=True):
    op = ct.ConvTranspose(w.cuda(), list(x.shape), b.cuda() if b is not None else None,
                          layout=layout, strides=case["strides"],
                          dilations=case.get("dilations"), pads=case.get("pads"),
                          output_padding=case.get("output_padding"),
                          auto_pad=case.get("auto_pad", "NOTSET"), group=case.get("group", 1),
                          kernel_shape=case.get("kernel_shape"),
                          output_shape=case.get("output_shape"), algo=algo,
                          activation=case.get("activation", "identity"))
    y = torch.empty(op.y_shape, dtype=x.dtype, device="cuda")
    if poison:
        y.fill_(float("nan"))
    op(x.cuda(), out=y)
    torch.cuda.synchronize()
    return op, y


def check_close(y_gpu, ref, absacc, dtype, where=""):
    rel, ab = TOL[dtype]
    y = y_gpu.double().cpu().numpy() if isinstance(y_gpu, torch.Tensor) else y_gpu
    assert y.shape == ref.shape, (y.shape, ref.shape)
    bound = rel * absacc + ab
    err = np.abs(y - ref)
    bad = ~(err <= bound)          # NaN counts as bad
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError("%s: %d of %d outside tolerance; first %s: got %s want %s bound %s"
                             % (where, int(bad.sum()), bad.size, idx.tolist(),
                                y[tuple(idx.T)], ref[tuple(idx.T)], bound[tuple(idx.T)]))
    return float(np.max(err / bound)) if err.size else 0.0


def full_parity(case, dtype, seed, layout="nchw", algo="auto", expect_kernel=None):
    x, w, b = draw_case(case, dtype, seed, layout)
    op, y = gpu_run(case, x, w, b, layout, algo)
    if expect_kernel is not None:
        assert op.kernel == expect_kernel, (op.kernel, expect_kernel)
    xa, wa, ba = to_oracle(x, w, b, layout)
    ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case),
                                     activation=case.get("activation", "identity"))
    if layout == "nhwc":
        ref = np.moveaxis(ref, 1, -1)
        absacc = np.moveaxis(absacc, 1, -1)
    return op, check_close(y, ref, absacc, dtype, "%s %s %s" % (case, layout, op.kernel))


def sampled_points(y_shape_cf, rng, n_random=1500):
    """Output points (n, m, o..) in channels-first coordinates: corners and
    edges of every axis, every residue of small strides, plus random ones."""
    pts = set()
    dims = list(y_shape_cf)
    r = len(dims) - 2
    for _ in range(n_random):
        pts.add(tuple(int(rng.integers(0, d)) for d in dims))
    for n in {0, dims[0] - 1}:
        for m in {0, dims[1] - 1, dims[1] // 2}:
            for a in range(r):
                for v in {0, 1, 2, 3, dims[2 + a] - 1, dims[2 + a] - 2, dims[2 + a] - 3}:
                    if 0 <= v < dims[2 + a]:
                        p = [n, m] + [int(rng.integers(0, dims[2 + b])) for b in range(r)]
                        p[2 + a] = v
                        pts.add(tuple(p))
    return np.array(sorted(pts), dtype=np.int64)


def stratified_points(y_shape_cf, strides, rng, chunk=16, mblock=32):
    """Output points (n, m, o..) in channels-first coordinates that reach every
    piece of work a kernel can own.  For every image n, every stride phase r
    (o mod s per axis), every block of `mblock` output channels and every run
    of `chunk` consecutive positions J of the phase (J numbered with the last
    axis fastest), one random point; plus the first and the last J of every
    row of every phase (row ends and tile edges).  A unit, CTA, warp or lane
    group that owns at least `chunk` consecutive positions of a phase row, or
    whole rows, for one block of channels therefore gets a point."""
    dims = [int(d) for d in y_shape_cf]
    n_img, m_all, out = dims[0], dims[1], dims[2:]
    r = len(out)
    s = [int(v) for v in strides]
    pts = []
    for ph in np.ndindex(*s):
        nj = [(out[a] - ph[a] + s[a] - 1) // s[a] if out[a] > ph[a] else 0 for a in range(r)]
        total = int(np.prod(nj))
        if total == 0:
            continue
        starts = np.arange(0, total, chunk)
        width = np.minimum(chunk, total - starts)
        mstarts = np.arange(0, m_all, mblock)
        mwidth = np.minimum(mblock, m_all - mstarts)
        for n in range(n_img):
            t = starts[:, None] + (rng.random((len(starts), len(mstarts))) * width[:, None]).astype(np.int64)
            m = mstarts[None, :] + (rng.random((len(starts), len(mstarts))) * mwidth[None, :]).astype(np.int64)
            t, m = t.reshape(-1), m.reshape(-1)
            J = np.stack(np.unravel_index(t, nj), axis=1)
            o = J * np.array(s)[None, :] + np.array(ph)[None, :]
            pts.append(np.concatenate([np.full((len(t), 1), n), m[:, None], o], axis=1))
            # both ends of every row of the phase
            rows = int(np.prod(nj[:-1]))
            for jx in {0, nj[-1] - 1}:
                rj = np.stack(np.unravel_index(np.arange(rows), nj[:-1]), axis=1) if r > 1 else \
                    np.zeros((1, 0), dtype=np.int64)
                J = np.concatenate([rj, np.full((rows, 1), jx)], axis=1)
                o = J * np.array(s)[None, :] + np.array(ph)[None, :]
                m = rng.integers(0, m_all, rows)
                pts.append(np.concatenate([np.full((rows, 1), n), m[:, None], o], axis=1))
    allp = np.concatenate(pts, axis=0).astype(np.int64)
    return np.unique(allp, axis=0)


def check_points(op, y, x, w, b, case, dtype, layout, pts, where):
    """Compare the GPU output at `pts` (channels-first coordinates) with the
    oracle evaluated at those points one by one."""
    xa, wa, ba = to_oracle(x, w, b, layout)
    ycf = y if layout == "nchw" else y.movedim(-1, 1)
    ref, absacc = conv_transpose_points(xa, wa, ba, attrs_from(case), pts,
                                        activation=case.get("activation", "identity"))
    got = ycf[tuple(torch.from_numpy(pts.T).to(y.device))].double().cpu().numpy()
    return check_close(got, ref, absacc, dtype, where)


def sampled_parity(op, y, x, w, b, case, dtype, layout, rng, n_random=1500):
    """Compare the full GPU output with oracle points one by one."""
    xa, wa, ba = to_oracle(x, w, b, layout)
    ycf = y if layout == "nchw" else y.movedim(-1, 1)
    pts = sampled_points(list(ycf.shape), rng, n_random)
    ref, absacc = conv_transpose_points(xa, wa, ba, attrs_from(case), pts,
                                        activation=case.get("activation", "identity"))
    got = ycf[tuple(torch.from_numpy(pts.T).to(y.device))].double().cpu().numpy()
    return check_close(got, ref, absacc, dtype, "sampled " + str(case))
