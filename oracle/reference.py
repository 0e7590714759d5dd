"""fp64 CPU oracle for ONNX ConvTranspose (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg
may import this module.  The CUDA product path never imports it, and it
imports nothing from the product package.

* ``conv_transpose_ref``   -- the scatter definition over whole tensors
  (ai.onnx.ConvTranspose README, "Description"; the C loop in ct_oracle.c).
* ``conv_transpose_points`` -- the same definition evaluated at chosen output
  points, for outputs too large to scatter in full.
* ``forward_conv_ref``     -- a plain gather forward convolution, used only to
  state the stride-1 and adjoint identities the transposed convolution obeys.
* ``to_channels_first``    -- reorders the channels-last call of
  ClikaRT::ops::conv_transpose (input [N, D.., C_in], weight
  [C_in, K.., O/groups]) into the channels-first tensors the oracle takes.

Inputs are the exact values the device receives (fp16 or fp32), widened to
fp64.  Pads and sizes come from ``oracle.resolver``.
"""

import ctypes
import os
import subprocess

import numpy as np

from .resolver import Attrs, resolve_full

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ct_oracle.c")
_LIB = os.path.join(_HERE, "libct_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ct_oracle.c into a shared library beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64p = ctypes.POINTER(ctypes.c_int64)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.ct_oracle_conv_transpose.restype = ctypes.c_int
        lib.ct_oracle_conv_transpose.argtypes = (
            [ctypes.c_int] + [ctypes.c_int64] * 4 + [i64p] * 6 + [dp] * 5)
        lib.ct_oracle_points.restype = ctypes.c_int
        lib.ct_oracle_points.argtypes = (
            [ctypes.c_int] + [ctypes.c_int64] * 4 + [i64p] * 6 + [dp] * 3
            + [i64p, ctypes.c_int64, dp, dp])
        _lib = lib
    return _lib


def _i64(v):
    a = np.ascontiguousarray(np.asarray(v, dtype=np.int64))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _f64(v):
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _geometry(x, w, bias, attrs):
    x = np.asarray(x)
    w = np.asarray(w)
    yshape, res = resolve_full(list(x.shape), list(w.shape), attrs,
                               None if bias is None else int(np.asarray(bias).size))
    rank = x.ndim - 2
    s = list(attrs.strides) if attrs.strides is not None else [1] * rank
    d = list(attrs.dilations) if attrs.dilations is not None else [1] * rank
    return yshape, res, rank, s, d


ACTIVATIONS = ("identity", "relu")


def apply_activation(y, activation="identity"):
    """The output activation of ClikaRT::ops::conv_transpose (parameter
    `activation`, default Identity), applied to the output after the bias.
    The page names the parameter but not the members of its enum; the two
    read here are identity and ReLU, max(y, 0)."""
    if activation == "identity":
        return y
    if activation == "relu":
        return np.maximum(y, 0.0)
    raise ValueError("unknown activation %r" % (activation,))


def conv_transpose_ref(x, w, bias=None, attrs: Attrs = None, activation="identity"):
    """Return (Y, A) in fp64: Y per the scatter definition (then the
    activation), A = sum |x*w|."""
    attrs = attrs or Attrs(strides=None)
    yshape, res, rank, s, d = _geometry(x, w, bias, attrs)
    N, C = x.shape[0], x.shape[1]
    M = yshape[1]
    lib = _load()
    keep = []
    args = []
    for v in (x.shape[2:], w.shape[2:], s, d, res.pad_begin, res.out):
        a, p = _i64(list(v))
        keep.append(a)
        args.append(p)
    xa, xp = _f64(x)
    wa, wp = _f64(w)
    if bias is not None:
        ba, bp = _f64(bias)
    else:
        ba, bp = None, None
    y = np.zeros(yshape, dtype=np.float64)
    a = np.zeros(yshape, dtype=np.float64)
    rc = lib.ct_oracle_conv_transpose(
        rank, N, C, M, attrs.group, *args, xp, wp, bp,
        y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise RuntimeError("oracle rejected the geometry (code %d)" % rc)
    return apply_activation(y, activation), a


def conv_transpose_points(x, w, bias, attrs: Attrs, points, activation="identity"):
    """Evaluate Y and A at output points (rows of n, m, o_1..o_r)."""
    yshape, res, rank, s, d = _geometry(x, w, bias, attrs)
    N, C = x.shape[0], x.shape[1]
    M = yshape[1]
    lib = _load()
    keep = []
    args = []
    for v in (x.shape[2:], w.shape[2:], s, d, res.pad_begin, res.out):
        a, p = _i64(list(v))
        keep.append(a)
        args.append(p)
    xa, xp = _f64(x)
    wa, wp = _f64(w)
    if bias is not None:
        ba, bp = _f64(bias)
    else:
        ba, bp = None, None
    pts = np.ascontiguousarray(np.asarray(points, dtype=np.int64).reshape(-1, 2 + rank))
    yv = np.zeros(len(pts), dtype=np.float64)
    av = np.zeros(len(pts), dtype=np.float64)
    rc = lib.ct_oracle_points(
        rank, N, C, M, attrs.group, *args, xp, wp, bp,
        pts.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(pts),
        yv.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        av.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise RuntimeError("oracle rejected the points (code %d)" % rc)
    return apply_activation(yv, activation), av


def forward_conv_ref(u, wf, strides, dilations, pad_begin, out_spatial, group):
    """Plain gather forward convolution (fp64), only for the identities.

    u[N, Cin, D..] and the weight wf[Cout, Cin/group, k..] give
    out[n, co, j] = sum_{ci, k} wf[co, ci, k] * u[n, g*Cin/g + ci, j*s - pb + k*d]
    with zeros outside u, for every j in the requested output box.
    """
    u = np.asarray(u, dtype=np.float64)
    wf = np.asarray(wf, dtype=np.float64)
    N, Cin = u.shape[:2]
    Cout = wf.shape[0]
    rank = u.ndim - 2
    Cig, Cog = Cin // group, Cout // group
    out = np.zeros([N, Cout] + list(out_spatial), dtype=np.float64)
    ksz = wf.shape[2:]
    for co in range(Cout):
        g = co // Cog
        for ci in range(Cig):
            c = g * Cig + ci
            for kidx in np.ndindex(*ksz):
                wv = wf[(co, ci) + kidx]
                for j in np.ndindex(*out_spatial):
                    src = [j[a] * strides[a] - pad_begin[a] + kidx[a] * dilations[a]
                           for a in range(rank)]
                    if all(0 <= src[a] < u.shape[2 + a] for a in range(rank)):
                        out[(slice(None), co) + j] += wv * u[(slice(None), c) + tuple(src)]
    return out


def to_channels_first(x_cl, w_cl):
    """Channels-last input [N, D.., C] and weight [C_in, K.., O/g] to the
    channels-first X[N, C, D..] and W[C, O/g, K..] of the same call."""
    x_cl = np.asarray(x_cl)
    w_cl = np.asarray(w_cl)
    r = x_cl.ndim - 2
    x = np.moveaxis(x_cl, -1, 1)
    w = np.moveaxis(w_cl, -1, 1)
    assert x.ndim == r + 2 and w.ndim == r + 2
    return np.ascontiguousarray(x), np.ascontiguousarray(w)
