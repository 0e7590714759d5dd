"""Seeded synthetic inputs for the ConvTranspose workloads.

This module only draws random tensors and states the workloads' attributes;
it holds none of the operator's arithmetic.  Tests, the benchmark and the
oracle-side checks all take their inputs from here.

Recipe: a CPU ``torch.Generator`` seeded with ``1000 * workload_id + j``
(j = 0 for X, 1 for W, 2 for the bias) draws fp32 values, which are then
rounded to the workload's dtype.  ``normal(std)`` means N(0, std^2);
``uniform(lo, hi)`` is U[lo, hi).
"""

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch


@dataclass
class Workload:
    wid: int
    name: str
    dtype: torch.dtype
    x_shape: Sequence[int]
    w_shape: Sequence[int]
    bias: bool
    strides: Sequence[int]
    pads: Optional[Sequence[int]] = None
    dilations: Optional[Sequence[int]] = None
    output_padding: Optional[Sequence[int]] = None
    auto_pad: str = "NOTSET"
    group: int = 1
    y_shape: Sequence[int] = field(default_factory=list)   # as stated by the workload
    x_dist: tuple = ("normal", 1.0)
    w_dist: tuple = ("normal", 1.0)
    b_dist: tuple = ("normal", 0.1)


WORKLOADS = {
    1: Workload(1, "2-D fp32 NCHW X[1,8,8,8] W[8,4,3,3] s2 p1 op1", torch.float32,
                [1, 8, 8, 8], [8, 4, 3, 3], True, [2, 2], pads=[1, 1, 1, 1],
                output_padding=[1, 1], y_shape=[1, 4, 16, 16],
                x_dist=("uniform", -1.0, 1.0), w_dist=("uniform", -1.0, 1.0),
                b_dist=("uniform", -1.0, 1.0)),
    2: Workload(2, "2-D decoder upsample fp16 X[8,256,64,64] W[256,128,4,4] s2 p1",
                torch.float16, [8, 256, 64, 64], [256, 128, 4, 4], True, [2, 2],
                pads=[1, 1, 1, 1], y_shape=[8, 128, 128, 128],
                w_dist=("normal", 1.0 / math.sqrt(256 * 4))),
    3: Workload(3, "3-D volumetric upsample fp16 X[2,64,32,32,32] W[64,32,3,3,3] s2 p1 op1",
                torch.float16, [2, 64, 32, 32, 32], [64, 32, 3, 3, 3], False, [2, 2, 2],
                pads=[1, 1, 1, 1, 1, 1], output_padding=[1, 1, 1],
                y_shape=[2, 32, 64, 64, 64],
                w_dist=("normal", 1.0 / math.sqrt(64 * 27 / 8))),
    4: Workload(4, "1-D vocoder upsample fp32 X[16,512,2048] W[512,256,16] s8 p4",
                torch.float32, [16, 512, 2048], [512, 256, 16], True, [8],
                pads=[4, 4], y_shape=[16, 256, 16384],
                w_dist=("normal", 1.0 / math.sqrt(512 * 2))),
    5: Workload(5, "2-D grouped+dilated fp16 X[16,512,56,56] W[512,16,3,3] g32 s2 d2 SAME_UPPER",
                torch.float16, [16, 512, 56, 56], [512, 16, 3, 3], True, [2, 2],
                dilations=[2, 2], auto_pad="SAME_UPPER", group=32,
                y_shape=[16, 512, 112, 112],
                w_dist=("normal", 1.0 / math.sqrt(16 * 9 / 4))),
}


def draw(shape, dist, seed, dtype):
    """Draw one tensor of ``shape`` from ``dist`` with a seeded CPU generator."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    if dist[0] == "normal":
        t = torch.randn(list(shape), generator=g, dtype=torch.float32) * float(dist[1])
    elif dist[0] == "uniform":
        lo, hi = float(dist[1]), float(dist[2])
        t = torch.rand(list(shape), generator=g, dtype=torch.float32) * (hi - lo) + lo
    else:
        raise ValueError("unknown distribution %r" % (dist,))
    return t.to(dtype)


def make_inputs(wl: Workload, m_out: Optional[int] = None):
    """X, W and bias (or None) of a workload, as CPU tensors in its dtype.

    ``m_out`` is the bias length (output channels); it defaults to
    W's second dim times the group count, which is how the workload states it.
    """
    x = draw(wl.x_shape, wl.x_dist, 1000 * wl.wid + 0, wl.dtype)
    w = draw(wl.w_shape, wl.w_dist, 1000 * wl.wid + 1, wl.dtype)
    b = None
    if wl.bias:
        m = m_out if m_out is not None else wl.w_shape[1] * wl.group
        b = draw([m], wl.b_dist, 1000 * wl.wid + 2, wl.dtype)
    return x, w, b
