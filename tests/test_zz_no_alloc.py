"""ct_run_noalloc against ct_run, on the GPU.

ct_run_noalloc serves callers that must not allocate device memory while
they run, for example a plugin inside an inference engine that owns all of
the device's memory and hands out only its own buffers.  Such a caller
still passes X, the packed weight, the bias and Y; the workspace comes from
a fixed array inside libct.so instead of from the caller.

Here a plan that needs a workspace (fp16 channels-first on the tensor-core
path, whose input is re-laid channels-last into it) runs twice in a row, on
two different inputs.  Each result must equal, bit for bit, what ct_run
gives with a torch-allocated workspace (the same kernels on the same
inputs), hence also lie within the fp16 parity tolerance of the oracle.  The
second call must not change the device's free memory.

This file sorts last so that a run that stops at the first failure has
already run every other test; it also passes when run alone.
"""

import numpy as np
import pytest
import torch

from parity import TOL, attrs_from, to_oracle
from oracle import conv_transpose_ref
from transposed_convolution_02_b200 import ct
from transposed_convolution_02_b200.workloads import draw

pytestmark = pytest.mark.gpu


def test_run_noalloc_matches_run_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    case = dict(x_shape=[2, 64, 20, 24], w_shape=[64, 48, 4, 4], strides=[2, 2],
                pads=[1, 1, 1, 1], bias=True)
    w = draw(case["w_shape"], ("normal", 0.125), 501, torch.float16)
    b = draw([48], ("normal", 0.1), 502, torch.float16)
    op = ct.ConvTranspose(w.cuda(), case["x_shape"], b.cuda(), strides=case["strides"],
                          pads=case["pads"])
    assert ct.ct_workspace_bytes(op.plan) > 0, "the case must need a workspace"
    assert ct.ct_workspace_bytes(op.plan) <= 32 * 1024 * 1024
    stream = ct._stream_ptr(None)
    rel, ab = TOL[torch.float16]
    xs = [draw(case["x_shape"], ("normal", 1.0), seed, torch.float16) for seed in (503, 504)]
    xds = [x.cuda() for x in xs]
    refs = [op(xd) for xd in xds]                         # ct_run, torch workspace
    ys = [torch.full(op.y_shape, float("nan"), dtype=torch.float16, device="cuda")
          for _ in xs]
    torch.cuda.synchronize()
    free = []
    for call in range(2):
        free.append(torch.cuda.mem_get_info()[0])
        ct.ct_run_noalloc(op.plan, ct._ptr(xds[call]), ct._ptr(op.w_packed), ct._ptr(op.bias),
                          ct._ptr(ys[call]), stream)
        torch.cuda.synchronize()
    free.append(torch.cuda.mem_get_info()[0])
    # the first call may load the module that holds the array; the second
    # call allocates nothing
    assert free[2] == free[1], free
    for call in range(2):
        assert torch.equal(ys[call], refs[call]), "call %d: ct_run_noalloc differs from ct_run" % call
        xa, wa, ba = to_oracle(xs[call], w, b, "nchw")
        ref, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
        err = np.abs(ys[call].double().cpu().numpy() - ref)
        assert np.all(err <= rel * absacc + ab), "call %d: outside the fp16 tolerance" % call


def test_run_noalloc_rejects_oversized_workspace():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # 8 x 256 x 128 x 128 fp16 input: a 64 MiB workspace, above the 32 MiB array
    d = ct.make_desc([8, 256, 128, 128], [256, 16, 2, 2], dtype=torch.float16,
                     strides=[2, 2])
    plan = ct.ct_plan(d)
    try:
        need = ct.ct_workspace_bytes(plan)
        assert need > 32 * 1024 * 1024
        with pytest.raises(ct.CtError) as e:
            ct.ct_run_noalloc(plan, ct.ctypes.c_void_p(256), ct.ctypes.c_void_p(256),
                              ct.ctypes.c_void_p(0), ct.ctypes.c_void_p(256), ct._stream_ptr(None))
        assert e.value.status == 8
    finally:
        ct.ct_plan_destroy(plan)
