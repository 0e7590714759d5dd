"""ct_run_noalloc against ct_run, on the GPU.

ct_run_noalloc serves callers that may not allocate device memory while they
run (for example a plugin inside an engine that owns all device memory): it
takes its workspace from a fixed array inside libct.so instead of from the
caller.  Here it runs a plan that needs a workspace (fp16 channels-first on
the tensor-core path, whose input is re-laid channels-last into it) twice in
a row, on two different inputs, and each result must match what ct_run gives
with a torch-allocated workspace, within the fp16 parity tolerance.

This file sorts last so that a run that stops at the first failure has
already run every other test.
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
    for call, seed in enumerate((503, 504)):
        x = draw(case["x_shape"], ("normal", 1.0), seed, torch.float16)
        xd = x.cuda()
        y_ref = op(xd)                                    # ct_run, torch workspace
        y = torch.full(op.y_shape, float("nan"), dtype=torch.float16, device="cuda")
        ct.ct_run_noalloc(op.plan, ct._ptr(xd), ct._ptr(op.w_packed), ct._ptr(op.bias),
                          ct._ptr(y), stream)
        torch.cuda.synchronize()
        xa, wa, ba = to_oracle(x, w, b, "nchw")
        _, absacc = conv_transpose_ref(xa, wa, ba, attrs_from(case))
        diff = (y.double() - y_ref.double()).abs().cpu().numpy()
        bound = rel * absacc + ab
        assert np.all(diff <= bound), "call %d: ct_run_noalloc differs from ct_run" % call


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
