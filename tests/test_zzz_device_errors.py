"""The kernels' bounded waits left no error code behind (GPU).

Runs after the other GPU test files (file name order): the device error
words of the tensor-core and grouped modules persist until read, so a clean
read here also shows that no wait ran out in any earlier test of this
process.  The failure path itself (a wait that gives up) is not provoked on
a GPU: its recording is the same atomic store for every wait site.
"""

import pytest
import torch

from parity import full_parity
from transposed_convolution_02_b200 import ct

pytestmark = pytest.mark.gpu


def test_device_error_words_clear_after_runs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    full_parity(dict(x_shape=[2, 64, 20, 24], w_shape=[64, 48, 4, 4], strides=[2, 2],
                     pads=[1, 1, 1, 1], bias=True), torch.float16, 71, algo="dense_tc_pair",
                expect_kernel="dense_tc_pair")
    full_parity(dict(x_shape=[1, 32, 6, 8, 8], w_shape=[32, 16, 3, 3, 3], strides=[2, 2, 2],
                     pads=[1, 1, 1, 1, 1, 1], bias=False), torch.float16, 72, algo="dense_tc",
                expect_kernel="dense_tc")
    full_parity(dict(x_shape=[2, 64, 13, 11], w_shape=[64, 16, 3, 3], strides=[2, 2],
                     dilations=[2, 2], auto_pad="SAME_UPPER", group=4, bias=True),
                torch.float16, 73, algo="grouped", expect_kernel="grouped")
    torch.cuda.synchronize()
    assert ct.ct_take_device_error() == 0
    assert ct.ct_take_device_error() == 0
