"""The kernels' bounded waits: clean after every other test, and the failure
path run on purpose (GPU).

Runs after the parity test files (file name order): the device error words
of the tensor-core and grouped modules persist until read, so a clean read
here also shows that no wait ran out in any earlier test of this process.
Then a wait is made to run out on purpose: the library's self-test kernel
starts a bulk copy into its shared memory and waits, with a short limit, on
an mbarrier nothing arrives at.  It must record its site (code 501), drain
its copy and return, and the device must still run a normal call afterwards.
No GPU fault or hang is involved: the wait is bounded and the kernel ends.
"""

import pytest
import torch

from parity import full_parity
from transposed_convolution_02_b200 import ct

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_device_error_words_clear_after_runs():
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


@pytest.mark.parametrize("limit", [1, 20000])
def test_wait_that_runs_out_is_reported_and_device_stays_usable(limit):
    assert ct.ct_take_device_error() == 0
    ct.ct_selftest_wait_timeout(limit)
    # site 1: the wait on the barrier nobody arrives at gave up; the drain of
    # the copy in flight completed (site 2 would say otherwise)
    assert ct.ct_take_device_error() == 501
    assert ct.ct_take_device_error() == 0          # read and cleared
    # the context is intact: a normal tensor-core call still matches the oracle
    full_parity(dict(x_shape=[2, 64, 11, 13], w_shape=[64, 40, 4, 4], strides=[2, 2],
                     pads=[1, 1, 1, 1], bias=True), torch.float16, 74 + limit % 7,
                algo="dense_tc_pair", expect_kernel="dense_tc_pair")
    torch.cuda.synchronize()
    assert ct.ct_take_device_error() == 0
