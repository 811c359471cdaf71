"""The failure path on the GPU, without a fault: a wait that nothing completes gives up after
its limit, the host reads LINATTN_ERR_TIMEOUT once, and the context stays usable."""
import numpy as np
import pytest

import oracle
from linear_attention_linattn_b200 import inputs
from tests.helpers import TOL, max_row_rel_err, to_dev, to_host

torch = pytest.importorskip("torch")
la = pytest.importorskip("linear_attention_linattn_b200")

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    lib = la.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    assert la.device_error() == la.LINATTN_OK          # nothing pending
    assert lib.linattn_selftest_wait_timeout(stream) == la.LINATTN_OK
    assert la.device_error() == la.LINATTN_ERR_TIMEOUT  # the wait gave up (about 2 s)
    assert la.device_error() == la.LINATTN_OK          # reported once, then cleared
    # the context still works
    q, k, v = inputs.forward_qkv(61, 1, 2, 300, 64, scaled=True)
    out = to_host(la.forward(to_dev(q, "f32"), to_dev(k, "f32"), to_dev(v, "f32"), True))
    assert la.device_error() == la.LINATTN_OK
    assert max_row_rel_err(out, oracle.forward(q, k, v, True)) <= TOL["f32"]
