"""linattn_forward_noalloc: the forward pass for callers that cannot allocate device memory
(hosts that reserve all device memory up front, runtimes that own the allocator and forbid
libraries from calling it).  It must give what linattn_forward gives, call after call, with
its temporary state in the library's fixed device scratch block, allocate nothing, and
report a kernel wait that gives up through linattn_device_error like every other entry point.

This file is collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.
"""
import numpy as np
import pytest

from linear_attention_linattn_b200 import inputs
from tests.helpers import TOL, as_io, max_row_rel_err, to_dev, to_host

torch = pytest.importorskip("torch")
la = pytest.importorskip("linear_attention_linattn_b200")

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, out, causal):
    B, H, n, d = q.shape
    dtype = la.LINATTN_BF16 if q.dtype == torch.bfloat16 else la.LINATTN_F32
    st = torch.cuda.current_stream().cuda_stream
    return lib.linattn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                       B, H, n, d, int(causal), dtype, st)


@pytest.mark.parametrize("dtype,B,H,n,d", [("bf16", 2, 3, 1000, 128), ("bf16", 1, 4, 4097, 64),
                                           ("f32", 1, 2, 777, 64),
                                           ("bf16", 1, 32, 131072, 128)])
@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_forward_on_two_calls(dtype, B, H, n, d, causal):
    lib = la.load_library()
    q, k, v = inputs.forward_qkv(17, B, H, n, d, scaled=True)
    qd, kd, vd = (to_dev(as_io(x, dtype), dtype) for x in (q, k, v))
    ref = to_host(la.forward(qd, kd, vd, causal))
    assert la.device_error() == la.LINATTN_OK
    for call in range(2):
        out = torch.full_like(qd, float("nan"))
        assert _noalloc(lib, qd, kd, vd, out, causal) == la.LINATTN_OK
        assert la.device_error() == la.LINATTN_OK, call
        got = to_host(out)
        assert np.all(np.isfinite(got)), call
        assert max_row_rel_err(got, ref) <= TOL[dtype], call


def test_noalloc_calls_leave_free_device_memory_unchanged():
    """After a first call (which looks the block's address up), further calls take no device
    memory: the driver's count of free memory is the same before and after them."""
    lib = la.load_library()
    B, H, n, d = 2, 8, 3000, 128
    q, k, v = inputs.forward_qkv(18, B, H, n, d, scaled=True)
    qd, kd, vd = (to_dev(as_io(x, "bf16"), "bf16") for x in (q, k, v))
    out = torch.empty_like(qd)
    for causal in (True, False):
        assert _noalloc(lib, qd, kd, vd, out, causal) == la.LINATTN_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for causal in (True, False, True):
        assert _noalloc(lib, qd, kd, vd, out, causal) == la.LINATTN_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert la.device_error() == la.LINATTN_OK


def test_noalloc_wait_give_up_is_reported_once():
    """A bounded wait that gives up writing into the static block's status word is reported by
    linattn_device_error once (then cleared), and the next call still matches."""
    lib = la.load_library()
    st = torch.cuda.current_stream().cuda_stream
    assert la.device_error() == la.LINATTN_OK
    assert lib.linattn_selftest_noalloc_wait_timeout(st) == la.LINATTN_OK
    assert la.device_error() == la.LINATTN_ERR_TIMEOUT
    assert la.device_error() == la.LINATTN_OK
    B, H, n, d = 1, 2, 500, 64
    q, k, v = (as_io(x, "bf16") for x in inputs.forward_qkv(19, B, H, n, d, scaled=True))
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    out = torch.empty_like(qd)
    ref = to_host(la.forward(qd, kd, vd, True))
    assert _noalloc(lib, qd, kd, vd, out, True) == la.LINATTN_OK
    assert la.device_error() == la.LINATTN_OK
    assert max_row_rel_err(to_host(out), ref) <= TOL["bf16"]


def test_noalloc_rejects_work_beyond_the_scratch_block():
    lib = la.load_library()
    # 4096 heads of d = 128 need 4096 x 66,048 B of state even with one segment each
    B, H, n, d = 1, 4096, 64, 128
    q = torch.zeros((B, H, n, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    assert _noalloc(lib, q, q, q, out, True) == la.LINATTN_ERR_INVALID_ARG
    assert _noalloc(lib, q, q, q, out, False) == la.LINATTN_ERR_INVALID_ARG
