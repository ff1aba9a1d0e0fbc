"""Failure detection without faulting the GPU (B200 only).

Every failure here is made on purpose and bounded: a kernel waits on a
barrier that nothing sets and must give up, record the timeout and return;
Adam must flag a non-finite update; the context stays usable afterwards.
(Host-side failures -- bad arguments, the SPIN4D_FAULT hook -- are covered
without a GPU in tests/test_abi.py.)"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sp():
    from spatiotemporal_neural_field_b200 import spin4d
    return spin4d


def test_bounded_wait_times_out_and_is_reported(sp):
    """The self-test kernel (libspin4d_probe.so) waits, through the decoder
    kernels' bounded mbarrier wait, on a barrier nothing arrives at."""
    from spatiotemporal_neural_field_b200 import probe as pr
    pr.check_device_errors(clear=True)                  # start clean
    pr.selftest_wait_timeout(max_iters=4096)
    torch.cuda.synchronize()
    with pytest.raises(sp.Spin4dError) as e:
        pr.check_device_errors(clear=True)
    assert e.value.status == sp.ERR_TIMEOUT
    pr.check_device_errors(clear=False)                 # cleared: no error any more
    sp.check_device_errors(clear=False)                 # the decoder library's word is untouched
    # the context is still usable: a real decode runs and is correct
    x = torch.arange(16, dtype=torch.float32, device="cuda").reshape(4, 4)
    assert float(x.sum()) == 120.0


def test_adam_flags_non_finite_updates(sp):
    n = 1000
    p = torch.zeros(n, device="cuda")
    g = torch.ones(n, device="cuda")
    g[123] = float("nan")
    m, v = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp.adam_step(p, g, m, v, 1, 1e-3, 0.9, 0.99, 1e-15, nonfinite_flag=flag)
    assert int(flag.item()) == 1
    ok = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp.adam_step(torch.zeros(n, device="cuda"), torch.ones(n, device="cuda"), torch.zeros(n, device="cuda"),
                 torch.zeros(n, device="cuda"), 1, 1e-3, 0.9, 0.99, 1e-15, nonfinite_flag=ok)
    assert int(ok.item()) == 0
