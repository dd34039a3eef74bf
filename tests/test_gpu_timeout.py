"""The bounded waits: a wait on a pipeline barrier that nothing ever signals
must give up after the configured limit, record FA_ERR_TIMEOUT in the device
status word, and leave the CUDA context usable (no trap, no fault, no hang)."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_wait_gives_up_reports_timeout_and_context_survives(lib):
    import torch

    from io_aware_exact_20_b200.workloads import make_qkvdo
    from oracle import attention_forward

    assert lib.last_device_status() == 0
    lib.set_wait_timeout_ns(50_000_000)  # 50 ms
    try:
        lib.wait_timeout_probe()
        assert lib.last_device_status() == 4  # FA_ERR_TIMEOUT
        assert lib.last_device_status() == 0  # reading clears it
    finally:
        lib.set_wait_timeout_ns(4_000_000_000)
    q, k, v, _ = make_qkvdo(1, 1, 256, 64, 3)
    o, lse = lib.forward(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    ro, _ = attention_forward(f(q), f(k), f(v), 64 ** -0.5)
    assert np.abs(f(o) - ro).max() < 1e-2
