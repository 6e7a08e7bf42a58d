"""Failure detection on the device, exercised without any fault.

Every wait in the library's kernels is bounded: when one runs out, the kernel
records a code in the per-device status word, releases its TMEM and returns,
and the host reads the code with qlora_device_status.  The self-test entry
point runs that path on a barrier nothing arrives at, with a 2 ms limit; the
test checks that the call returns, that the code is reported once, that the
kernel released its TMEM before finishing, and that the context stays usable
(a layer call afterwards still matches the oracle)."""
import time

import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_f32


def test_bounded_wait_runs_out_and_reports():
    assert Q.qlora_device_status() == 0
    t0 = time.perf_counter()
    result = Q.qlora_selftest_wait_timeout(2000)      # 2 ms limit
    elapsed = time.perf_counter() - t0
    assert result == 2                                # gave up, then released its TMEM
    assert elapsed < 5.0
    assert Q.qlora_device_status() == 7               # DEV_WAIT_TIMEOUT_SELFTEST
    assert Q.qlora_device_status() == 0               # read once, then cleared

    # the context is still usable: the tiny layer matches the oracle
    L = synth.layer(16, 512, 512, 8, seed=0, a_std=1.0 / 8)
    q = Q.nf4_quantize(dev_bf16(L["W0"]))
    X, A, B = (dev_bf16(L[n]) for n in ("X", "A", "B"))
    Y, _ = Q.qlora_linear_fwd(X, q, A, B, 16.0)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0
    Wh = O.dequantize_tensor(O.quantize_tensor(L["W0"].reshape(-1), True)).reshape(512, 512)
    Y_ref, _ = O.qlora_forward(L["X"], Wh, L["A"], L["B"], 16.0, 8)
    assert_close(host_f32(Y), Y_ref, "Y after the self-test")


def test_selftest_rejects_bad_limits():
    res = torch.zeros(1, dtype=torch.int32, device="cuda")
    L = Q.lib()
    assert L.qlora_selftest_wait_timeout(0, res.data_ptr(), None) == -1
    assert L.qlora_selftest_wait_timeout(2000000, res.data_ptr(), None) == -1
    assert L.qlora_selftest_wait_timeout(100, None, None) == -1
    assert np.all(res.cpu().numpy() == 0)             # nothing was launched
