"""nf4_quantize_noalloc: quantisation for callers that cannot allocate device
memory (for example a plugin whose host application owns all device memory,
or a service that reserves its memory at start-up and may not call cudaMalloc
later).  It keeps its scratch in a fixed array inside the library instead of a
caller workspace, and must give exactly what nf4_quantize gives.

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_lora_02_b200 as Q
from bit_quantized_lora_02_b200 import synth


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16).cuda()


def _arrays(q):
    n = q.d * q.k
    nblk = -(-n // 64)
    out = {"codes": q.codes[: (n + 1) // 2].cpu().numpy()}
    if q.double_quant:
        out["c2"] = q.c2[:nblk].cpu().numpy()
        out["c1"] = q.c1[: -(-nblk // 256)].cpu().numpy().view(np.uint32)
        out["mean"] = q.mean[:1].cpu().numpy().view(np.uint32)
    else:
        out["absmax"] = q.absmax[:nblk].cpu().numpy().view(np.uint32)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("dq", [1, 0, 2])
def test_noalloc_matches_workspace_entry_point_twice(dq):
    """Two calls in a row on different weights: each result equals the
    workspace entry point's bit for bit (the tolerance of every quantisation
    test here), and the second call is not disturbed by what the first left in
    the shared scratch.  dq: 0 single-level constants, 1 Int8 and 2 E4M3
    second-level constants."""
    shapes = [(1024, 4096), (777, 320)]
    results = []
    for i, (d, k) in enumerate(shapes):
        W = _dev(synth.weight(d, k, seed=40 + i, outliers=True))
        ref = Q.nf4_quantize(W, double_quant=dq)
        out = Q.nf4_alloc(d, k, dq, W.device)
        got = Q.nf4_quantize_noalloc(W, double_quant=dq, out=out)
        torch.cuda.synchronize()
        a, b = _arrays(ref), _arrays(got)
        for key in a:
            assert np.array_equal(a[key], b[key]), (d, k, key)
        results.append(b)
    assert Q.qlora_device_status() == 0


def test_noalloc_rejects_weights_above_the_scratch_limit():
    """Sizes beyond the built-in scratch fail with a clear error before any
    device work (fake, aligned pointers are never dereferenced)."""
    L = Q.lib()
    d, k = 1 << 15, 1 << 14          # 2^29 weights > 2^28
    st = Q.QloraNF4(d, k, 64, 1, 0x10000, None, 0x20000, 0x30000, 0x40000)
    rc = L.nf4_quantize_noalloc(0x50000, ctypes.byref(st), None)
    assert rc == -2
    msg = L.qlora_last_error().decode()
    assert "scratch limit" in msg and str(Q.NOALLOC_MAX_WEIGHTS) in msg
