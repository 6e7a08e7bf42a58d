"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and its host-only functions (sizes, validation, codebook)
behave as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_quantized_lora_02_b200 as Q
from oracle import qlora_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from bit_quantized_lora_02_b200 import build
    build.build()
    return Q.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    declared = header_functions()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(declared) == sorted(Q.EXPORTS)


def test_codebook_matches_oracle_bitwise(L):
    lib_table = np.array(Q.qlora_nf4_codebook(), np.float32)
    assert np.array_equal(lib_table.view(np.uint32), O.nf4_codebook().view(np.uint32))


def test_sizes_closed_form(golden):
    g = golden("storage_accounting.json")
    sizes, ws = Q.qlora_nf4_sizes(4096, 4096, 64, True)
    assert sizes == [8388608, 0, 262144, 4096, 4]
    assert sum(sizes) == 8654852
    n = 4096 * 4096
    bits_consts = (sizes[2] + sizes[3]) * 8 / n
    assert bits_consts == g["bits_per_weight_after"]
    sizes0, ws0 = Q.qlora_nf4_sizes(4096, 4096, 64, False)
    assert sizes0 == [8388608, 4 * 262144, 0, 0, 0] and ws0 == 0
    assert sizes0[1] * 8 / n == g["bits_per_weight_before"]
    assert ws > 0


def test_sizes_ragged():
    sizes, _ = Q.qlora_nf4_sizes(3, 37, 64, True)   # N = 111 -> 2 blocks, 1 group
    assert sizes == [56, 0, 2, 4, 4]
    sizes, _ = Q.qlora_nf4_sizes(0, 5, 64, True)
    assert sizes[0] == 0 and sizes[2] == 0


def test_unsupported_blocksize_and_bad_args(L):
    with pytest.raises(Q.QLoRAError) as e:
        Q.qlora_nf4_sizes(64, 64, 32, True)
    assert e.value.code == -2 and "blocksize" in str(e.value)
    with pytest.raises(Q.QLoRAError) as e:
        Q.qlora_nf4_sizes(-1, 64, 64, True)
    assert e.value.code == -1


def test_quantize_rejects_null_and_misaligned_without_gpu(L):
    st = Q.QloraNF4(64, 64, 64, 1, None, None, None, None, None)
    rc = L.nf4_quantize(None, ctypes.byref(st), None, 0, None)
    assert rc == -1 and b"codes" in L.qlora_last_error()
    st = Q.QloraNF4(64, 64, 64, 1, 0x1000, None, 0x2000, 0x3000, 0x4000)
    rc = L.nf4_quantize(0x1001, ctypes.byref(st), 0x5000, 1 << 20, None)
    assert rc == -3 and b"W0" in L.qlora_last_error()
    rc = L.nf4_quantize(0x1000, ctypes.byref(st), 0x5000, 4, None)
    assert rc == -4 and b"workspace" in L.qlora_last_error()
    st = Q.QloraNF4(64, 64, 64, 1, 0x1000, None, 0x2001, 0x3000, 0x4000)
    assert L.nf4_quantize(0x1000, ctypes.byref(st), 0x5000, 1 << 20, None) == -3


def test_linear_shape_validation(L):
    n = ctypes.c_size_t()
    assert L.qlora_linear_workspace_size(16, 512, 512, 8, 0, ctypes.byref(n)) == 0 and n.value > 0
    assert L.qlora_linear_workspace_size(16, 512, 500, 8, 0, ctypes.byref(n)) == -2      # k % 64
    assert L.qlora_linear_workspace_size(16, 510, 512, 8, 0, ctypes.byref(n)) == -2      # d % 8
    assert L.qlora_linear_workspace_size(16, 512, 512, 0, 0, ctypes.byref(n)) == -2      # r
    assert L.qlora_linear_workspace_size(16, 512, 512, 257, 0, ctypes.byref(n)) == -2
    assert L.qlora_linear_workspace_size(-1, 512, 512, 8, 0, ctypes.byref(n)) == -1
    assert L.qlora_rank_pad(8) == 64 and L.qlora_rank_pad(64) == 64 and L.qlora_rank_pad(65) == 128


def test_linear_rejects_null_inputs_without_gpu(L):
    st = Q.QloraNF4(512, 512, 64, 1, 0x1000, None, 0x2000, 0x3000, 0x4000)
    rc = L.qlora_linear_fwd(None, 16, ctypes.byref(st), 0x10000, 0x20000, 8, 16.0, 0x30000, None, 0x40000,
                            1 << 30, None)
    assert rc == -1 and b"X" in L.qlora_last_error()
    rc = L.qlora_linear_fwd(0x10000, 16, ctypes.byref(st), 0x10000, 0x20000, 8, 16.0, 0x30000, None, None, 0, None)
    assert rc == -4
    # M == 0 is a no-op that succeeds without touching memory
    assert L.qlora_linear_fwd(None, 0, ctypes.byref(st), None, None, 8, 16.0, None, None, None, 0, None) == 0


def test_fp8_constants_mode(L):
    sizes = (ctypes.c_size_t * 5)()
    ws = ctypes.c_size_t()
    assert L.qlora_nf4_sizes(512, 512, 64, 2, sizes, ctypes.byref(ws)) == 0
    fp8 = (list(sizes), ws.value)
    assert L.qlora_nf4_sizes(512, 512, 64, 1, sizes, ctypes.byref(ws)) == 0
    assert fp8 == (list(sizes), ws.value)            # one byte per block either way, same c1, mean and scratch
    assert L.qlora_nf4_sizes(512, 512, 64, 3, sizes, ctypes.byref(ws)) == -1


def test_merge_validation_without_gpu(L):
    st = Q.QloraNF4(512, 512, 64, 1, 0x1000, None, 0x2000, 0x3000, 0x4000)
    rc = L.qlora_lora_merge(ctypes.byref(st), None, 0x20000, 8, 16.0, 0x30000, None)
    assert rc == -1 and b"A" in L.qlora_last_error()
    assert L.qlora_lora_merge(ctypes.byref(st), 0x10000, 0x20000, 0, 16.0, 0x30000, None) == -2     # r
    assert L.qlora_lora_merge(ctypes.byref(st), 0x10000, 0x20000, 257, 16.0, 0x30000, None) == -2
    assert L.qlora_lora_merge(ctypes.byref(st), 0x10000, 0x20000, 8, 16.0, 0x30008, None) == -3     # W_out
    bad = Q.QloraNF4(512, 500, 64, 1, 0x1000, None, 0x2000, 0x3000, 0x4000)
    assert L.qlora_lora_merge(ctypes.byref(bad), 0x10000, 0x20000, 8, 16.0, 0x30000, None) == -2    # k % 64
    odd = Q.QloraNF4(512, 512, 64, 1, 0x1004, None, 0x2000, 0x3000, 0x4000)
    assert L.qlora_lora_merge(ctypes.byref(odd), 0x10000, 0x20000, 8, 16.0, 0x30000, None) == -3    # codes


def test_param_count_matches_buffer_shapes(golden):
    g = golden("lora_param_count.json")
    # A is r x k and B is d x r: the entries the backward writes
    assert g["r"] * g["k"] + g["d"] * g["r"] == g["trainable"]


def test_dropout_validation_without_gpu(L):
    """Adapter dropout entry points: the probability must lie in [0, 1), the
    workspace grows by the keep bitmask (M k / 8 bytes rounded up to 256), and
    every refusal happens before any device work (fake aligned pointers)."""
    n, nd = ctypes.c_size_t(), ctypes.c_size_t()
    for bwd in (0, 1):
        assert L.qlora_linear_workspace_size(200, 520, 704, 16, bwd, ctypes.byref(n)) == 0
        assert L.qlora_linear_dropout_workspace_size(200, 520, 704, 16, bwd, ctypes.byref(nd)) == 0
        mask = -(-200 * 704 // 32) * 4
        assert nd.value == -(-n.value // 256) * 256 + -(-mask // 256) * 256
    assert L.qlora_linear_dropout_workspace_size(16, 512, 500, 8, 0, ctypes.byref(nd)) == -2   # k % 64
    st = Q.QloraNF4(512, 512, 64, 1, 0x1000, None, 0x2000, 0x3000, 0x4000)
    for p in (1.0, 1.5, -0.1, float("nan")):
        drop = Q.QloraDropout(p, 1, 2)
        rc = L.qlora_linear_fwd_dropout(0x10000, 16, ctypes.byref(st), 0x10000, 0x20000, 8, 16.0, ctypes.byref(drop),
                                        0x30000, None, 0x40000, 1 << 30, None)
        assert rc == -1 and b"[0, 1)" in L.qlora_last_error(), p
        rc = L.qlora_linear_bwd_dropout(0x10000, 0x10000, 16, ctypes.byref(st), 0x10000, 0x20000, 8, 16.0,
                                        ctypes.byref(drop), None, 0x30000, 0x40000, 0x50000, 0x60000, 1 << 30, None)
        assert rc == -1, p
        assert L.qlora_dropout_mask(4, 64, ctypes.byref(drop), 0x10000, None) == -1
    drop = Q.QloraDropout(0.05, 1, 2)
    # a workspace sized for the plain layer is too small once the mask is needed
    L.qlora_linear_workspace_size(16, 512, 512, 8, 0, ctypes.byref(n))
    rc = L.qlora_linear_fwd_dropout(0x10000, 16, ctypes.byref(st), 0x10000, 0x20000, 8, 16.0, ctypes.byref(drop),
                                    0x30000, None, 0x40000, n.value, None)
    assert rc == -4
    assert L.qlora_dropout_mask(4, 64, None, 0x10000, None) == -1
    assert L.qlora_dropout_mask(4, 64, ctypes.byref(drop), None, None) == -1
    assert L.qlora_dropout_mask(4, 64, ctypes.byref(drop), 0x10002, None) == -3       # 4-byte alignment
    assert L.qlora_dropout_mask(0, 64, ctypes.byref(drop), None, None) == 0            # nothing to do


def test_selftest_validation_without_gpu(L):
    assert L.qlora_selftest_wait_timeout(0, 0x10000, None) == -1
    assert L.qlora_selftest_wait_timeout(1000001, 0x10000, None) == -1
    assert L.qlora_selftest_wait_timeout(100, None, None) == -1
    assert L.qlora_selftest_wait_timeout(100, 0x10002, None) == -3


def test_grouped_validation_without_gpu(L):
    """Grouped projections: 1..4 projections, all but the last a multiple of
    256 rows summing to the stacked weight, n r <= 256 and r % 8 == 0; the
    workspace equals the plain layer's for the stacked rows and ranks."""
    def group(ds, k=512, total=None):
        g = Q.QloraNF4Group()
        g.n = len(ds)
        for i, x in enumerate(ds):
            g.d[i] = x
        g.w = Q.QloraNF4(sum(ds) if total is None else total, k, 64, 1, 0x1000, None, 0x2000, 0x3000, 0x4000)
        return g
    n, n1 = ctypes.c_size_t(), ctypes.c_size_t()
    g = group([256, 256, 520])
    for bwd in (0, 1):
        assert L.qlora_grouped_workspace_size(300, ctypes.byref(g), 16, bwd, ctypes.byref(n)) == 0
        assert L.qlora_linear_workspace_size(300, 1032, 512, 48, bwd, ctypes.byref(n1)) == 0
        assert n.value == n1.value
    assert L.qlora_grouped_workspace_size(300, ctypes.byref(group([200, 256])), 16, 0, ctypes.byref(n)) == -2
    assert L.qlora_grouped_workspace_size(300, ctypes.byref(group([256, 256], total=768)), 16, 0,
                                          ctypes.byref(n)) == -1
    assert L.qlora_grouped_workspace_size(300, ctypes.byref(group([256, 256, 256])), 96, 0, ctypes.byref(n)) == -2
    assert L.qlora_grouped_workspace_size(300, ctypes.byref(group([256, 256])), 12, 0, ctypes.byref(n)) == -2
    assert L.qlora_grouped_workspace_size(300, ctypes.byref(group([])), 16, 0, ctypes.byref(n)) == -1
    assert L.qlora_grouped_workspace_size(300, None, 16, 0, ctypes.byref(n)) == -1
    g = group([256, 256])
    rc = L.qlora_linear_fwd_grouped(0x10000, 300, ctypes.byref(g), 0x10000, 0x20000, 16, 16.0, 0x30000, None, None,
                                    0, None)
    assert rc == -4                                   # workspace missing, before any device work
    rc = L.qlora_linear_bwd_grouped(0x10000, 0x10000, 300, ctypes.byref(g), 0x10000, 0x20000, 16, 16.0, None,
                                    None, 0x30000, 0x40000, None, 0, None)
    assert rc == -4


def test_group_buffers_are_slices_of_the_stack():
    """The binding's stacked allocation: slice i starts where the earlier
    projections' buffers end (codes, c2, c1) and holds projection i's mean."""
    import torch
    ds, k = (256, 512, 264), 1024
    sizes = [Q.qlora_nf4_sizes(d, k, 64, 1)[0] for d in ds]
    codes = torch.zeros(sum(s[0] for s in sizes) + 16, dtype=torch.uint8)
    off = 0
    for d, s in zip(ds, sizes):
        assert s[0] == d * k // 2 and s[2] == d * k // 64
        off += s[0]
    assert off == sum(ds) * k // 2
    assert all(s[3] == d * k // 64 // 256 * 4 for d, s in zip(ds[:-1], sizes[:-1]))
    st = Q.qlora_nf4_sizes(sum(ds), k, 64, 1)[0]
    assert st[0] == off and st[2] == sum(s[2] for s in sizes) and st[3] == sum(s[3] for s in sizes)
    del codes
