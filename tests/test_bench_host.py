"""Host-side checks of bench.py's arithmetic and report logic (no GPU)."""
import importlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
bench = importlib.import_module("bench")


def _gemm(m, n, k):
    return 2 * m * n * k


@pytest.mark.parametrize("M,d,k,r", [(4096, 4096, 4096, 64), (4096, 11008, 4096, 64), (7, 520, 704, 5)])
def test_flop_counts_enumerate_the_products(M, d, k, r):
    # forward: T = X A^T (M x r over k), Y = X W^T (M x d over k), + T B^T (M x d over r)
    fwd = _gemm(M, r, k) + _gemm(M, d, k) + _gemm(M, d, r)
    # backward: U = dY B (M x r over d), dX = dY W (M x k over d) + U A (M x k over r),
    # dA = U^T X (r x k over M), dB = dY^T T (d x r over M); T is saved by the forward
    bwd = _gemm(M, r, d) + _gemm(M, k, d) + _gemm(M, k, r) + _gemm(r, k, M) + _gemm(d, r, M)
    assert bench.flops_fwd(M, d, k, r) == fwd
    assert bench.flops_bwd(M, d, k, r) == bwd
    assert bench.main_fwd_flops(M, d, k, r) == _gemm(M, d, k) + _gemm(M, d, r)
    assert bench.main_bwd_flops(M, d, k, r) == _gemm(M, k, d) + _gemm(M, k, r)


def test_default_step_flops():
    from bit_quantized_lora_02_b200 import synth
    work = synth.WORKLOADS["llama7b_proj_set_m4096"]
    M, r = work["m"], work["r"]
    total = sum(bench.flops_fwd(M, d, k, r) + bench.flops_bwd(M, d, k, r) for _, d, k in work["proj"])
    assert abs(total / 1e12 - 3.4385) < 5e-4


def test_traffic_counts_only_under_matching_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic_fwd_gemm_wl.txt").write_text("# comment = ignored\nbytes_per_launch = 1234\nsource_hash = abc\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.read_traffic("fwd_gemm", "wl") == 1234.0
    assert bench.read_traffic("fwd_gemm", "other") is None   # another workload has its own file
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "def")
    assert bench.read_traffic("fwd_gemm", "wl") is None
    assert bench.read_traffic("bwd_gemm", "wl") is None   # no file


def test_65b_step_flops():
    from bit_quantized_lora_02_b200 import synth
    work = synth.WORKLOADS["llama65b_block_m8192"]
    M, r = work["m"], work["r"]
    total = sum(bench.flops_fwd(M, d, k, r) + bench.flops_bwd(M, d, k, r) for _, d, k in work["proj"])
    assert abs(total / 1e12 - 27.017) < 5e-3


def test_source_hash_ignores_comments():
    src = "int f(int a) {  // add one\n  /* body */ return a + 1;\n}\n"
    assert bench._code_only(src) == bench._code_only("int f(int a) {\n   return a + 1;\n}\n")
    assert bench._code_only(src) != bench._code_only("int f(int a) {\n  return a + 2;\n}\n")
