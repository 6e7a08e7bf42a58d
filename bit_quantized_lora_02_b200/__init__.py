"""QLoRA linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding of ``libqlora.so`` (C ABI in ``include/qlora.h``).  The
functions below only marshal arguments: every step of quantisation,
dequantisation, forward and backward runs in the library's CUDA kernels.
PyTorch is used for device memory and streams.  There is no fallback: if the
library is missing or a call fails, a ``QLoRAError`` is raised.

Names follow the C ABI: ``nf4_quantize``, ``nf4_dequantize``,
``qlora_linear_fwd``, ``qlora_linear_bwd``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QLORA_OK = 0
_STATUS = {0: "QLORA_OK", -1: "QLORA_ERR_INVALID_ARG", -2: "QLORA_ERR_UNSUPPORTED", -3: "QLORA_ERR_ALIGNMENT",
           -4: "QLORA_ERR_WORKSPACE", -5: "QLORA_ERR_CUDA", -6: "QLORA_ERR_DEVICE"}

EXPORTS = ("qlora_nf4_sizes", "nf4_quantize", "nf4_quantize_noalloc", "nf4_dequantize", "qlora_lora_merge",
           "qlora_rank_pad", "qlora_linear_workspace_size",
           "qlora_linear_fwd", "qlora_linear_bwd", "qlora_nf4_codebook", "qlora_device_status", "qlora_last_error",
           "qlora_profile_enable", "qlora_profile_read",
           "qlora_dropout_mask", "qlora_linear_dropout_workspace_size", "qlora_linear_fwd_dropout",
           "qlora_linear_bwd_dropout", "qlora_selftest_wait_timeout", "qlora_grouped_workspace_size",
           "qlora_linear_fwd_grouped", "qlora_linear_bwd_grouped")

KERNEL_CLASSES = ("quant", "dq_const", "dequant", "fwd_gemm", "bwd_gemm", "lora_gemm", "aux")


class QLoRAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_STATUS.get(code, code)}: {msg}")
        self.code = code


class QloraNF4(ctypes.Structure):
    """Mirror of ``qlora_nf4_t``."""
    _fields_ = [("d", ctypes.c_int64), ("k", ctypes.c_int64), ("blocksize", ctypes.c_int32),
                ("double_quant", ctypes.c_int32), ("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("c2", ctypes.c_void_p), ("c1", ctypes.c_void_p), ("mean", ctypes.c_void_p)]


MAX_GROUP = 4


class QloraNF4Group(ctypes.Structure):
    """Mirror of ``qlora_nf4_group_t``."""
    _fields_ = [("n", ctypes.c_int32), ("d", ctypes.c_int64 * MAX_GROUP), ("w", QloraNF4)]


class QloraDropout(ctypes.Structure):
    """Mirror of ``qlora_dropout_t``: adapter dropout probability p and the
    generator's (seed, offset)."""
    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqlora.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise QLoRAError(-5, f"{LIB_PATH} is missing; build it with `python -m bit_quantized_lora_02_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    c_i64, c_i32, c_sz, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
    L.qlora_nf4_sizes.argtypes = [c_i64, c_i64, c_i32, c_i32, ctypes.POINTER(c_sz), ctypes.POINTER(c_sz)]
    L.nf4_quantize.argtypes = [vp, ctypes.POINTER(QloraNF4), vp, c_sz, vp]
    L.nf4_quantize_noalloc.argtypes = [vp, ctypes.POINTER(QloraNF4), vp]
    L.nf4_dequantize.argtypes = [ctypes.POINTER(QloraNF4), vp, vp]
    L.qlora_lora_merge.argtypes = [ctypes.POINTER(QloraNF4), vp, vp, c_i32, ctypes.c_float, vp, vp]
    L.qlora_rank_pad.argtypes = [c_i32]
    L.qlora_rank_pad.restype = c_i32
    L.qlora_linear_workspace_size.argtypes = [c_i64, c_i64, c_i64, c_i32, c_i32, ctypes.POINTER(c_sz)]
    L.qlora_linear_fwd.argtypes = [vp, c_i64, ctypes.POINTER(QloraNF4), vp, vp, c_i32, ctypes.c_float, vp, vp, vp,
                                   c_sz, vp]
    L.qlora_linear_bwd.argtypes = [vp, vp, c_i64, ctypes.POINTER(QloraNF4), vp, vp, c_i32, ctypes.c_float, vp, vp,
                                   vp, vp, vp, c_sz, vp]
    L.qlora_nf4_codebook.argtypes = [ctypes.POINTER(ctypes.c_float)]
    L.qlora_device_status.argtypes = [vp, ctypes.POINTER(c_i32)]
    L.qlora_dropout_mask.argtypes = [c_i64, c_i64, ctypes.POINTER(QloraDropout), vp, vp]
    L.qlora_linear_dropout_workspace_size.argtypes = [c_i64, c_i64, c_i64, c_i32, c_i32, ctypes.POINTER(c_sz)]
    L.qlora_linear_fwd_dropout.argtypes = [vp, c_i64, ctypes.POINTER(QloraNF4), vp, vp, c_i32, ctypes.c_float,
                                           ctypes.POINTER(QloraDropout), vp, vp, vp, c_sz, vp]
    L.qlora_linear_bwd_dropout.argtypes = [vp, vp, c_i64, ctypes.POINTER(QloraNF4), vp, vp, c_i32, ctypes.c_float,
                                           ctypes.POINTER(QloraDropout), vp, vp, vp, vp, vp, c_sz, vp]
    L.qlora_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp, vp]
    G = ctypes.POINTER(QloraNF4Group)
    L.qlora_grouped_workspace_size.argtypes = [c_i64, G, c_i32, c_i32, ctypes.POINTER(c_sz)]
    L.qlora_linear_fwd_grouped.argtypes = [vp, c_i64, G, vp, vp, c_i32, ctypes.c_float, vp, vp, vp, c_sz, vp]
    L.qlora_linear_bwd_grouped.argtypes = [vp, vp, c_i64, G, vp, vp, c_i32, ctypes.c_float, vp, vp, vp, vp, vp,
                                           c_sz, vp]
    L.qlora_last_error.restype = ctypes.c_char_p
    L.qlora_profile_enable.argtypes = [c_i32]
    L.qlora_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
    for name in ("qlora_nf4_sizes", "nf4_quantize", "nf4_quantize_noalloc", "nf4_dequantize", "qlora_lora_merge",
                 "qlora_linear_workspace_size",
                 "qlora_linear_fwd", "qlora_linear_bwd", "qlora_nf4_codebook", "qlora_device_status",
                 "qlora_profile_enable", "qlora_profile_read", "qlora_dropout_mask",
                 "qlora_linear_dropout_workspace_size", "qlora_linear_fwd_dropout", "qlora_linear_bwd_dropout",
                 "qlora_selftest_wait_timeout", "qlora_grouped_workspace_size", "qlora_linear_fwd_grouped",
                 "qlora_linear_bwd_grouped"):
        getattr(L, name).restype = c_i32
    _lib = L
    return L


def _check(rc: int) -> None:
    if rc != QLORA_OK:
        raise QLoRAError(rc, lib().qlora_last_error().decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _expect(t: Optional[torch.Tensor], name: str, shape, dtype, required: bool = True) -> None:
    """The C ABI sees raw pointers only: check dtype, exact shape and row-major
    contiguity here, so that a mismatched tensor raises instead of being read
    or written past its end."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(int(x) for x in shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def _same_device(dev, **tensors) -> None:
    """Every pointer of one call must live on the device the call runs on."""
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the call runs on {dev}")


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# quantized weight container
# ---------------------------------------------------------------------------
@dataclass
class NF4Weight:
    """Device buffers of one quantized weight (layout of ``qlora_nf4_t``)."""
    d: int
    k: int
    double_quant: int          # 0: fp32 absmax; 1 (or True): Int8 c2; 2: FP8 E4M3 c2
    codes: torch.Tensor
    absmax: Optional[torch.Tensor] = None
    c2: Optional[torch.Tensor] = None
    c1: Optional[torch.Tensor] = None
    mean: Optional[torch.Tensor] = None
    blocksize: int = 64

    def struct(self, device=None) -> QloraNF4:
        """The C struct, after checking every buffer against the sizes the
        library needs for a d x k weight in this mode: dtype, byte size,
        contiguity and device (``device``: the activations' device, when the
        call has activations).  A short or misplaced buffer raises here instead
        of being read or written past its end."""
        mode = int(self.double_quant)
        if mode not in (0, 1, 2):
            raise ValueError(f"double_quant must be 0, 1 or 2, got {self.double_quant!r}")
        sizes, _ = qlora_nf4_sizes(self.d, self.k, self.blocksize, mode)
        dev = self.codes.device if device is None else torch.device(device)
        want = [("codes", self.codes, sizes[0], (torch.uint8,)),
                ("absmax", self.absmax, sizes[1], (torch.float32,)),
                ("c2", self.c2, sizes[2], (torch.uint8,) if mode == 2 else (torch.int8,)),
                ("c1", self.c1, sizes[3], (torch.float32,)),
                ("mean", self.mean, sizes[4], (torch.float32,))]
        for name, t, need, dtypes in want:
            if need == 0:
                continue
            if t is None:
                raise ValueError(f"NF4Weight.{name} is required for double_quant={mode}")
            if t.dtype not in dtypes:
                raise ValueError(f"NF4Weight.{name}: dtype {t.dtype}, expected {dtypes[0]}")
            if not t.is_contiguous():
                raise ValueError(f"NF4Weight.{name} must be contiguous")
            if t.device != dev:
                raise ValueError(f"NF4Weight.{name} is on {t.device}, the call runs on {dev}")
            if _nbytes(t) < need:
                raise ValueError(f"NF4Weight.{name}: {_nbytes(t)} bytes, a {self.d}x{self.k} weight needs {need}")
        return QloraNF4(self.d, self.k, self.blocksize, mode, _ptr(self.codes), _ptr(self.absmax),
                        _ptr(self.c2), _ptr(self.c1), _ptr(self.mean))

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.absmax, self.c2, self.c1, self.mean)
                   if t is not None)


def qlora_nf4_sizes(d: int, k: int, blocksize: int = 64, double_quant: bool = True):
    """(sizes of codes, absmax, c2, c1, mean in bytes, quantize workspace bytes)."""
    sizes = (ctypes.c_size_t * 5)()
    ws = ctypes.c_size_t()
    _check(lib().qlora_nf4_sizes(d, k, blocksize, int(double_quant), sizes, ctypes.byref(ws)))
    return list(sizes), ws.value


def nf4_alloc(d: int, k: int, double_quant: bool = True, device=None) -> NF4Weight:
    device = device or torch.device("cuda", torch.cuda.current_device())
    sizes, _ = qlora_nf4_sizes(d, k, 64, double_quant)

    def buf(n, dtype, esize):
        # 16 extra bytes of slack keep vector accesses inside the allocation
        return torch.empty(max(n // esize, 1) + 16 // esize, dtype=dtype, device=device)
    codes = buf(sizes[0], torch.uint8, 1)
    mode = int(double_quant)
    if mode:
        c2_dtype = torch.uint8 if mode == 2 else torch.int8   # E4M3 bytes / Int8
        return NF4Weight(d, k, mode, codes, None, buf(sizes[2], c2_dtype, 1), buf(sizes[3], torch.float32, 4),
                         buf(sizes[4], torch.float32, 4))
    return NF4Weight(d, k, 0, codes, buf(sizes[1], torch.float32, 4))


def nf4_quantize(W0: torch.Tensor, double_quant: bool = True, out: Optional[NF4Weight] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> NF4Weight:
    """Blockwise NF4 (+ double quantisation) of a bf16 (d, k) weight."""
    assert W0.dtype == torch.bfloat16 and W0.dim() == 2 and W0.is_contiguous()
    d, k = W0.shape
    q = out or nf4_alloc(d, k, double_quant, W0.device)
    if (q.d, q.k) != (d, k):
        raise ValueError(f"out describes a {q.d}x{q.k} weight, W0 is {d}x{k}")
    _, ws_bytes = qlora_nf4_sizes(d, k, 64, q.double_quant)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=W0.device)
    if workspace is not None and workspace.device != W0.device:
        raise ValueError(f"workspace is on {workspace.device}, W0 on {W0.device}")
    st = q.struct(W0.device)
    _check(lib().nf4_quantize(W0.data_ptr(), ctypes.byref(st), _ptr(workspace), _nbytes(workspace),
                              _stream(stream)))
    return q


NOALLOC_MAX_WEIGHTS = 1 << 28


def nf4_quantize_noalloc(W0: torch.Tensor, double_quant: bool = True, out: Optional[NF4Weight] = None,
                         stream=None) -> NF4Weight:
    """nf4_quantize without a workspace: for callers that cannot allocate device
    memory, the library uses its own fixed scratch (weights up to 2^28 elements).
    Only `out`'s buffers are the caller's; pass them pre-allocated to allocate
    nothing in this call."""
    assert W0.dtype == torch.bfloat16 and W0.dim() == 2 and W0.is_contiguous()
    d, k = W0.shape
    q = out or nf4_alloc(d, k, double_quant, W0.device)
    if (q.d, q.k) != (d, k):
        raise ValueError(f"out describes a {q.d}x{q.k} weight, W0 is {d}x{k}")
    if int(q.double_quant) != int(double_quant):
        raise ValueError(f"out holds double_quant={int(q.double_quant)} buffers, the call asks for {int(double_quant)}")
    st = q.struct(W0.device)
    _check(lib().nf4_quantize_noalloc(W0.data_ptr(), ctypes.byref(st), _stream(stream)))
    return q


def nf4_dequantize(q: NF4Weight, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """doubleDequant into a bf16 (d, k) tensor."""
    if out is None:
        out = torch.empty(q.d, q.k, dtype=torch.bfloat16, device=q.codes.device)
    _expect(out, "out", (q.d, q.k), torch.bfloat16)
    st = q.struct(out.device)
    _check(lib().nf4_dequantize(ctypes.byref(st), out.data_ptr(), _stream(stream)))
    return out


def qlora_lora_merge(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """W_merged = BF16(W^ + (alpha/r) B A) as a bf16 (d, k) tensor."""
    r = A.shape[0]
    if out is None:
        out = torch.empty(q.d, q.k, dtype=torch.bfloat16, device=q.codes.device)
    _expect(A, "A", (r, q.k), torch.bfloat16)
    _expect(B, "B", (q.d, r), torch.bfloat16)
    _expect(out, "out", (q.d, q.k), torch.bfloat16)
    _same_device(out.device, A=A, B=B)
    st = q.struct(out.device)
    _check(lib().qlora_lora_merge(ctypes.byref(st), A.data_ptr(), B.data_ptr(), r, float(alpha), out.data_ptr(),
                                  _stream(stream)))
    return out


# ---------------------------------------------------------------------------
# grouped projections (several weights that share their input X)
# ---------------------------------------------------------------------------
@dataclass
class NF4Group:
    """Stacked NF4 buffers of n projections that share X (layout of
    ``qlora_nf4_group_t``): `w` describes all rows together and `parts[i]` is
    the slice of projection i (quantise W_i into it with nf4_quantize)."""
    ds: tuple
    w: NF4Weight
    parts: list

    def struct(self, device=None) -> QloraNF4Group:
        n = len(self.ds)
        st = QloraNF4Group()
        st.n = n
        for i in range(MAX_GROUP):
            st.d[i] = int(self.ds[i]) if i < n else 0
        st.w = self.w.struct(device)
        if self.w.double_quant and _nbytes(self.w.mean) < 4 * n:
            raise ValueError(f"the group's mean buffer holds {_nbytes(self.w.mean)} bytes, {n} means need {4 * n}")
        return st


def nf4_alloc_group(ds, k: int, double_quant: bool = True, device=None) -> NF4Group:
    """Stacked buffers for projections of ds[i] x k rows (ds[i] % 256 == 0 for
    all but the last) and per-projection slice descriptors."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    ds = tuple(int(x) for x in ds)
    if not 1 <= len(ds) <= MAX_GROUP:
        raise ValueError(f"1..{MAX_GROUP} projections, got {len(ds)}")
    if any(x % 256 for x in ds[:-1]):
        raise ValueError("every projection but the last needs a multiple of 256 rows")
    mode = int(double_quant)
    per = [qlora_nf4_sizes(d, k, 64, mode)[0] for d in ds]
    tot = [sum(sz[j] for sz in per) for j in range(5)]

    def buf(nbytes, dtype, esize):
        return torch.empty(max(nbytes // esize, 1) + 16 // esize, dtype=dtype, device=device)
    codes = buf(tot[0], torch.uint8, 1)
    c2_dtype = torch.uint8 if mode == 2 else torch.int8
    absmax = buf(tot[1], torch.float32, 4) if not mode else None
    c2 = buf(tot[2], c2_dtype, 1) if mode else None
    c1 = buf(tot[3], torch.float32, 4) if mode else None
    mean = buf(4 * len(ds), torch.float32, 4) if mode else None
    w = NF4Weight(sum(ds), k, mode, codes, absmax, c2, c1, mean)
    parts, off = [], [0] * 5
    for i, (d, sz) in enumerate(zip(ds, per)):
        def sl(t, j, esize):
            return None if t is None else t[off[j] // esize: (off[j] + sz[j]) // esize]
        parts.append(NF4Weight(d, k, mode, sl(codes, 0, 1), sl(absmax, 1, 4), sl(c2, 2, 1), sl(c1, 3, 4),
                               None if mean is None else mean[i:i + 1]))
        off = [o + x for o, x in zip(off, sz)]
    return NF4Group(ds, w, parts)


def nf4_quantize_group(Ws, double_quant: bool = True, out: Optional[NF4Group] = None, stream=None) -> NF4Group:
    """Quantise each W_i (d_i x k bf16) on its own into the group's stacked buffers."""
    k = Ws[0].shape[1]
    g = out or nf4_alloc_group([W.shape[0] for W in Ws], k, double_quant, Ws[0].device)
    for W, part in zip(Ws, g.parts):
        nf4_quantize(W, double_quant=part.double_quant, out=part, stream=stream)
    return g


def qlora_grouped_workspace_size(M: int, g: NF4Group, r: int, backward: bool) -> int:
    n = ctypes.c_size_t()
    st = g.struct()
    _check(lib().qlora_grouped_workspace_size(M, ctypes.byref(st), r, int(backward), ctypes.byref(n)))
    return n.value


def qlora_linear_fwd_grouped(X: torch.Tensor, g: NF4Group, A: torch.Tensor, B: torch.Tensor, alpha: float,
                             r: Optional[int] = None, Y: Optional[torch.Tensor] = None,
                             T_save: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                             stream=None, save_T: bool = True):
    """Y = [Y_0 | Y_1 | ...], Y_i = X W_i^T + (alpha/r) (X A_i^T) B_i^T with
    A = stacked A_i ((n r) x k) and B = stacked B_i (sum d_i x r)."""
    n = len(g.ds)
    M, k = X.shape
    r = A.shape[0] // n if r is None else r
    dev = X.device
    dt = g.w.d
    if Y is None:
        Y = torch.empty(M, dt, dtype=torch.bfloat16, device=dev)
    if T_save is None and save_T:
        T_save = torch.empty(M, qlora_rank_pad(n * r), dtype=torch.bfloat16, device=dev)
    _expect(X, "X", (M, g.w.k), torch.bfloat16)
    _expect(A, "A", (n * r, g.w.k), torch.bfloat16)
    _expect(B, "B", (dt, r), torch.bfloat16)
    _expect(Y, "Y", (M, dt), torch.bfloat16)
    _expect(T_save, "T_save", (M, qlora_rank_pad(n * r)), torch.bfloat16, required=False)
    if workspace is None:
        nws = qlora_grouped_workspace_size(M, g, r, False)
        workspace = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev) if nws else None
    _same_device(dev, A=A, B=B, Y=Y, T_save=T_save, workspace=workspace)
    st = g.struct(dev)
    _check(lib().qlora_linear_fwd_grouped(X.data_ptr(), M, ctypes.byref(st), A.data_ptr(), B.data_ptr(), r,
                                          float(alpha), Y.data_ptr(), _ptr(T_save), _ptr(workspace),
                                          _nbytes(workspace), _stream(stream)))
    return Y, T_save


def qlora_linear_bwd_grouped(dY: torch.Tensor, X: torch.Tensor, g: NF4Group, A: torch.Tensor, B: torch.Tensor,
                             alpha: float, r: Optional[int] = None, T_save: Optional[torch.Tensor] = None,
                             dX: Optional[torch.Tensor] = None, dA: Optional[torch.Tensor] = None,
                             dB: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                             stream=None, need_dX: bool = True):
    """Backward of qlora_linear_fwd_grouped; returns (dX, dA stacked, dB stacked)."""
    n = len(g.ds)
    M = dY.shape[0]
    r = A.shape[0] // n if r is None else r
    dev = dY.device
    dt = g.w.d
    if dX is None and need_dX:
        dX = torch.empty(M, g.w.k, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(n * r, g.w.k, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(dt, r, dtype=torch.float32, device=dev)
    _expect(dY, "dY", (M, dt), torch.bfloat16)
    _expect(X, "X", (M, g.w.k), torch.bfloat16)
    _expect(A, "A", (n * r, g.w.k), torch.bfloat16)
    _expect(B, "B", (dt, r), torch.bfloat16)
    _expect(T_save, "T_save", (M, qlora_rank_pad(n * r)), torch.bfloat16, required=False)
    _expect(dX, "dX", (M, g.w.k), torch.bfloat16, required=False)
    _expect(dA, "dA", (n * r, g.w.k), torch.float32)
    _expect(dB, "dB", (dt, r), torch.float32)
    if workspace is None:
        nws = qlora_grouped_workspace_size(M, g, r, True)
        workspace = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev) if nws else None
    _same_device(dev, X=X, A=A, B=B, T_save=T_save, dX=dX, dA=dA, dB=dB, workspace=workspace)
    st = g.struct(dev)
    _check(lib().qlora_linear_bwd_grouped(_ptr(dY), _ptr(X), M, ctypes.byref(st), A.data_ptr(), B.data_ptr(), r,
                                          float(alpha), _ptr(T_save), _ptr(dX), dA.data_ptr(), dB.data_ptr(),
                                          _ptr(workspace), _nbytes(workspace), _stream(stream)))
    return dX, dA, dB


def qlora_rank_pad(r: int) -> int:
    return int(lib().qlora_rank_pad(r))


def qlora_linear_workspace_size(M: int, d: int, k: int, r: int, backward: bool) -> int:
    n = ctypes.c_size_t()
    _check(lib().qlora_linear_workspace_size(M, d, k, r, int(backward), ctypes.byref(n)))
    return n.value


def _dropout_struct(dropout) -> Optional[QloraDropout]:
    """(p, seed, offset) -> qlora_dropout_t, or None for no dropout."""
    if dropout is None:
        return None
    p, seed, offset = dropout
    if not (0.0 <= float(p) < 1.0):
        raise ValueError(f"dropout probability {p} outside [0, 1)")
    return QloraDropout(float(p), int(seed) & (2 ** 64 - 1), int(offset) & (2 ** 64 - 1))


def qlora_linear_dropout_workspace_size(M: int, d: int, k: int, r: int, backward: bool) -> int:
    n = ctypes.c_size_t()
    _check(lib().qlora_linear_dropout_workspace_size(M, d, k, r, int(backward), ctypes.byref(n)))
    return n.value


def qlora_dropout_mask(M: int, k: int, p: float, seed: int, offset: int = 0, out: Optional[torch.Tensor] = None,
                       device=None, stream=None) -> torch.Tensor:
    """Keep bitmask of an M x k activation as int32 words (bit b of word w is
    flat element 32 w + b; 1 = kept)."""
    nw = (M * k + 31) // 32
    if out is None:
        device = device or torch.device("cuda", torch.cuda.current_device())
        out = torch.empty(max(nw, 1), dtype=torch.int32, device=device)
    if out.dtype != torch.int32 or out.numel() < nw or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous int32 tensor of at least {nw} words")
    st = _dropout_struct((p, seed, offset))
    _check(lib().qlora_dropout_mask(M, k, ctypes.byref(st), out.data_ptr() if nw else None, _stream(stream)))
    return out


def qlora_linear_fwd_dropout(X: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                             dropout, **kw):
    """qlora_linear_fwd with adapter dropout; dropout = (p, seed, offset)."""
    return qlora_linear_fwd(X, q, A, B, alpha, dropout=dropout, **kw)


def qlora_linear_bwd_dropout(dY: torch.Tensor, X: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                             alpha: float, dropout, **kw):
    """qlora_linear_bwd for the dropout forward with the same (p, seed, offset)."""
    return qlora_linear_bwd(dY, X, q, A, B, alpha, dropout=dropout, **kw)


def qlora_linear_fwd(X: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     Y: Optional[torch.Tensor] = None, T_save: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None, save_T: bool = True, dropout=None):
    """Y = X W^T + (alpha/r) (X A^T) B^T.  Returns (Y, T_save).  With
    dropout = (p, seed, offset) the adapter sees drop(X) instead of X."""
    M, k = X.shape
    r = A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty(M, q.d, dtype=torch.bfloat16, device=dev)
    if T_save is None and save_T:
        T_save = torch.empty(M, qlora_rank_pad(r), dtype=torch.bfloat16, device=dev)
    _expect(X, "X", (M, q.k), torch.bfloat16)
    _expect(A, "A", (r, q.k), torch.bfloat16)
    _expect(B, "B", (q.d, r), torch.bfloat16)
    _expect(Y, "Y", (M, q.d), torch.bfloat16)
    _expect(T_save, "T_save", (M, qlora_rank_pad(r)), torch.bfloat16, required=False)
    drop = _dropout_struct(dropout)
    if workspace is None:
        n = (qlora_linear_dropout_workspace_size(M, q.d, q.k, r, False) if drop is not None
             else qlora_linear_workspace_size(M, q.d, q.k, r, False))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=dev) if n else None
    _same_device(dev, A=A, B=B, Y=Y, T_save=T_save, workspace=workspace)
    st = q.struct(dev)
    if drop is None:
        _check(lib().qlora_linear_fwd(X.data_ptr(), M, ctypes.byref(st), A.data_ptr(), B.data_ptr(), r, float(alpha),
                                      Y.data_ptr(), _ptr(T_save), _ptr(workspace), _nbytes(workspace),
                                      _stream(stream)))
    else:
        _check(lib().qlora_linear_fwd_dropout(X.data_ptr(), M, ctypes.byref(st), A.data_ptr(), B.data_ptr(), r,
                                              float(alpha), ctypes.byref(drop), Y.data_ptr(), _ptr(T_save),
                                              _ptr(workspace), _nbytes(workspace), _stream(stream)))
    return Y, T_save


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                     alpha: float, T_save: Optional[torch.Tensor] = None, dX: Optional[torch.Tensor] = None,
                     dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None, need_dX: bool = True, dropout=None):
    """Gradients for the adapters and the input; returns (dX, dA, dB).  With
    dropout = (p, seed, offset), the backward of the dropout forward."""
    M = dY.shape[0]
    r = A.shape[0]
    dev = dY.device
    if dX is None and need_dX:
        dX = torch.empty(M, q.k, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(r, q.k, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(q.d, r, dtype=torch.float32, device=dev)
    _expect(dY, "dY", (M, q.d), torch.bfloat16)
    _expect(X, "X", (M, q.k), torch.bfloat16)
    _expect(A, "A", (r, q.k), torch.bfloat16)
    _expect(B, "B", (q.d, r), torch.bfloat16)
    _expect(T_save, "T_save", (M, qlora_rank_pad(r)), torch.bfloat16, required=False)
    _expect(dX, "dX", (M, q.k), torch.bfloat16, required=False)
    _expect(dA, "dA", (r, q.k), torch.float32)
    _expect(dB, "dB", (q.d, r), torch.float32)
    drop = _dropout_struct(dropout)
    if workspace is None:
        n = (qlora_linear_dropout_workspace_size(M, q.d, q.k, r, True) if drop is not None
             else qlora_linear_workspace_size(M, q.d, q.k, r, True))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=dev) if n else None
    _same_device(dev, X=X, A=A, B=B, T_save=T_save, dX=dX, dA=dA, dB=dB, workspace=workspace)
    st = q.struct(dev)
    if drop is None:
        _check(lib().qlora_linear_bwd(_ptr(dY), _ptr(X), M, ctypes.byref(st), A.data_ptr(), B.data_ptr(), r,
                                      float(alpha), _ptr(T_save), _ptr(dX), dA.data_ptr(), dB.data_ptr(),
                                      _ptr(workspace), _nbytes(workspace), _stream(stream)))
    else:
        _check(lib().qlora_linear_bwd_dropout(_ptr(dY), _ptr(X), M, ctypes.byref(st), A.data_ptr(), B.data_ptr(),
                                              r, float(alpha), ctypes.byref(drop), _ptr(T_save), _ptr(dX),
                                              dA.data_ptr(), dB.data_ptr(), _ptr(workspace), _nbytes(workspace),
                                              _stream(stream)))
    return dX, dA, dB


def qlora_nf4_codebook():
    buf = (ctypes.c_float * 16)()
    _check(lib().qlora_nf4_codebook(buf))
    return list(buf)


def qlora_device_status(stream=None) -> int:
    """Synchronize and return (and clear) the device status word; 0 = clean."""
    s = ctypes.c_int32()
    rc = lib().qlora_device_status(_stream(stream), ctypes.byref(s))
    if rc not in (QLORA_OK, -6):
        _check(rc)
    return s.value


def qlora_selftest_wait_timeout(limit_us: int = 1000, stream=None) -> int:
    """Run the bounded-wait self-test (a wait nothing ends, given up after
    limit_us); returns the kernel's result word (2: gave up and released its
    TMEM).  The status word then holds code 7 until qlora_device_status()."""
    res = torch.zeros(1, dtype=torch.int32, device=torch.device("cuda", torch.cuda.current_device()))
    _check(lib().qlora_selftest_wait_timeout(int(limit_us), res.data_ptr(), _stream(stream)))
    return int(res.item())


def qlora_profile_enable(on: bool = True) -> None:
    _check(lib().qlora_profile_enable(int(on)))


def qlora_profile_read():
    """Returns ({class: device ms}, {class: launches}) since the last read."""
    ms = (ctypes.c_double * len(KERNEL_CLASSES))()
    n = (ctypes.c_int64 * len(KERNEL_CLASSES))()
    _check(lib().qlora_profile_read(ms, n))
    return dict(zip(KERNEL_CLASSES, list(ms))), dict(zip(KERNEL_CLASSES, list(n)))
