"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

from oracle import qlora_oracle as O

REL_FRO = 1e-2      # relative Frobenius error bound for Y, dX, dA, dB
MAX_ABS = 2e-2      # element max-abs bound, as a fraction of max |ref|


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16)
    return t.cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return O.bf16_bits_to_f32(host_bits(t))
    return t.float().cpu().numpy()


def assert_close(got: np.ndarray, ref: np.ndarray, what: str):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    den = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / den if den > 0 else np.linalg.norm(got)
    mx = np.max(np.abs(got - ref)) if got.size else 0.0
    lim = MAX_ABS * (np.max(np.abs(ref)) if ref.size else 0.0)
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e}"
    assert mx <= lim + 1e-30, f"{what}: max abs error {mx:.3e} > {lim:.3e}"
    return rel, mx


def gpu_quantized_arrays(q, n):
    """Copy a quantized weight back: packed bytes and constants as numpy."""
    nb = (n + 1) // 2
    nblk = -(-n // 64)
    out = {"packed": q.codes[:nb].cpu().numpy()}
    if q.double_quant:
        out["c2"] = q.c2[:nblk].cpu().numpy()
        out["c1"] = q.c1[:-(-nblk // 256)].cpu().numpy()
        out["mean"] = q.mean[:1].cpu().numpy()
    else:
        out["absmax"] = q.absmax[:nblk].cpu().numpy()
    return out
