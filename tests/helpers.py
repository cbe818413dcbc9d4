"""Shared test utilities: bf16 bit conversions between numpy and torch, tolerance checks."""
import numpy as np

# Float parity bar: |gpu - ref| <= RTOL * (|ref| + rms(ref)) element by element, i.e. a
# relative error of 2e-2 with a floor at the tensor's RMS so that entries near zero are
# compared on the tensor's scale.  bf16 path: 2e-2; NVFP4 path: 6e-2.
RTOL_BF16 = 2e-2
RTOL_NVFP4 = 6e-2


def to_torch_bf16(bits, device="cuda"):
    import torch
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def from_torch_bf16(t):
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_f64(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref) + np.sqrt(np.mean(ref ** 2)) + 1e-30
    return float(np.max(np.abs(got - ref) / scale))


def assert_close(got, ref, rtol=RTOL_BF16, what=""):
    e = rel_err(got, ref)
    assert e <= rtol, "%s: relative error %.3e > %.1e" % (what, e, rtol)
    return e


def unambiguous_argmax(logits, gap=1e-3):
    """Mask of rows whose top-2 logit gap is at least `gap`."""
    l = np.sort(np.asarray(logits, np.float64), axis=1)
    return (l[:, -1] - l[:, -2]) >= gap
