"""Device-buffer helpers for the GPU parity tests (torch supplies memory only)."""
import numpy as np

CANARY = 0x7FC0BEEF  # a NaN bit pattern no kernel writes


def torch():
    import torch as t
    return t


def dev(a: np.ndarray):
    """Copy a numpy array to a new device tensor (same dtype, 256-B aligned)."""
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a)).cuda()


def guarded_f32(n: int, guard: int = 64):
    """fp32 device buffer of n elements inside canary guard bands.
    Returns (full tensor, offset of element 0); the body starts 256-B aligned."""
    t = torch()
    buf = t.full((n + 2 * guard,), CANARY, dtype=t.int32, device="cuda")
    return buf, guard


def body(buf, off, n):
    return buf[off:off + n].view(torch().float32)


def check_guards(buf, off, n):
    h = buf.cpu().numpy().view(np.uint32)
    assert np.all(h[:off] == CANARY), "write below the output buffer"
    assert np.all(h[off + n:] == CANARY), "write past the end of the output buffer"


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
