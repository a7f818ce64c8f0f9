"""Helpers for the GPU parity tests: moving tensors between torch (device) and
the oracle's numpy arrays (raw 16-bit patterns)."""
import numpy as np
import torch

from group_wise_affine_quant_b200.inputs import as_u16

DEV = "cuda:0"
TDT = {0: torch.float16, 1: torch.bfloat16}


def to_dev(t):
    return t.to(DEV).contiguous()


def dev_u16(t):
    """Device fp16/bf16 tensor -> numpy uint16 patterns."""
    return as_u16(t.detach().cpu())


def dev_u8(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def u16_to_dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(TDT[dt]).to(DEV)


def canon_nan(a, dt):
    """Map every NaN pattern of T to one value (a NaN has no unique encoding)."""
    a = np.array(a, dtype=np.uint16, copy=True)
    exp = 0x7C00 if dt == 0 else 0x7F80
    frac = 0x03FF if dt == 0 else 0x007F
    nan = ((a & exp) == exp) & ((a & frac) != 0)
    a[nan] = 0x7FFF
    return a


def assert_equal_bits(got, want, what, nan_dt=None):
    got = np.asarray(got)
    want = np.asarray(want)
    if nan_dt is not None:
        got, want = canon_nan(got, nan_dt), canon_nan(want, nan_dt)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError("%s: %d of %d differ; first at %s: got %r want %r"
                             % (what, len(bad), got.size, i, got[i], want[i]))
