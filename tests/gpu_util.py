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


def assert_equal_bits(got, want, what):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError("%s: %d of %d differ; first at %s: got %r want %r"
                             % (what, len(bad), got.size, i, got[i], want[i]))
