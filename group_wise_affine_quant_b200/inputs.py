"""Seeded synthetic inputs for the five workloads.

This module draws random numbers and nothing else: it holds none of the
quantizer's, dequantizer's or matmul's arithmetic.  The tests, the benchmark
and the smoke check feed the same tensors to the CUDA library and to the CPU
oracle.  Everything is generated on the host with a seeded
``torch.Generator`` in fp32 and then rounded to the activation dtype.

Distributions (``N(0, v)`` is read as variance ``v`` where the workload
writes a fan-in fraction, and as standard deviation where it writes 0.02):

* tiny qmv/qmm (fp16): x ~ N(0, 1) [M, 512], W ~ N(0, 1/512) [512, 512], seed 0
* decode sweep (bf16): Llama-3.2-1B-like projections, W ~ N(0, 0.02^2),
  x ~ N(0, 1)
* chained qmm (fp16): x ~ N(0, 1) [1024, 1024], W1 [4096, 1024] and
  W2 [1024, 4096] ~ N(0, 1), seed 3
* conv2d (bf16): x ~ N(0, 1) [2, 64, 64, 320], W ~ N(0, 1/2880)
  [320, 3, 3, 320/groups]
* FP4 (bf16): E2M1 code bytes uniform over 0..255 (both nibbles uniform),
  E8M0 scales uniform over 0..254 ("literal") or 117..137 ("finite"), E4M3
  scales uniform over 0x00..0x7E, x ~ N(0, 1)
"""
import torch

F16, BF16 = 0, 1
TORCH_DTYPE = {F16: torch.float16, BF16: torch.bfloat16}

# Llama-3.2-1B-like layer: (name, N, K) for y = x . W^T with W [N, K].
LLAMA_1B_PROJ = (
    ("q", 2048, 2048), ("k", 512, 2048), ("v", 512, 2048), ("o", 2048, 2048),
    ("gate", 8192, 2048), ("up", 8192, 2048), ("down", 2048, 8192),
)
DECODE_M = (1, 2, 4, 8, 16, 32, 64)


def gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def normal(shape, std, dt, g):
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(TORCH_DTYPE[dt])


def as_u16(t: torch.Tensor):
    """Raw 16-bit patterns of an fp16/bf16 tensor as a numpy uint16 array."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def tiny(M, seed=0):
    g = gen(seed)
    w = normal((512, 512), 512 ** -0.5, F16, g)
    x = normal((M, 512), 1.0, F16, g)
    return x, w


def decode_layer(seed=0, dt=BF16):
    """Weights of one Llama-3.2-1B-shaped layer: dict name -> W [N, K]."""
    g = gen(seed)
    return {name: normal((n, k), 0.02, dt, g) for name, n, k in LLAMA_1B_PROJ}


def decode_x(M, K, seed=1, dt=BF16):
    return normal((M, K), 1.0, dt, gen(seed))


def chained(seed=3):
    g = gen(seed)
    x = normal((1024, 1024), 1.0, F16, g)
    w1 = normal((4096, 1024), 1.0, F16, g)
    w2 = normal((1024, 4096), 1.0, F16, g)
    return x, w1, w2


def conv(groups, seed=0, B=2, H=64, W=64, C=320, Cout=320, kh=3, kw=3, dt=BF16):
    g = gen(seed)
    x = normal((B, H, W, C), 1.0, dt, g)
    w = normal((Cout, kh, kw, C // groups), (kh * kw * C) ** -0.5, dt, g)
    return x, w


def flatten_pad_conv_weight(w, group_size):
    """[Cout, kh, kw, Cg] -> [Cout, Kp]: flatten (kh, kw, Cg), zero-pad to a
    multiple of group_size (the layout the quantized conv consumes)."""
    cout = w.shape[0]
    w2 = w.reshape(cout, -1)
    k = w2.shape[1]
    kp = (k + group_size - 1) // group_size * group_size
    if kp != k:
        w2 = torch.cat([w2, torch.zeros(cout, kp - k, dtype=w2.dtype)], dim=1)
    return w2.contiguous()


def fp4(N, K, group_size, scale_range="finite", seed=0):
    """FP4 weights: codes [N, K/2] uint8, scales [N, K/group_size] uint8."""
    g = gen(seed)
    codes = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    G = K // group_size
    if group_size == 32:
        lo, hi = (0, 254) if scale_range == "literal" else (117, 137)
    else:
        lo, hi = (0x00, 0x7E) if scale_range == "literal" else (0x30, 0x48)
    scales = torch.randint(lo, hi + 1, (N, G), generator=g, dtype=torch.int32).to(torch.uint8)
    return codes, scales


def fp4_x(M, K, seed=1, dt=BF16):
    return normal((M, K), 1.0, dt, gen(seed))
