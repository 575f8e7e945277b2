"""Seeded synthetic inputs and the named workload shapes.

This module is shared by the GPU library's tests and benchmark and by the
float64 oracle's tests.  It holds no attention arithmetic: it only draws
iid N(0, 1) values from NumPy's ``default_rng(seed)`` in float32 and rounds
them to bfloat16 (round to nearest even, as ``torch.Tensor.to`` does).
The oracle is fed the same bfloat16 values widened to float64, so a
comparison measures kernel arithmetic, not input quantisation.

Seeds: q = 0, k = 1, v = 2, dO = 3 (plus ``seed_offset``).

The workloads stand in for the data the Sparse Transformer pages model
(CIFAR-10 32x32x3 images, Enwik8 bytes, ImageNet 64x64x3 images and
~65,000-sample classical-music audio); there is no dataset here, only
random tensors of those sequence shapes.
"""

import numpy as np

# name -> pattern, B, H, N, D, l, c, block
WORKLOADS = {
    # strided, one head, tiny: exercised against the oracle element by element
    "tiny-strided": dict(mode="strided", B=1, H=1, N=256, D=32, l=16, c=0, block=16),
    # 32x32x3 image bytes, one image row = 96 positions
    "image32-strided": dict(mode="strided", B=4, H=2, N=3072, D=128, l=96, c=0, block=32),
    # byte-level text, fixed pattern with 32 summary columns per 128-block
    "text-fixed": dict(mode="fixed", B=2, H=8, N=12288, D=64, l=128, c=32, block=64),
    # 64x64x3 image bytes, one image row = 192 positions
    "image64-strided": dict(mode="strided", B=1, H=16, N=12288, D=64, l=192, c=0, block=64),
    # same shape, dense causal, for comparison
    "image64-all": dict(mode="all", B=1, H=16, N=12288, D=64, l=192, c=0, block=64),
    # raw audio, 65536 samples
    "audio-strided": dict(mode="strided", B=1, H=4, N=65536, D=64, l=256, c=0, block=64),
    # the image64 strided pattern in its two-head form: row head and column head
    "image64-local": dict(mode="local", B=1, H=16, N=12288, D=64, l=192, c=0, block=64),
    "image64-column": dict(mode="column", B=1, H=16, N=12288, D=64, l=192, c=0, block=64),
    # longer sequences, the strided pattern with l = sqrt(N): 2^18 and 2^20 positions
    "long-strided-262144": dict(mode="strided", B=1, H=4, N=1 << 18, D=64, l=512, c=0, block=64),
    "long-strided-1048576": dict(mode="strided", B=1, H=4, N=1 << 20, D=64, l=1024, c=0, block=64),
}


def normal_f32(shape, seed):
    """iid N(0, 1) float32 array from ``default_rng(seed)``."""
    return np.random.default_rng(seed).standard_normal(tuple(shape), dtype=np.float32)


def normal_bf16(shape, seed):
    """The same draw rounded to bfloat16, as a CPU ``torch.Tensor``."""
    import torch

    return torch.from_numpy(normal_f32(shape, seed)).to(torch.bfloat16)


def inputs(B, H, N, D, seed_offset=0):
    """q, k, v, dO as CPU bfloat16 tensors of shape ``[B, H, N, D]``."""
    shape = (B, H, N, D)
    return {name: normal_bf16(shape, seed + seed_offset)
            for name, seed in (("q", 0), ("k", 1), ("v", 2), ("dO", 3))}


def to_f64(t):
    """bfloat16 (or any) CPU tensor -> float64 NumPy array, exactly."""
    return t.detach().to("cpu").double().numpy()


# Inputs of the Sparse Transformer block around the op (model width C = H * D,
# hidden width 4C).  Projections are drawn N(0, 1) and scaled by 1/sqrt(fan
# in), then rounded to bfloat16; the layer-norm gains are 1 + 0.1 N(0, 1) and
# the biases 0.1 N(0, 1) in float32 (so the affine part is exercised).
BLOCK_WEIGHTS = (("w_qkv", 1, 3), ("w_o", 1, 1), ("w_1", 1, 4), ("w_2", 4, 1))  # name, rows / C, cols / C


def block_inputs(B, N, C, seed_offset=0):
    """x and the upstream gradient dy as CPU bfloat16 ``[B, N, C]`` tensors."""
    return {"x": normal_bf16((B, N, C), 10 + seed_offset), "dy": normal_bf16((B, N, C), 11 + seed_offset)}


def block_params(C, seed=20):
    """The block's parameters as CPU tensors: bfloat16 projections (``[in, out]``
    row-major) and float32 layer-norm gains and biases."""
    import torch

    p = {}
    for i, (name, r, c) in enumerate(BLOCK_WEIGHTS):
        w = normal_f32((r * C, c * C), seed + i) / np.float32(np.sqrt(r * C))
        p[name] = torch.from_numpy(w).to(torch.bfloat16)
    for i, name in enumerate(("ln1", "ln2")):
        p[name + "_g"] = torch.from_numpy(1.0 + 0.1 * normal_f32((C,), seed + 10 + 2 * i))
        p[name + "_b"] = torch.from_numpy(0.1 * normal_f32((C,), seed + 11 + 2 * i))
    return p
