"""Seeded synthetic inputs for the five workloads (no quantization arithmetic).

The pages' workloads (MoE activations and expert weights of the models they
train) are not available; these generators stand in for them with the shapes
and value distributions the workloads are described with.  Every generator is
deterministic in its seed.  BF16 values are made from FP32 by
round-to-nearest-even (torch's cast) and are returned as uint16 bit patterns.

Rollout copies model the train/rollout numerical wobble of the TRACE explainer
(blog.ontle.kr/blog/286, rounding-analogy paragraph): rollout = bf16(x * (1 + eps)),
eps ~ N(0, (2^-8)^2) i.i.d., with x the train tensor's BF16 value.

Host generators use numpy ``Generator(PCG64)``; per-layer streams come from
``SeedSequence(seed).spawn``.  The 48-layer throughput stack is generated on
the GPU with a seeded torch generator (12.9 G elements per copy).
"""
from __future__ import annotations

import math

import numpy as np
import torch

ROLLOUT_REL_STD = 2.0 ** -8

# Workload shapes.
CFG0_SHAPE = (1024, 2048)
CFG1_LAYERS, CFG1_SHAPE, CFG1_HINT_FROM = 24, (8192, 2048), 12
CFG2_SHAPE = (128, 512, 2048)
CFG3_SHAPE = (16384, 4096)
CFG3_OUTLIERS = 67109            # 0.1% of 16384 * 4096, rounded
CFG4_LAYERS, CFG4_SHAPE, CFG4_HINT_FROM = 48, (65536, 4096), 24


def bf16_bits(a) -> np.ndarray:
    """FP32 array -> BF16 bit patterns (uint16) by round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def rollout_copy(x_bf16, rng: np.random.Generator, rel_std: float = ROLLOUT_REL_STD) -> np.ndarray:
    x = bf16_to_f32(x_bf16)
    eps = rng.standard_normal(x.shape, dtype=np.float32) * np.float32(rel_std)
    return bf16_bits(x * (np.float32(1.0) + eps))


def normal_pair(shape, seed: int, std: float = 1.0):
    """(train, rollout) BF16 pair, train ~ N(0, std^2)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))
    return x, rollout_copy(x, rng)


def cfg0():
    """Single 1024x2048 tensor, N(0,1), seed 0 -> (train, rollout)."""
    return normal_pair(CFG0_SHAPE, 0)


def cfg1_layer(layer: int):
    """MoE activation layer: 8192x2048 Student-t (nu=4), 16 random outlier
    channels x50 per layer; layer streams spawned from seed 1."""
    ss = np.random.SeedSequence(1).spawn(CFG1_LAYERS)[layer]
    rng = np.random.Generator(np.random.PCG64(ss))
    rows, cols = CFG1_SHAPE
    x = rng.standard_t(4.0, size=(rows, cols)).astype(np.float32)
    ch = rng.choice(cols, size=16, replace=False)
    x[:, ch] *= np.float32(50.0)
    xb = bf16_bits(x)
    return xb, rollout_copy(xb, rng)


def cfg2():
    """Expert weight stack 128 x 512 x 2048, N(0, 0.02^2), seed 2 (BF16)."""
    rng = np.random.Generator(np.random.PCG64(2))
    w = rng.standard_normal(CFG2_SHAPE, dtype=np.float32) * np.float32(0.02)
    return bf16_bits(w)


def cfg3():
    """Activation 16384x4096, N(0,1) with 0.1% of positions x100, seed 3."""
    rng = np.random.Generator(np.random.PCG64(3))
    x = rng.standard_normal(CFG3_SHAPE, dtype=np.float32)
    flat = x.reshape(-1)
    pos = rng.choice(flat.size, size=CFG3_OUTLIERS, replace=False)
    flat[pos] *= np.float32(100.0)
    return bf16_bits(x)


CFG3_SIGN_SEED = 3
CFG2_SR_SEED = 2


def random_case(shape, seed: int, kind: str = "normal") -> np.ndarray:
    """Small edge-case inputs: 'normal', 'tiny' (subnormal block scales),
    'outlier' (one huge value), 'zeros', 'ties' (values near grid midpoints),
    'heavy' (Student-t nu=2), 'sparse' (half exact zeros, BF16 subnormals)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if kind == "normal":
        x = rng.standard_normal(shape, dtype=np.float32)
    elif kind == "tiny":
        x = rng.standard_normal(shape, dtype=np.float32)
        x.reshape(-1)[rng.integers(0, x.size)] = 1.0e4  # makes most block scales tiny
        x *= np.float32(1.0e-3)
    elif kind == "outlier":
        x = rng.standard_normal(shape, dtype=np.float32)
        x.reshape(-1)[rng.integers(0, x.size)] = 3.0e5
    elif kind == "zeros":
        x = np.zeros(shape, np.float32)
        x.reshape(-1)[::7] = -0.0
    elif kind == "ties":
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 3.0], np.float32)
        x = rng.choice(mids, size=shape) * rng.choice(np.array([-1, 1], np.float32), size=shape)
        x.reshape(-1)[::16] = 6.0  # block max 6 -> scale close to 1 so ties survive
    elif kind == "heavy":
        x = rng.standard_t(2.0, size=shape).astype(np.float32)
    elif kind == "sparse":
        # half exact zeros (some -0), BF16 subnormals, normal values, one outlier
        x = rng.standard_normal(shape, dtype=np.float32)
        flat = x.reshape(-1)
        u = rng.random(flat.size)
        flat[u < 0.5] = 0.0
        flat[(u >= 0.5) & (u < 0.55)] = -0.0
        sub = (u >= 0.55) & (u < 0.65)
        bits = bf16_bits(x).reshape(-1)
        bits[sub] = rng.integers(1, 0x80, int(sub.sum())).astype(np.uint16) | \
            (rng.integers(0, 2, int(sub.sum())).astype(np.uint16) << 15)
        bits[rng.integers(0, bits.size)] = bf16_bits(np.float32([4.0e5]))[0]
        return bits.reshape(shape)
    else:
        raise ValueError(kind)
    return bf16_bits(x)


# --------------------------------------------------------------------------- device
def cfg4_layer_device(layer: int, device, rank: int = 0, shape=CFG4_SHAPE):
    """48-layer throughput stack, one layer on the GPU: 65536x4096, N(0,1) times
    per-column scales c_j = exp(U(ln 0.1, ln 10)); seed 4, layer and rank mixed
    into the generator seed (every rank of a multi-GPU run gets its own stack).
    Returns (train, rollout) as torch.bfloat16 on ``device``."""
    rows, cols = shape
    g = torch.Generator(device=device)
    g.manual_seed((4 << 40) | (rank << 20) | layer)
    c = torch.empty(cols, device=device, dtype=torch.float32)
    c.uniform_(math.log(0.1), math.log(10.0), generator=g)
    c.exp_()
    x = torch.randn(rows, cols, device=device, dtype=torch.float32, generator=g)
    x.mul_(c)
    xb = x.to(torch.bfloat16)
    del x
    eps = torch.randn(rows, cols, device=device, dtype=torch.float32, generator=g)
    eps.mul_(ROLLOUT_REL_STD).add_(1.0)
    eps.mul_(xb.float())
    rb = eps.to(torch.bfloat16)
    del eps
    return xb, rb


def cfg1_layer_device(layer: int, device, rank: int = 0, shape=CFG1_SHAPE):
    """MoE activation layer generated on the GPU, for timing: Student-t with
    nu = 4 as z / sqrt(chi2_4 / 4) (z and the four squared normals of chi2_4
    independent N(0, 1)), 16 random outlier channels x50, rollout copy as
    everywhere.  Same distribution as cfg1_layer, not the same numbers (the
    parity tests use cfg1_layer).  Returns (train, rollout) torch.bfloat16."""
    rows, cols = shape
    g = torch.Generator(device=device)
    g.manual_seed((1 << 40) | (rank << 20) | layer)
    chi2 = torch.zeros(rows, cols, device=device, dtype=torch.float32)
    for _ in range(4):
        z = torch.randn(rows, cols, device=device, dtype=torch.float32, generator=g)
        chi2.addcmul_(z, z)
    x = torch.randn(rows, cols, device=device, dtype=torch.float32, generator=g)
    x.div_(chi2.div_(4.0).sqrt_())
    del chi2
    ch = torch.randperm(cols, device=device, generator=g)[:16]
    x[:, ch] *= 50.0
    xb = x.to(torch.bfloat16)
    eps = torch.randn(rows, cols, device=device, dtype=torch.float32, generator=g)
    eps.mul_(ROLLOUT_REL_STD).add_(1.0)
    eps.mul_(xb.float())
    return xb, eps.to(torch.bfloat16)
