"""Seeded synthetic inputs for tests and the benchmark.

This module only draws random numbers and describes workload shapes; it holds
none of the shard step's arithmetic.  Both the CUDA path and the CPU oracle are
fed from here, and nothing here depends on either.

Recipe (the pages measure no dataset, so every input is synthetic):
  * gradient contributions: N(0, std) * loss_scale per rank, rounded to fp16
    (std = 1e-3 in every workload);
  * fp32 master weights: N(0, 0.02); momentum and variance start at zero
    unless a test asks for random state;
  * pads of the rank buffers (flat positions >= Psi) hold a fill value that the
    step must never read (NaN in the tests).
Host draws use ``torch.Generator`` on the CPU; large device-resident buffers
are drawn on the GPU in fixed-size chunks with a per-chunk seed, so the values
at a given position depend only on (seed, position), never on the chunking of
a particular run.
"""
from __future__ import annotations

import numpy as np
import torch

# chunk of the device-side generator (elements); part of the recipe, since a
# position's value is drawn from the chunk that contains it
DEVICE_CHUNK = 1 << 24


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal_f32(n: int, seed: int, std: float, mean: float = 0.0) -> np.ndarray:
    """n fp32 samples of N(mean, std) drawn on the host."""
    x = torch.randn(int(n), generator=_gen(seed), dtype=torch.float32)
    return (x * std + mean).numpy()


def grads_f16(nd: int, n: int, seed: int, std: float = 1e-3, scale: float = 1.0,
              stride: int | None = None, pad_fill: float = float("nan")) -> np.ndarray:
    """Nd rank buffers of fp16 gradient contributions as uint16 bits [nd, stride].

    Rank r's first n entries are N(0, std) * scale rounded to fp16 (seed + r);
    entries n..stride-1 (the pad) are ``pad_fill``.
    """
    stride = n if stride is None else stride
    assert stride >= n
    out = np.empty((nd, stride), dtype=np.float16)
    for r in range(nd):
        x = torch.randn(int(n), generator=_gen(seed * 1000003 + r), dtype=torch.float32)
        out[r, :n] = (x * (std * scale)).to(torch.float16).numpy()
        out[r, n:] = pad_fill
    return out.view(np.uint16)


def grads_bf16(nd: int, n: int, seed: int, std: float = 1e-3, scale: float = 1.0,
               stride: int | None = None, pad_fill: float = float("nan")) -> np.ndarray:
    """As ``grads_f16`` (same draws), rounded to bfloat16 instead: uint16 bits [nd, stride]."""
    stride = n if stride is None else stride
    assert stride >= n
    out = torch.empty((nd, stride), dtype=torch.bfloat16)
    for r in range(nd):
        x = torch.randn(int(n), generator=_gen(seed * 1000003 + r), dtype=torch.float32)
        out[r, :n] = (x * (std * scale)).to(torch.bfloat16)
        out[r, n:] = pad_fill
    return out.view(torch.int16).numpy().view(np.uint16)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bfloat16 bit patterns via torch's round-to-nearest-even cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def fp16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> fp16 bit patterns via numpy's round-to-nearest-even cast."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


# --------------------------------------------------------------------------
# device-side draws for buffers too large to draw on the host
# --------------------------------------------------------------------------

def fill_normal_(t: torch.Tensor, seed: int, std: float, scale: float = 1.0) -> torch.Tensor:
    """Fill a 1-D CUDA tensor (fp16 or fp32) with N(0, std) * scale, chunk by chunk."""
    assert t.dim() == 1 and t.is_cuda
    n = t.numel()
    for c, start in enumerate(range(0, n, DEVICE_CHUNK)):
        stop = min(n, start + DEVICE_CHUNK)
        x = torch.randn(stop - start, generator=_gen(seed * 7919 + c, "cuda"),
                        dtype=torch.float32, device=t.device)
        x.mul_(std * scale)
        t[start:stop].copy_(x)
    return t


# --------------------------------------------------------------------------
# workload shapes
# --------------------------------------------------------------------------

def transformer_tensor_sizes(n_layer: int, d: int, vocab: int, n_pos: int) -> list[int]:
    """Flat tensor list of a GPT-2-style decoder (biases, pre-LN, 4x MLP).

    Per layer: LN1 weight+bias, fused QKV weight [d, 3d] + bias, attention
    projection [d, d] + bias, LN2 weight+bias, MLP up [d, 4d] + bias, MLP down
    [4d, d] + bias; then token embedding [vocab, d], position embedding
    [n_pos, d] and the final LN weight+bias.
    """
    sizes: list[int] = []
    for _ in range(n_layer):
        sizes += [d, d, d * 3 * d, 3 * d, d * d, d, d, d, d * 4 * d, 4 * d, 4 * d * d, d]
    sizes += [vocab * d, n_pos * d, d, d]
    return sizes


def gpt2_xl_tensor_sizes() -> list[int]:
    """GPT-2 1.5B (48 layers, d = 1600, vocab 50257, 1024 positions)."""
    return transformer_tensor_sizes(48, 1600, 50257, 1024)


def transformer_24l_d2048_tensor_sizes() -> list[int]:
    """24 layers, d = 2048, vocab 50257, 2048 positions."""
    return transformer_tensor_sizes(24, 2048, 50257, 2048)


def inject_schedule(steps: int, rate: float, seed: int, nd: int, psi: int,
                    force_step: int | None = None) -> dict[int, tuple[int, int, float]]:
    """Seeded overflow-injection schedule: {step: (rank, flat index, value)}.

    Each step is picked with probability ``rate``; ``force_step`` is always
    picked so a short run still exercises the skip path.  The value is +inf.
    """
    rs = np.random.default_rng(seed)
    out = {}
    for s in range(steps):
        hit = rs.random() < rate
        rank = int(rs.integers(0, nd))
        idx = int(rs.integers(0, psi))
        if hit or s == force_step:
            out[s] = (rank, idx, float("inf"))
    return out
