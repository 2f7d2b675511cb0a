"""Seeded synthetic inputs and workload shapes.

This module holds no arithmetic of the method: it only draws random bytes and
numbers with the distributions the workloads call for, and lays the bytes out
in the GGUF block order.  Both the oracle-side tests and the CUDA-side tests
and benchmark take their inputs from here.

Distributions (the synthetic stand-ins for real GGUF weights, which are not used):
  * Q4_K: the 12 scale bytes and 128 quant bytes are uniform random bytes, so
    every 4-bit quant is uniform on 0..15 and every 6-bit scale and min is
    uniform on 0..63; d and dmin are uniform on [1e-3, 1e-2] rounded to f16.
  * Q6_K: the 128 low-bit bytes and 64 high-bit bytes are uniform random bytes,
    so every 6-bit quant is uniform on 0..63; the 16 int8 scales are uniform on
    -32..31 (configurable); d as above.
  * Q5_K: as Q4_K, plus 32 uniform random bytes of fifth bits, so every 5-bit quant
    is uniform on 0..31.
  * Q8_0: every 34-byte block has d uniform on [1e-4, 1e-3] rounded to f16 and 32
    int8 quants uniform on -127..127.
  * Activations: f32 standard normal.
  * Attention inputs: q, k, v standard normal rounded to f16, q and k times a
    spread factor (1 gives logits q.k/sqrt(128) of unit standard deviation; larger
    factors give the peaked softmax rows of a trained model); optionally the key
    rows grow linearly in norm along the sequence (each block of 128 keys then
    raises the running maximum of the rows whose query leans the same way).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

Q8_0 = 8
Q4_K = 12
Q5_K = 13
Q6_K = 14
QK_K = 256
BLOCK_BYTES = {Q4_K: 144, Q5_K: 176, Q6_K: 210, Q8_0: 272}  # bytes per 256 weights


def _rng(seed, *sub):
    return np.random.default_rng([int(seed), *[int(s) for s in sub]])


def _f16_bytes(rng, n, lo=1e-3, hi=1e-2):
    v = rng.uniform(lo, hi, size=n).astype(np.float16)
    return v.view(np.uint8).reshape(n, 2)


def q4k_weights(N: int, K: int, seed, *sub) -> np.ndarray:
    """uint8 [N, K/256, 144] GGUF Q4_K blocks: d | dmin | 12 scale bytes | 128 quant bytes."""
    assert K % QK_K == 0
    nb = N * (K // QK_K)
    rng = _rng(seed, 4, *sub)
    blk = np.empty((nb, 144), np.uint8)
    blk[:, 0:2] = _f16_bytes(rng, nb)
    blk[:, 2:4] = _f16_bytes(rng, nb)
    blk[:, 4:144] = rng.integers(0, 256, size=(nb, 140), dtype=np.uint8)
    return blk.reshape(N, K // QK_K, 144)


def q6k_weights(N: int, K: int, seed, *sub, sc_lo: int = -32, sc_hi: int = 31) -> np.ndarray:
    """uint8 [N, K/256, 210] GGUF Q6_K blocks: 128 low | 64 high | 16 int8 scales | d."""
    assert K % QK_K == 0
    nb = N * (K // QK_K)
    rng = _rng(seed, 6, *sub)
    blk = np.empty((nb, 210), np.uint8)
    blk[:, 0:192] = rng.integers(0, 256, size=(nb, 192), dtype=np.uint8)
    blk[:, 192:208] = rng.integers(sc_lo, sc_hi + 1, size=(nb, 16)).astype(np.int8).view(np.uint8)
    blk[:, 208:210] = _f16_bytes(rng, nb)
    return blk.reshape(N, K // QK_K, 210)


def q5k_weights(N: int, K: int, seed, *sub) -> np.ndarray:
    """uint8 [N, K/256, 176] GGUF Q5_K blocks: d | dmin | 12 scale bytes | 32 qh | 128 qs."""
    assert K % QK_K == 0
    nb = N * (K // QK_K)
    rng = _rng(seed, 5, *sub)
    blk = np.empty((nb, 176), np.uint8)
    blk[:, 0:2] = _f16_bytes(rng, nb)
    blk[:, 2:4] = _f16_bytes(rng, nb)
    blk[:, 4:176] = rng.integers(0, 256, size=(nb, 172), dtype=np.uint8)
    return blk.reshape(N, K // QK_K, 176)


def q80_weights(N: int, K: int, seed, *sub) -> np.ndarray:
    """uint8 [N, K/256, 272]: per 256 weights, eight GGUF Q8_0 blocks d | 32 int8."""
    assert K % QK_K == 0
    nb = N * (K // 32)
    rng = _rng(seed, 11, *sub)
    blk = np.empty((nb, 34), np.uint8)
    blk[:, 0:2] = _f16_bytes(rng, nb, 1e-4, 1e-3)
    blk[:, 2:34] = rng.integers(-127, 128, size=(nb, 32)).astype(np.int8).view(np.uint8)
    return blk.reshape(N, K // QK_K, 272)


def weights(qtype: int, N: int, K: int, seed, *sub) -> np.ndarray:
    gen = {Q4_K: q4k_weights, Q5_K: q5k_weights, Q6_K: q6k_weights, Q8_0: q80_weights}[qtype]
    return gen(N, K, seed, *sub)


def activations(M: int, K: int, seed, *sub) -> np.ndarray:
    """f32 [M, K] standard normal."""
    return _rng(seed, 8, *sub).standard_normal((M, K), dtype=np.float32)


def attention_inputs(Lq: int, Lk: int, H: int, Hkv: int, dh: int, seed, *sub, spread: float = 1.0,
                     key_growth: float = 0.0):
    """f16 q [Lq][H][dh], k and v [Lk][Hkv][dh]."""
    rng = _rng(seed, 11, *sub)
    q = (rng.standard_normal((Lq, H, dh)) * spread).astype(np.float16)
    k = rng.standard_normal((Lk, Hkv, dh)) * spread
    k *= (1.0 + key_growth * np.arange(Lk))[:, None, None]
    v = rng.standard_normal((Lk, Hkv, dh)).astype(np.float16)
    return q, k.astype(np.float16), v


def norm_weights(n: int, K: int, seed, *sub) -> np.ndarray:
    """f32 [n, K] RMSNorm gains, uniform in [0.5, 1.5) (trained gains sit around 1)."""
    return (_rng(seed, 10, *sub).random((n, K)) + 0.5).astype(np.float32)


def block_rows(M: int, n_rows: int, seed, *sub, block: int | None = None) -> np.ndarray:
    """n_rows distinct canvas rows in random order, drawn from one 32-row window
    [32 + 32b, 64 + 32b) of an M-row canvas whose first 32 rows are the prompt."""
    rng = _rng(seed, 9, *sub)
    nblk = max(1, (M - 32) // 32)
    b = int(rng.integers(0, nblk)) if block is None else block
    lo = min(32 + 32 * b, M - 32)
    return (lo + rng.permutation(32)[:n_rows]).astype(np.int32)


@dataclass(frozen=True)
class Proj:
    """One projection GEMM of a layer: N output features, K inputs, weight type."""
    name: str
    qtype: int
    N: int
    K: int


@dataclass(frozen=True)
class Model:
    name: str
    hidden: int
    ffn: int
    n_layers: int
    q_out: int
    kv_out: int
    vocab: int
    out_rows: int = 32
    layer: tuple = field(default=())
    norm_eps: float = 1e-5
    heads: int = 32  # attention heads; head dim = hidden / heads = 128 for both models

    @property
    def kv_heads(self) -> int:
        return self.kv_out // (self.hidden // self.heads)


def llada_8b() -> Model:
    h, f = 4096, 12288
    return Model("llada-8b", h, f, 32, h, h, 126464, 32,
                 (Proj("q", Q4_K, h, h), Proj("k", Q4_K, h, h), Proj("v", Q4_K, h, h),
                  Proj("o", Q4_K, h, h), Proj("gate", Q4_K, f, h), Proj("up", Q4_K, f, h),
                  Proj("down", Q6_K, h, f)))


def dream_7b() -> Model:
    h, f = 3584, 18944
    return Model("dream-7b", h, f, 28, h, 512, 152064, 32,
                 (Proj("q", Q4_K, h, h), Proj("k", Q4_K, 512, h), Proj("v", Q4_K, 512, h),
                  Proj("o", Q4_K, h, h), Proj("gate", Q4_K, f, h), Proj("up", Q4_K, f, h),
                  Proj("down", Q6_K, h, f)), norm_eps=1e-6, heads=28)


MODELS = {"llada-8b": llada_8b, "dream-7b": dream_7b}


# ---------------------------------------------------------------------------
# Device-side draws with the same distributions (for the multi-GB benchmark
# models, which would take minutes to draw and copy from the host).

def _torch_gen(device, seed, *sub):
    import torch
    g = torch.Generator(device=device)
    h = int(seed) & 0xFFFFFFFF
    for s in sub:
        h = (h * 1000003 + (int(s) & 0xFFFFFFFF)) & 0x7FFFFFFFFFFFFFFF
    g.manual_seed(h)
    return g


def device_weights(qtype: int, N: int, K: int, seed, *sub, device="cuda"):
    """GGUF blocks as a flat uint8 device tensor, drawn on the device (torch generator)."""
    import torch
    assert K % QK_K == 0
    nb = N * (K // QK_K)
    g = _torch_gen(device, seed, qtype, *sub)
    bb = BLOCK_BYTES[qtype]
    blk = torch.empty((nb, bb), dtype=torch.uint8, device=device)
    if qtype == Q8_0:  # eight 34-byte blocks per 256 weights: d in [1e-4, 1e-3), 32 int8 codes
        b8 = blk.view(nb * 8, 34)
        d8 = (torch.rand((nb * 8, 1), generator=g, device=device) * (1e-3 - 1e-4) + 1e-4).to(torch.float16)
        b8[:, 0:2] = d8.contiguous().view(torch.uint8).reshape(nb * 8, 2)
        b8[:, 2:] = torch.randint(-127, 128, (nb * 8, 32), generator=g, device=device,
                                  dtype=torch.int8).view(torch.uint8)
        return blk.reshape(-1)
    d = (torch.rand((nb, 2 if qtype == Q4_K else 1), generator=g, device=device) * (1e-2 - 1e-3) + 1e-3)
    d16 = d.to(torch.float16).contiguous().view(torch.uint8).reshape(nb, -1)
    if qtype == Q4_K:
        blk[:, 0:4] = d16
        blk[:, 4:] = torch.randint(0, 256, (nb, 140), generator=g, device=device, dtype=torch.uint8)
    else:
        blk[:, 0:192] = torch.randint(0, 256, (nb, 192), generator=g, device=device, dtype=torch.uint8)
        blk[:, 192:208] = torch.randint(-32, 32, (nb, 16), generator=g, device=device,
                                        dtype=torch.int8).view(torch.uint8)
        blk[:, 208:210] = d16
    return blk.reshape(-1)


def device_activations(M: int, K: int, seed, *sub, device="cuda"):
    import torch
    g = _torch_gen(device, seed, 8, *sub)
    return torch.randn((M, K), generator=g, device=device, dtype=torch.float32)


def device_attention_inputs(Lq: int, Lk: int, H: int, Hkv: int, dh: int, seed, *sub, device="cuda"):
    """f16 q [Lq][H][dh], k and v [Lk][Hkv][dh], standard normal, drawn on the device."""
    import torch
    g = _torch_gen(device, seed, 11, *sub)
    q = torch.randn((Lq, H, dh), generator=g, device=device).to(torch.float16)
    k = torch.randn((Lk, Hkv, dh), generator=g, device=device).to(torch.float16)
    v = torch.randn((Lk, Hkv, dh), generator=g, device=device).to(torch.float16)
    return q, k, v
