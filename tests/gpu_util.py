"""Helpers shared by the GPU tests: run the CUDA path through the C-ABI binding, and
convert its tiled outputs back to the plain row-major views the oracle uses."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm, synth

QK = 256


def untile_q(q_t: torch.Tensor, M: int, K: int) -> np.ndarray:
    """[K/256][Mp/8][16][8][16] int8 -> [M][K]."""
    Mp = (M + 15) // 16 * 16
    a = q_t.cpu().numpy().reshape(K // QK, Mp // 8, 16, 8, 16)
    return a.transpose(1, 3, 0, 2, 4).reshape(Mp, K)[:M]


def untile_scale(s_t: torch.Tensor, M: int, K: int) -> np.ndarray:
    Mp = (M + 15) // 16 * 16
    return s_t.cpu().numpy().reshape(K // QK, Mp).T[:M]


def untile_sums(u_t: torch.Tensor, M: int, K: int):
    """-> (hi, lo) float32 [M][K/32]: the scaled per-32 sums split as hi + lo."""
    Mp = (M + 15) // 16 * 16
    u = u_t.cpu().numpy().view(np.float32).reshape(K // QK, Mp // 8, 2, 2, 8, 4)  # s, g, hi/lo, j-chunk, row, j
    a = u.transpose(1, 4, 0, 2, 3, 5).reshape(Mp, K // QK, 2, 8)                  # row, s, hi/lo, j
    return a[:M, :, 0, :].reshape(M, K // 32), a[:M, :, 1, :].reshape(M, K // 32)


def repack_reference(qtype: int, blocks: np.ndarray) -> np.ndarray:
    """Independent restatement of the documented tile layout, in numpy (byte work)."""
    N, nsb, bb = blocks.shape
    tiles = []
    for t in range(N // 128):
        for s in range(nsb):
            blk = blocks[128 * t:128 * t + 128, s]
            if qtype == dllm.DLLM_Q4_K:
                parts = [blk[:, 16:144].reshape(128, 8, 16).transpose(1, 0, 2), blk[:, 4:16], blk[:, 0:4]]
            else:
                parts = [blk[:, 0:128].reshape(128, 8, 16).transpose(1, 0, 2),
                         blk[:, 128:192].reshape(128, 4, 16).transpose(1, 0, 2), blk[:, 192:208], blk[:, 208:210]]
            tiles.append(np.concatenate([p.reshape(-1) for p in parts]))
    return np.concatenate(tiles)


class Act:
    """Quantized activations of an f32 canvas, on the device."""

    def __init__(self, x: np.ndarray, stream=None):
        self.M, self.K = x.shape
        self.x = torch.from_numpy(np.ascontiguousarray(x)).cuda()
        self.q, self.scale, self.sums = dllm.alloc_act(self.M, self.K)
        dllm.dllm_quantize_act(self.x, self.M, self.K, self.K, self.q, self.scale, self.sums, stream)

    def host(self):
        return (untile_q(self.q, self.M, self.K), untile_scale(self.scale, self.M, self.K),
                untile_sums(self.sums, self.M, self.K))


def gemm(w_dev, qtype, N, K, act: Act, rows=None, ldo=None, stream=None):
    ldo = N if ldo is None else ldo
    n_out = act.M if rows is None else len(rows)
    out = torch.full((n_out, ldo), float("nan"), dtype=torch.float32, device="cuda")
    r = None if rows is None else torch.tensor(np.asarray(rows, np.int32), device="cuda")
    nr = 0 if rows is None else len(rows)
    wsb = dllm.dllm_qgemm_workspace_bytes(qtype, N, K, act.M, nr)
    ws = dllm.alloc_workspace(wsb)
    dllm.dllm_qgemm(w_dev, qtype, N, K, act.q, act.scale, act.sums, act.M, r, nr, out, ldo, ws, wsb, stream)
    return out


def tol_ok(got: np.ndarray, ref: np.ndarray, T: np.ndarray):
    """The pass criterion: |gpu - ref| <= max(1e-5 |ref|, 1e-6 T) elementwise."""
    bound = np.maximum(1e-5 * np.abs(ref), 1e-6 * T)
    err = np.abs(got.astype(np.float64) - ref)
    return bool(np.all(err <= bound)), float(np.max(err / np.maximum(bound, 1e-300)))


def make_case(qtype, M, N, K, seed):
    w = synth.weights(qtype, N, K, seed, M, N, K)
    x = synth.activations(M, K, seed, M, N, K)
    return w, x
