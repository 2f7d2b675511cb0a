"""An independent numpy restatement of the exact Q5_K -> two Q4_K-form super-blocks
split (byte work only): the low nibbles keep d, dmin, the scales and qs; the fifth bits
become 0/1 nibbles with d' = 16 d, dmin' = 0 and the same scale bytes."""
import numpy as np


def split_q5k(blocks: np.ndarray) -> np.ndarray:
    """uint8 [N][nsb][176] Q5_K -> uint8 [N][2 nsb][144] Q4_K-form (low blocks, then high)."""
    N, nsb, bb = blocks.shape
    assert bb == 176
    lo = np.zeros((N, nsb, 144), np.uint8)
    hi = np.zeros((N, nsb, 144), np.uint8)
    lo[..., 0:4] = blocks[..., 0:4]
    lo[..., 4:16] = blocks[..., 4:16]
    lo[..., 16:144] = blocks[..., 48:176]
    d = blocks[..., 0:2].copy().view(np.float16)[..., 0]
    hi[..., 0:2] = (d.astype(np.float32) * 16).astype(np.float16)[..., None].view(np.uint8)
    hi[..., 4:16] = blocks[..., 4:16]
    qh = blocks[..., 16:48]                                  # [N][nsb][32]
    for c in range(4):
        b0 = (qh >> (2 * c)) & 1
        b1 = (qh >> (2 * c + 1)) & 1
        hi[..., 16 + 32 * c:16 + 32 * c + 32] = b0 | (b1 << 4)
    return np.concatenate([lo, hi], axis=1)
