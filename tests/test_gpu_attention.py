"""Tensor-core attention (dllm_attention) vs the oracle's fp64 attention, element by
element, on the same f16 inputs.  Both kernels are covered: one query tile per CTA
(grids of at most one wave) and two query tiles per CTA in ping-pong (larger grids);
each case states which one its shape takes on the device.

Tolerance, from the kernel's arithmetic (both sides see the same f16 q, k, v):
  * each weight p_j = 2^(s_j c - m) is rounded to f16 (relative 2^-11, or absolute
    2^-25 below the normal range, against a maximum weight >= 1) and exp2f adds a
    few ulp of f32;
  * s_j = q.k_j is an f32 sum of exact f16 products: |error| <= dh 2^-24 sum|q k_j|,
    which moves p_j by ln2 c dh 2^-24 sum|q k_j| relative (c = log2(e)/sqrt(dh));
  * the common factor 2^-m cancels between the weights and the normaliser (which sums
    the weights before the f16 rounding): a relative perturbation of at most delta
    per weight moves each normalised weight by at most 2 delta of itself;
  * P V and the normaliser are f32 sums over Lk terms (relative (Lk + dh) 2^-24).
So |gpu - oracle| <= (2 delta + 2 (Lk + dh) 2^-24) A + 2^-24 Lk max|v| elementwise,
with A = sum_j w_j |v_j| = the oracle's attention over |v|.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_int8_gemm_q4_b200 import dllm, synth

pytestmark = pytest.mark.gpu

DH = 128
C = np.log2(np.e) / np.sqrt(DH)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from quantized_int8_gemm_q4_b200 import build
    build.build()
    dllm.load()
    yield
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK


def tiles(Lq, H):
    return dllm.dllm_debug_attention_tiles(Lq, H, torch.cuda.get_device_properties(0).multi_processor_count)


def run(q, k, v):
    Lq, H, dh = q.shape
    Lk, Hkv, _ = k.shape
    qd, kd, vd = (torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (q, k, v))
    o = torch.full((Lq, H, dh), float("nan"), dtype=torch.float32, device="cuda")
    dllm.dllm_attention(qd, kd, vd, Lq, Lk, H, Hkv, dh, o)
    torch.cuda.synchronize()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    return o.cpu().numpy()


def tolerance(q, k, v):
    """Elementwise bound of the module docstring, shape [Lq][H][dh]."""
    Lq, H, dh = q.shape
    Lk, Hkv, _ = k.shape
    g = H // Hkv
    qa, ka = np.abs(q.astype(np.float64)), np.abs(k.astype(np.float64))
    qk_abs = max(float(np.max(qa[:, h] @ ka[:, h // g].T)) for h in range(H))
    delta = 2.0 ** -11 + 2.0 ** -21 + np.log(2) * C * dh * 2.0 ** -24 * qk_abs
    A = oracle.attention(q.astype(np.float32), k.astype(np.float32), np.abs(v).astype(np.float32))
    vmax = float(np.max(np.abs(v.astype(np.float64))))
    return (2 * delta + 2 * (Lk + dh) * 2.0 ** -24) * A + 2.0 ** -24 * Lk * vmax


def check(q, k, v, rows=None):
    got = run(q, k, v)
    if rows is not None:
        got, q = got[rows], q[rows]
    ref = oracle.attention(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32))
    tol = tolerance(q, k, v)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err / tol), err.shape)
    assert np.all(err <= tol), f"worst at {worst}: |{got[worst]} - {ref[worst]}| > {tol[worst]}"
    return float(np.max(err / tol))


@pytest.mark.parametrize("Lq,Lk,H,Hkv,nt", [
    (1, 1, 1, 1, 1),        # one query, one key: the output is v exactly up to rounding
    (5, 3, 2, 1, 1),        # far below one tile, grouped heads
    (128, 128, 2, 2, 1),    # one full tile and one full key block
    (130, 200, 4, 2, 1),    # ragged query tile and ragged key block
    (257, 384, 2, 1, 1),    # three query tiles, three key blocks, the last query tile of 1
    (160, 160, 32, 32, 1),  # LLaDA-8B heads at the 160-position canvas
    (200, 200, 28, 4, 1),   # Dream-7B heads (28 query heads over 4 key/value heads)
    (300, 333, 64, 8, 2),   # two tiles per CTA; the last CTA of each head has one tile
    (400, 130, 48, 48, 2),  # two tiles per CTA, the second of the last CTA 16 rows long
    (640, 1, 32, 4, 2),     # one key: every output row is that key's value
    (512, 700, 40, 5, 2),   # two full tiles per CTA, ragged keys, 8 query heads per K/V head
])
def test_attention_matches_oracle(Lq, Lk, H, Hkv, nt):
    assert tiles(Lq, H) == nt
    q, k, v = synth.attention_inputs(Lq, Lk, H, Hkv, DH, 1, Lq, Lk, H)
    check(q, k, v)


@pytest.mark.parametrize("spread", [2.0, 4.0])
@pytest.mark.parametrize("Lq,H,nt", [(192, 2, 1), (260, 64, 2)])
def test_attention_peaked_softmax(spread, Lq, H, nt):
    """Logits of standard deviation spread^2: nearly one-hot rows."""
    assert tiles(Lq, H) == nt
    q, k, v = synth.attention_inputs(Lq, 640, H, 1, DH, 2, int(spread))
    check(q, k, v)


@pytest.mark.parametrize("Lq,H,nt", [(130, 2, 1), (300, 64, 2)])
def test_attention_running_max_raised_across_blocks(Lq, H, nt):
    """Key norms grow along the sequence: for queries leaning with the growth direction
    later 128-key blocks raise the running maximum by more than 2^8, so the output
    accumulator is rescaled in tensor memory; the other rows of the same warps keep
    theirs (the rescale factor is 1 for them)."""
    assert tiles(Lq, H) == nt
    q, k, v = synth.attention_inputs(Lq, 600, H, 1, DH, 3, key_growth=0.02)
    s = np.einsum("qhd,kd->qhk", q.astype(np.float64), k[:, 0].astype(np.float64)) * C
    m = s[..., :128].max(-1)
    raised, mixed = 0, 0
    n = Lq // 32 * 32
    for b in range(1, 5):
        bm = s[..., b * 128:(b + 1) * 128].max(-1)
        r = bm > m + 8
        m = np.where(r, bm, m)
        raised += int(r.sum())
        w = r[:n].reshape(n // 32, 32, -1)  # the softmax warps' 32-row groups
        mixed += int(np.sum(w.any(1) & ~w.all(1)))
    assert raised > 0, "inputs do not exercise the rescale"
    assert mixed > 0, "no warp mixes raised and kept maxima"
    check(q, k, v)


def test_attention_hard_attention_and_zero_query():
    """One key far above the rest (the output is that key's value) and all-zero queries
    (uniform weights: the mean of the values)."""
    q, k, v = synth.attention_inputs(130, 300, 1, 1, DH, 4)
    k[257] = (q[7, 0].astype(np.float32) * 4).astype(np.float16)
    q[100:] = 0
    got = run(q, k, v)
    assert np.allclose(got[7, 0], v[257, 0].astype(np.float32), rtol=0, atol=1e-3)
    assert np.allclose(got[100:], v[:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-4)
    check(q, k, v)


@pytest.mark.parametrize("L,H,Hkv", [(1024, 32, 32), (1024, 28, 4), (4096, 32, 32)])
def test_attention_full_canvas_sampled_rows(L, H, Hkv):
    """Full canvases at LLaDA-8B (32/32) and Dream-7B (28/4) heads, two tiles per CTA:
    every output row is computed by the kernel; 48 rows drawn across all query tiles
    are compared with the oracle run on those queries alone."""
    assert tiles(L, H) == 2
    q, k, v = synth.attention_inputs(L, L, H, Hkv, DH, 5)
    rows = np.sort(np.random.default_rng(5).choice(L, 48, replace=False))
    check(q, k, v, rows=rows)


def test_attention_empty_query_set_is_a_no_op():
    o = torch.full((4,), 7.0, device="cuda")
    dllm.dllm_attention(None, None, None, 0, 0, 2, 2, DH, None)
    assert torch.all(o == 7.0)


def test_attention_rejects_misaligned_and_bad_shapes():
    x = torch.zeros(4 * 2 * DH + 8, dtype=torch.float16, device="cuda")
    o = torch.zeros(4 * 2 * DH, dtype=torch.float32, device="cuda")
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_attention(x[1:], x, x, 4, 4, 2, 2, DH, o)
    assert e.value.code == dllm.DLLM_ERR_ALIGN
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_attention(x, x, x, 4, 4, 3, 2, DH, o)
    assert e.value.code == dllm.DLLM_ERR_ARG


def test_attention_on_requested_query_rows_only():
    """The last layer needs attention outputs at the requested canvas rows only (keys and
    values still span the whole canvas): the queries of those rows, gathered, give the
    same rows as the full canvas's attention, within the bound, through either kernel."""
    L, H, Hkv = 1024, 32, 32
    q, k, v = synth.attention_inputs(L, L, H, Hkv, DH, 6)
    rows = np.sort(synth.block_rows(L, 32, 6))
    assert tiles(len(rows), H) == 1 and tiles(L, H) == 2
    got_rows = run(np.ascontiguousarray(q[rows]), k, v)
    got_full = run(q, k, v)[rows]
    ref = oracle.attention(q[rows].astype(np.float32), k.astype(np.float32), v.astype(np.float32))
    tol = tolerance(q[rows], k, v)
    for got in (got_rows, got_full):
        assert np.all(np.abs(got - ref) <= tol)
