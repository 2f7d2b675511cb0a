"""CPU oracle for the Q4_K/Q6_K x int8 projection GEMM (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline leg
may import this package.  It wraps ``oracle.c`` (plain C, fp64 combine) through
ctypes and shares nothing with the CUDA library.

Parity status of each function (what pins it) is listed in the module
docstrings of ``tests/test_oracle_*.py``; every function here is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "oracle.c"
LIB = HERE / "_build" / "liboracle.so"

Q8_0 = 8
Q4_K = 12
Q5_K = 13
Q6_K = 14
QK_K = 256
# bytes per 256 weights of a row: one K-quant super-block, or eight 34-byte Q8_0 blocks
BLOCK_BYTES = {Q4_K: 144, Q5_K: 176, Q6_K: 210, Q8_0: 272}

_lib = None


def build(force: bool = False) -> Path:
    """Compile oracle.c into a shared library (plain C, no intrinsics)."""
    LIB.parent.mkdir(parents=True, exist_ok=True)
    if force or not LIB.exists() or LIB.stat().st_mtime < SRC.stat().st_mtime:
        cmd = ["gcc", "-std=c99", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", str(SRC), "-o", str(LIB) + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(str(LIB) + ".tmp", LIB)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(LIB))
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_f16_to_f64.restype = ctypes.c_double
        L.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_q4k_decode.argtypes = [P, P, P, P, P, P]
        L.oracle_q6k_decode.argtypes = [P, P, P, P]
        L.oracle_q5k_decode.argtypes = [P, P, P, P, P, P]
        L.oracle_q80_decode.argtypes = [P, P, P]
        L.oracle_dequant.argtypes = [ctypes.c_int, P, I64, I64, P]
        L.oracle_quantize_act.argtypes = [P, I64, I64, I64, P, P, P]
        L.oracle_qgemm.argtypes = [ctypes.c_int, P, I64, I64, P, P, I64, P, I64, I64, I64,
                                   P, P, P, I64, ctypes.c_int]
        L.oracle_sb_ints.argtypes = [ctypes.c_int, P, I64, I64, P, I64, P, P, P]
        L.oracle_rmsnorm.argtypes = [P, I64, I64, I64, P, ctypes.c_float, ctypes.c_double, P]
        L.oracle_swiglu.argtypes = [P, P, I64, I64, I64, ctypes.c_double, P]
        L.oracle_attention.argtypes = [P, P, P, I64, I64, I64, I64, I64, P, ctypes.c_int]
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _chk(rc):
    if rc != 0:
        raise ValueError("oracle rejected its arguments")


def max_threads() -> int:
    return lib().oracle_max_threads()


def f16_to_f64(bits: int) -> float:
    return lib().oracle_f16_to_f64(bits & 0xFFFF)


def q4k_decode(block: np.ndarray):
    """One 144-byte Q4_K block -> (d, dmin, sc[8], m[8], q[256])."""
    b = np.ascontiguousarray(block, dtype=np.uint8)
    assert b.size == 144
    d = np.zeros(1, np.float64)
    dmin = np.zeros(1, np.float64)
    sc = np.zeros(8, np.uint8)
    mn = np.zeros(8, np.uint8)
    q = np.zeros(256, np.uint8)
    lib().oracle_q4k_decode(_p(b), _p(d), _p(dmin), _p(sc), _p(mn), _p(q))
    return float(d[0]), float(dmin[0]), sc, mn, q


def q5k_decode(block: np.ndarray):
    """One 176-byte Q5_K block -> (d, dmin, sc[8], m[8], q[256] in [0,31])."""
    b = np.ascontiguousarray(block, dtype=np.uint8)
    assert b.size == 176
    d = np.zeros(1, np.float64)
    dmin = np.zeros(1, np.float64)
    sc = np.zeros(8, np.uint8)
    mn = np.zeros(8, np.uint8)
    q = np.zeros(256, np.uint8)
    lib().oracle_q5k_decode(_p(b), _p(d), _p(dmin), _p(sc), _p(mn), _p(q))
    return float(d[0]), float(dmin[0]), sc, mn, q


def q80_decode(block: np.ndarray):
    """One 34-byte Q8_0 block -> (d, q[32] int8)."""
    b = np.ascontiguousarray(block, dtype=np.uint8)
    assert b.size == 34
    d = np.zeros(1, np.float64)
    q = np.zeros(32, np.int8)
    lib().oracle_q80_decode(_p(b), _p(d), _p(q))
    return float(d[0]), q


def q6k_decode(block: np.ndarray):
    """One 210-byte Q6_K block -> (d, sc[16] int8, q[256] in [0,63])."""
    b = np.ascontiguousarray(block, dtype=np.uint8)
    assert b.size == 210
    d = np.zeros(1, np.float64)
    sc = np.zeros(16, np.int8)
    q = np.zeros(256, np.uint8)
    lib().oracle_q6k_decode(_p(b), _p(d), _p(sc), _p(q))
    return float(d[0]), sc, q


def dequant(qtype: int, w: np.ndarray, N: int, K: int) -> np.ndarray:
    """Row-major blocks ([N][K/256] super-blocks, or [N][K/32] Q8_0 blocks) -> fp64 [N][K]."""
    w = np.ascontiguousarray(w, dtype=np.uint8)
    assert w.size == N * (K // QK_K) * BLOCK_BYTES[qtype]
    out = np.zeros((N, K), np.float64)
    _chk(lib().oracle_dequant(qtype, _p(w), N, K, _p(out)))
    return out


def quantize_act(x: np.ndarray):
    """f32 [M][K] -> (q int8 [M][K], scale f32 [M][K/256], asum32 int32 [M][K/32])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    M, K = x.shape
    q = np.zeros((M, K), np.int8)
    s = np.zeros((M, K // QK_K), np.float32)
    a = np.zeros((M, K // 32), np.int32)
    _chk(lib().oracle_quantize_act(_p(x), M, K, K, _p(q), _p(s), _p(a)))
    return q, s, a


def qgemm(qtype: int, w: np.ndarray, N: int, K: int, q: np.ndarray, scale: np.ndarray,
          rows=None, n0: int = 0, n1: int | None = None, nthreads: int | None = None):
    """Returns (out f32, out fp64, T fp64), each [n_out][n1-n0]."""
    w = np.ascontiguousarray(w, dtype=np.uint8)
    q = np.ascontiguousarray(q, dtype=np.int8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    M = q.shape[0]
    n1 = N if n1 is None else n1
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n_out = M if r is None else r.size
    width = n1 - n0
    out = np.zeros((n_out, width), np.float32)
    out64 = np.zeros((n_out, width), np.float64)
    T = np.zeros((n_out, width), np.float64)
    nt = max_threads() if nthreads is None else nthreads
    _chk(lib().oracle_qgemm(qtype, _p(w), N, K, _p(q), _p(scale), M, _p(r),
                            0 if r is None else r.size, n0, n1, _p(out), _p(out64), _p(T),
                            width, nt))
    return out, out64, T


def sb_ints(qtype: int, w: np.ndarray, N: int, K: int, q: np.ndarray):
    """Integer intermediates: (dots [M][N][nsub_total] int32, S, Smin [M][N][K/256] int64)."""
    w = np.ascontiguousarray(w, dtype=np.uint8)
    q = np.ascontiguousarray(q, dtype=np.int8)
    M = q.shape[0]
    nsub = K // 16 if qtype == Q6_K else K // 32
    dots = np.zeros((M, N, nsub), np.int32)
    S = np.zeros((M, N, K // QK_K), np.int64)
    Smin = np.zeros((M, N, K // QK_K), np.int64)
    _chk(lib().oracle_sb_ints(qtype, _p(w), N, K, _p(q), M, _p(dots), _p(S), _p(Smin)))
    return dots, S, Smin


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float, ss_scale: float = 1.0) -> np.ndarray:
    """f32 [M][K] -> f32 [M][K]: f32((x * r) * gamma), r = 1/sqrt(ss/K + eps) in fp64.
    ss_scale != 1 scales the sum of squares (tests use it to bracket summation order)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    M, K = x.shape
    assert g.shape == (K,)
    y = np.zeros((M, K), np.float32)
    _chk(lib().oracle_rmsnorm(_p(x), M, K, K, _p(g), float(eps), float(ss_scale), _p(y)))
    return y


def swiglu(gate: np.ndarray, up: np.ndarray, h_scale: float = 1.0) -> np.ndarray:
    """f32 [M][K] x2 -> f32 [M][K]: f32((g / (1 + exp(-g))) * u) in fp64.
    h_scale != 1 scales the fp64 value before rounding (tests use it to bracket exp)."""
    g = np.ascontiguousarray(gate, dtype=np.float32)
    u = np.ascontiguousarray(up, dtype=np.float32)
    assert g.shape == u.shape
    M, K = g.shape
    h = np.zeros((M, K), np.float32)
    _chk(lib().oracle_swiglu(_p(g), _p(u), M, K, K, float(h_scale), _p(h)))
    return h


def rmsnorm_quantize(x: np.ndarray, gamma: np.ndarray, eps: float):
    """quantize_act(rmsnorm(x)): the definition the fused library kernel follows."""
    return quantize_act(rmsnorm(x, gamma, eps))


def swiglu_quantize(gate: np.ndarray, up: np.ndarray):
    """quantize_act(swiglu(gate, up)): the definition the fused library kernel follows."""
    return quantize_act(swiglu(gate, up))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """Bidirectional attention, fp64: q [Lq][H][dh], k and v [Lk][Hkv][dh] -> o [Lq][H][dh].
    Head h attends with key/value head h // (H / Hkv)."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    Lq, H, dh = q.shape
    Lk, Hkv, dh2 = k.shape
    assert v.shape == k.shape and dh2 == dh
    o = np.zeros((Lq, H, dh), np.float64)
    nt = max_threads() if nthreads is None else nthreads
    _chk(lib().oracle_attention(_p(q), _p(k), _p(v), Lq, Lk, H, Hkv, dh, _p(o), nt))
    return o
