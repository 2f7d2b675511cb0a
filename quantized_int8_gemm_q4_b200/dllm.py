"""Python binding of the dllm_qgemm C-ABI (include/dllm_qgemm.h).

Argument marshalling only: every step runs in the CUDA library.  torch supplies
device memory and streams.  There is no CPU fallback: if the compiled library is
missing, importing a function raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().parent / "_build" / "libdllm_qgemm.so"

DLLM_Q4_K = 12
DLLM_Q6_K = 14
DLLM_Q5_K = 13
DLLM_Q8_0 = 8
QK_K = 256
BLOCK_BYTES = {DLLM_Q4_K: 144, DLLM_Q6_K: 210}

DLLM_OK = 0
DLLM_ERR_ARG = -1
DLLM_ERR_ALIGN = -2
DLLM_ERR_UNSUPPORTED = -3
DLLM_ERR_CUDA = -4
DLLM_ERR_ROW_RANGE = -5
DLLM_ERR_TIMEOUT = -6
DLLM_ERR_WORKSPACE = -7
DLLM_ERR_SCRATCH_LIMIT = -8
DLLM_ERR_SCALE_RANGE = -9
DLLM_NOALLOC_SCRATCH_BYTES = 32 << 20

EXPORTS = (
    "dllm_repacked_bytes", "dllm_repack_q4k", "dllm_repack_q6k", "dllm_repack_q5k", "dllm_repack_q80",
    "dllm_act_bytes",
    "dllm_quantize_act",
    "dllm_rmsnorm_quantize", "dllm_swiglu_quantize",
    "dllm_qgemm_workspace_bytes", "dllm_qgemm", "dllm_qgemm_noalloc", "dllm_qkv_qgemm", "dllm_attention",
    "dllm_get_device_status",
    "dllm_status_string", "dllm_debug_subblock_dots", "dllm_debug_sb_ints", "dllm_debug_bounded_wait",
    "dllm_bench_mma_i8", "dllm_debug_plan", "dllm_debug_attention_tiles",
    "dllm_debug_attention_stall",
)


class DllmError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


_lib = None


def load() -> ctypes.CDLL:
    """Load the compiled library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"dllm_qgemm CUDA library not built: {LIB_PATH} is missing "
                          "(run __graft_entry__.build() or python -m quantized_int8_gemm_q4_b200.build)")
    L = ctypes.CDLL(str(LIB_PATH))
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    SZ = ctypes.c_size_t
    PSZ = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "dllm_repacked_bytes": [I, I64, I64, PSZ],
        "dllm_repack_q4k": [P, I64, I64, P, P],
        "dllm_repack_q6k": [P, I64, I64, P, P],
        "dllm_repack_q5k": [P, I64, I64, P, P],
        "dllm_repack_q80": [P, I64, I64, P, P],
        "dllm_act_bytes": [I64, I64, PSZ, PSZ, PSZ],
        "dllm_quantize_act": [P, I64, I64, I64, P, P, P, P],
        "dllm_rmsnorm_quantize": [P, I64, I64, I64, P, ctypes.c_float, P, I64, P, P, P, P],
        "dllm_swiglu_quantize": [P, P, I64, I64, I64, P, P, P, P],
        "dllm_qgemm_workspace_bytes": [I, I64, I64, I64, I64, PSZ],
        "dllm_qgemm": [P, I, I64, I64, P, P, P, I64, P, I64, P, I64, P, SZ, P],
        "dllm_qgemm_noalloc": [P, I, I64, I64, P, P, P, I64, P, I64, P, I64, P],
        "dllm_qkv_qgemm": [P, P, P, I, I64, I64, I64, P, P, P, I64, P, I64, P, P, I64, P, SZ, P],
        "dllm_attention": [P, P, P, I64, I64, I64, I64, I64, P, P],
        "dllm_get_device_status": [P],
        "dllm_status_string": [I],
        "dllm_debug_subblock_dots": [P, I, I64, I64, P, I64, P, P],
        "dllm_debug_sb_ints": [P, I, I64, I64, P, P, P, I64, P, P],
        "dllm_debug_bounded_wait": [P],
        "dllm_bench_mma_i8": [I, I, I, I, I, I, P, P],
        "dllm_debug_plan": [I64, I64, I64, I64, I, ctypes.POINTER(ctypes.c_int64)],
        "dllm_debug_attention_tiles": [I64, I64, I],
        "dllm_debug_attention_stall": [I, P],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name == "dllm_status_string" else ctypes.c_int
    _lib = L
    return L


def status_string(code: int) -> str:
    try:
        return load().dllm_status_string(code).decode()
    except ImportError:
        return "library not loaded"


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != DLLM_OK:
        raise DllmError(rc, where)


# ------------------------------------------------------------------ C-ABI, same names

def dllm_repacked_bytes(qtype: int, N: int, K: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load().dllm_repacked_bytes(qtype, N, K, ctypes.byref(out)), "dllm_repacked_bytes")
    return out.value


def dllm_repack_q4k(gguf_blocks, N: int, K: int, dst, stream=None):
    _check(load().dllm_repack_q4k(_ptr(gguf_blocks), N, K, _ptr(dst), _stream(stream)), "dllm_repack_q4k")


def dllm_repack_q5k(gguf_blocks, N: int, K: int, dst, stream=None):
    _check(load().dllm_repack_q5k(_ptr(gguf_blocks), N, K, _ptr(dst), _stream(stream)), "dllm_repack_q5k")


def dllm_repack_q80(gguf_blocks, N: int, K: int, dst, stream=None):
    _check(load().dllm_repack_q80(_ptr(gguf_blocks), N, K, _ptr(dst), _stream(stream)), "dllm_repack_q80")


def dllm_repack_q6k(gguf_blocks, N: int, K: int, dst, stream=None):
    _check(load().dllm_repack_q6k(_ptr(gguf_blocks), N, K, _ptr(dst), _stream(stream)), "dllm_repack_q6k")


def dllm_act_bytes(M: int, K: int):
    a, b, c = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load().dllm_act_bytes(M, K, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)), "dllm_act_bytes")
    return a.value, b.value, c.value


def dllm_quantize_act(x, M: int, K: int, ldx: int, q, scale, sums, stream=None):
    _check(load().dllm_quantize_act(_ptr(x), M, K, ldx, _ptr(q), _ptr(scale), _ptr(sums), _stream(stream)),
           "dllm_quantize_act")


def dllm_rmsnorm_quantize(x, M: int, K: int, ldx: int, gamma, eps: float, rows, n_rows: int, q, scale, sums,
                          stream=None):
    _check(load().dllm_rmsnorm_quantize(_ptr(x), M, K, ldx, _ptr(gamma), float(eps), _ptr(rows), n_rows, _ptr(q),
                                        _ptr(scale), _ptr(sums), _stream(stream)), "dllm_rmsnorm_quantize")


def dllm_swiglu_quantize(gate, up, M: int, K: int, ld: int, q, scale, sums, stream=None):
    _check(load().dllm_swiglu_quantize(_ptr(gate), _ptr(up), M, K, ld, _ptr(q), _ptr(scale), _ptr(sums),
                                       _stream(stream)), "dllm_swiglu_quantize")


def dllm_qgemm_workspace_bytes(qtype: int, N: int, K: int, M: int, n_rows: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(load().dllm_qgemm_workspace_bytes(qtype, N, K, M, n_rows, ctypes.byref(out)),
           "dllm_qgemm_workspace_bytes")
    return out.value


def dllm_qgemm(w, qtype: int, N: int, K: int, q, scale, sums, M: int, rows, n_rows: int, out, ldo: int,
               workspace=None, workspace_bytes: int = 0, stream=None):
    _check(load().dllm_qgemm(_ptr(w), qtype, N, K, _ptr(q), _ptr(scale), _ptr(sums), M, _ptr(rows), n_rows,
                             _ptr(out), ldo, _ptr(workspace), workspace_bytes, _stream(stream)), "dllm_qgemm")


def dllm_qgemm_noalloc(w, qtype: int, N: int, K: int, q, scale, sums, M: int, rows, n_rows: int, out, ldo: int,
                       stream=None):
    _check(load().dllm_qgemm_noalloc(_ptr(w), qtype, N, K, _ptr(q), _ptr(scale), _ptr(sums), M, _ptr(rows),
                                     n_rows, _ptr(out), ldo, _stream(stream)), "dllm_qgemm_noalloc")


def dllm_qkv_qgemm(wq, wk, wv, qtype: int, Nq: int, Nkv: int, K: int, q, scale, sums, M: int, oq, ldo_q: int,
                   ok, ov, ldo_kv: int, workspace=None, workspace_bytes: int = 0, stream=None):
    _check(load().dllm_qkv_qgemm(_ptr(wq), _ptr(wk), _ptr(wv), qtype, Nq, Nkv, K, _ptr(q), _ptr(scale), _ptr(sums),
                                 M, _ptr(oq), ldo_q, _ptr(ok), _ptr(ov), ldo_kv, _ptr(workspace), workspace_bytes,
                                 _stream(stream)), "dllm_qkv_qgemm")


def dllm_attention(q, k, v, Lq: int, Lk: int, H: int, Hkv: int, dh: int, o, stream=None):
    _check(load().dllm_attention(_ptr(q), _ptr(k), _ptr(v), Lq, Lk, H, Hkv, dh, _ptr(o), _stream(stream)),
           "dllm_attention")


def dllm_get_device_status(stream=None) -> int:
    return load().dllm_get_device_status(_stream(stream))


def dllm_status_string(code: int) -> str:
    return status_string(code)


def dllm_debug_subblock_dots(w, qtype: int, N: int, K: int, q, M: int, dots, stream=None):
    _check(load().dllm_debug_subblock_dots(_ptr(w), qtype, N, K, _ptr(q), M, _ptr(dots), _stream(stream)),
           "dllm_debug_subblock_dots")


def dllm_debug_sb_ints(w, qtype: int, N: int, K: int, q, scale, sums, M: int, S, stream=None):
    _check(load().dllm_debug_sb_ints(_ptr(w), qtype, N, K, _ptr(q), _ptr(scale), _ptr(sums), M, _ptr(S),
                                     _stream(stream)), "dllm_debug_sb_ints")


def dllm_debug_bounded_wait(stream=None):
    _check(load().dllm_debug_bounded_wait(_stream(stream)), "dllm_debug_bounded_wait")


def dllm_debug_attention_stall(two_tiles: bool, stream=None):
    _check(load().dllm_debug_attention_stall(1 if two_tiles else 0, _stream(stream)), "dllm_debug_attention_stall")


def dllm_bench_mma_i8(n: int, n_acc: int, a_from_tmem: int, issuers: int, iters: int, ctas: int, ns_out,
                      stream=None):
    _check(load().dllm_bench_mma_i8(n, n_acc, a_from_tmem, issuers, iters, ctas, _ptr(ns_out), _stream(stream)),
           "dllm_bench_mma_i8")


# ------------------------------------------------------------------ small conveniences (allocation via torch)

def repack(qtype: int, blocks, N: int, K: int, device="cuda", stream=None):
    """GGUF blocks (numpy uint8 [N, K/256, bytes] or a device tensor) -> repacked device tensor."""
    import torch
    if not isinstance(blocks, torch.Tensor):
        blocks = torch.from_numpy(blocks.reshape(-1).copy())
    src = blocks.reshape(-1).to(device)
    dst = torch.empty(dllm_repacked_bytes(qtype, N, K), dtype=torch.uint8, device=device)
    fn = {DLLM_Q4_K: dllm_repack_q4k, DLLM_Q5_K: dllm_repack_q5k, DLLM_Q6_K: dllm_repack_q6k,
          DLLM_Q8_0: dllm_repack_q80}[qtype]
    fn(src, N, K, dst, stream)
    return dst


def alloc_workspace(nbytes: int, device="cuda"):
    """A zero-filled device workspace of at least nbytes (None when nbytes is 0)."""
    import torch
    if nbytes == 0:
        return None
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def alloc_act(M: int, K: int, device="cuda"):
    """Device buffers (q, scale, sums) for M x K quantized activations."""
    import torch
    qb, sb, ub = dllm_act_bytes(M, K)
    return (torch.empty(qb, dtype=torch.int8, device=device),
            torch.empty(sb // 4, dtype=torch.float32, device=device),
            torch.empty(ub // 4, dtype=torch.float32, device=device))


def dllm_debug_plan(n_tiles: int, K: int, M: int, n_rows: int, sms: int) -> dict:
    """The GEMM's work split for a shape (host only): see include/dllm_qgemm.h."""
    out = (ctypes.c_int64 * 8)()
    _check(load().dllm_debug_plan(n_tiles, K, M, n_rows, sms, out), "dllm_debug_plan")
    keys = ("kc", "full_tiles", "tail_k", "tail_big", "n_units", "n_st", "mu", "bytes")
    return dict(zip(keys, list(out)))


def dllm_debug_attention_tiles(Lq: int, H: int, sms: int) -> int:
    """Query tiles per CTA dllm_attention uses (host only): see include/dllm_qgemm.h."""
    rc = load().dllm_debug_attention_tiles(Lq, H, sms)
    if rc < 0:
        _check(rc, "dllm_debug_attention_tiles")
    return rc
