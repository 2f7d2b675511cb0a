"""C-ABI checks that need no GPU: the library builds and loads, exports every entry
point include/*.h declares, and rejects bad arguments on the host before any launch.
No compute call is made here."""
import ctypes
import re
from pathlib import Path

import pytest

from quantized_int8_gemm_q4_b200 import build as nbuild
from quantized_int8_gemm_q4_b200 import dllm

ROOT = Path(__file__).resolve().parent.parent


@pytest.fixture(scope="module")
def lib():
    nbuild.build()
    return dllm.load()


def declared_symbols():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        text = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names |= set(re.findall(r"\b(dllm_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for must in ("dllm_repack_q4k", "dllm_repack_q6k", "dllm_quantize_act", "dllm_qgemm", "dllm_qkv_qgemm",
                 "dllm_rmsnorm_quantize", "dllm_swiglu_quantize", "dllm_get_device_status", "dllm_status_string", "dllm_debug_subblock_dots"):
        assert must in syms


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) <= set(dllm.EXPORTS) | {"dllm_repacked_bytes"}


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9):
        assert dllm.status_string(code) not in ("", "unknown status")
    assert dllm.status_string(-99) == "unknown status"


def test_sizes_on_host(lib):
    assert dllm.dllm_repacked_bytes(dllm.DLLM_Q4_K, 256, 512) == 256 * 2 * 144
    assert dllm.dllm_repacked_bytes(dllm.DLLM_Q6_K, 128, 4096) == 128 * 16 * 210
    q, s, u = dllm.dllm_act_bytes(17, 512)
    assert (q, s, u) == (32 * 512, 32 * 2 * 4, 32 * 2 * 64)


@pytest.mark.parametrize("N,K", [(100, 512), (128, 300), (0, 256), (128, 0), (-128, 256)])
def test_bad_shapes_rejected(lib, N, K):
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_repacked_bytes(dllm.DLLM_Q4_K, N, K)
    assert e.value.code == dllm.DLLM_ERR_ARG


def test_bad_qtype_rejected(lib):
    out = ctypes.c_size_t(0)
    for t in (0, 2, 9, 10, 11, 15):
        assert lib.dllm_repacked_bytes(t, 128, 256, ctypes.byref(out)) == dllm.DLLM_ERR_ARG


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_gemm_argument_checks_before_launch(lib):
    A = 0x10000  # never dereferenced: validation fails first
    args = dict(w=_fake(A), t=dllm.DLLM_Q4_K, N=256, K=512, q=_fake(A), s=_fake(A), u=_fake(A), M=64,
                rows=None, n_rows=0, out=_fake(A), ldo=256)

    def call(**kw):
        a = {**args, **kw}
        return lib.dllm_qgemm(a["w"], a["t"], a["N"], a["K"], a["q"], a["s"], a["u"], a["M"], a["rows"],
                              a["n_rows"], a["out"], a["ldo"], None, 0, None)

    assert call(K=300) == dllm.DLLM_ERR_ARG
    assert call(N=200) == dllm.DLLM_ERR_ARG
    assert call(M=0) == dllm.DLLM_ERR_ARG
    assert call(ldo=128) == dllm.DLLM_ERR_ARG
    assert call(w=None) == dllm.DLLM_ERR_ARG
    assert call(q=None) == dllm.DLLM_ERR_ARG
    assert call(q=_fake(A + 4)) == dllm.DLLM_ERR_ALIGN
    assert call(out=_fake(A + 8)) == dllm.DLLM_ERR_ALIGN
    assert call(ldo=258) == dllm.DLLM_ERR_ALIGN
    assert call(rows=_fake(A), n_rows=0) == dllm.DLLM_ERR_ARG
    assert call(rows=_fake(A), n_rows=33) == dllm.DLLM_ERR_ARG
    assert call(t=9) == dllm.DLLM_ERR_ARG
    assert call(t=dllm.DLLM_Q8_0, K=300) == dllm.DLLM_ERR_ARG


def test_quantize_argument_checks(lib):
    A = 0x10000
    f = lib.dllm_quantize_act
    assert f(None, 4, 256, 256, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert f(_fake(A), 4, 300, 300, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert f(_fake(A), 4, 256, 128, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert f(_fake(A + 4), 4, 256, 256, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ALIGN
    assert f(_fake(A), 4, 256, 258, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ALIGN


def test_fused_quantize_argument_checks(lib):
    A = 0x10000
    f = lib.dllm_rmsnorm_quantize
    ok = (_fake(A), 4, 256, 256, _fake(A), 1e-5, None, 0, _fake(A), _fake(A), _fake(A), None)

    def rms(**kw):
        a = list(ok)
        for i, k in enumerate(("x", "M", "K", "ldx", "gamma", "eps", "rows", "n_rows", "q", "scale", "sums")):
            if k in kw:
                a[i] = kw[k]
        return f(*a)
    assert rms(x=None) == dllm.DLLM_ERR_ARG
    assert rms(gamma=None) == dllm.DLLM_ERR_ARG
    assert rms(K=300, ldx=300) == dllm.DLLM_ERR_ARG
    assert rms(ldx=128) == dllm.DLLM_ERR_ARG
    assert rms(K=65536 + 256, ldx=65536 + 256) == dllm.DLLM_ERR_ARG   # the documented K <= 65536
    assert rms(M=0) == dllm.DLLM_ERR_ARG
    assert rms(eps=0.0) == dllm.DLLM_ERR_ARG
    assert rms(eps=-1e-5) == dllm.DLLM_ERR_ARG
    assert rms(eps=float("inf")) == dllm.DLLM_ERR_ARG
    assert rms(eps=float("nan")) == dllm.DLLM_ERR_ARG
    assert rms(x=_fake(A + 4)) == dllm.DLLM_ERR_ALIGN
    assert rms(gamma=_fake(A + 8)) == dllm.DLLM_ERR_ALIGN
    assert rms(ldx=258) == dllm.DLLM_ERR_ALIGN
    assert rms(q=_fake(A + 1)) == dllm.DLLM_ERR_ALIGN
    assert rms(rows=_fake(A), n_rows=0) == dllm.DLLM_ERR_ARG      # a row list needs n_rows >= 1
    assert rms(rows=_fake(A), n_rows=-3) == dllm.DLLM_ERR_ARG
    assert rms(rows=None, n_rows=5) == dllm.DLLM_ERR_ARG          # n_rows without a list
    assert rms(rows=_fake(A + 4), n_rows=2) == dllm.DLLM_ERR_ALIGN
    g = lib.dllm_swiglu_quantize
    assert g(None, _fake(A), 4, 256, 256, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert g(_fake(A), None, 4, 256, 256, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert g(_fake(A), _fake(A), 4, 256, 128, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert g(_fake(A), _fake(A), 4, 260, 512, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert g(_fake(A), _fake(A), 0, 256, 256, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ARG
    assert g(_fake(A), _fake(A + 4), 4, 256, 256, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ALIGN
    assert g(_fake(A), _fake(A), 4, 256, 514, _fake(A), _fake(A), _fake(A), None) == dllm.DLLM_ERR_ALIGN
    assert g(_fake(A), _fake(A), 4, 256, 256, _fake(A), _fake(A + 2), _fake(A), None) == dllm.DLLM_ERR_ALIGN


def test_repack_rejects_overlap(lib):
    A = 0x10000
    assert lib.dllm_repack_q4k(_fake(A), 128, 256, _fake(A + 16), None) == dllm.DLLM_ERR_ARG


def test_qkv_argument_checks(lib):
    A = 0x10000
    f = lib.dllm_qkv_qgemm
    ok = f(_fake(A), _fake(A), None, dllm.DLLM_Q4_K, 256, 100, 512, _fake(A), _fake(A), _fake(A), 16,
           _fake(A), 256, _fake(A), None, 128, None, 0, None)
    assert ok == dllm.DLLM_ERR_ARG


def test_q80_repacked_size_is_the_gguf_size(lib):
    """Q8_0 keeps its 272 bytes per 256 weights (codes plane, then block scales)."""
    out = ctypes.c_size_t(0)
    assert lib.dllm_repacked_bytes(dllm.DLLM_Q8_0, 384, 4096, ctypes.byref(out)) == dllm.DLLM_OK
    assert out.value == 384 * 16 * 272
    assert lib.dllm_repacked_bytes(dllm.DLLM_Q8_0, 100, 4096, ctypes.byref(out)) == dllm.DLLM_ERR_ARG


def test_q5k_repacked_size_is_the_split_form(lib):
    """Q5_K keeps two Q4_K-form super-blocks (2 x 144 bytes) per 256 weights."""
    out = ctypes.c_size_t(0)
    assert lib.dllm_repacked_bytes(dllm.DLLM_Q5_K, 256, 4096, ctypes.byref(out)) == dllm.DLLM_OK
    assert out.value == 256 * 16 * 288
