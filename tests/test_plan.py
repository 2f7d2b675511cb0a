"""The GEMM's work split, checked on the host through dllm_debug_plan (no GPU).

The split decides which K range of which weight tile each work unit covers.  It must
cover every (tile, super-block, token super-tile) exactly once, keep every tail-split
piece at least 4 super-blocks long with at most 15 pieces per tile (arrival counters
advance by 16), and depend on the weight shape and SM count only, so that results do not depend on
M or on a row list.  `units` below restates the kernel's unit mapping from the plan's
fields, to check that those fields describe an exact cover.
"""
import pytest

from quantized_int8_gemm_q4_b200 import build as nbuild
from quantized_int8_gemm_q4_b200 import dllm

SMS = 148  # B200
LLADA = {"qkv": (96, 4096), "o": (32, 4096), "gate_up": (192, 4096), "down": (32, 12288), "output": (988, 4096)}
DREAM = {"qkv": (36, 3584), "o": (28, 3584), "gate_up": (296, 3584), "down": (28, 18944), "output": (1188, 3584)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    nbuild.build()
    dllm.load()


def plan(n_tiles, K, M=128, n_rows=0, sms=SMS):
    return dllm.dllm_debug_plan(n_tiles, K, M, n_rows, sms)


def units(p, n_tiles, nsb):
    """(tile, st, piece, pieces, sb0, sb1) of every unit, in unit order."""
    out = []
    for u in range(p["n_units"]):
        if p["tail_k"] == 0:
            kc = p["kc"]
            ch, ts = u % kc, u // kc
            st, t, np_ = ts % p["n_st"], ts // p["n_st"], kc
        else:
            cu, st = divmod(u, p["n_st"])
            if cu < p["full_tiles"]:
                t, ch, np_ = cu, 0, 1
            else:
                i = cu - p["full_tiles"]
                big = p["tail_big"] * (p["tail_k"] + 1)
                np_ = p["tail_k"] + 1 if i < big else p["tail_k"]
                i2 = i if i < big else i - big
                j, ch = divmod(i2, np_)
                t = p["full_tiles"] + (j if i < big else p["tail_big"] + j)
        out.append((t, st, ch, np_, ch * nsb // np_, (ch + 1) * nsb // np_))
    return out


def check_cover(p, n_tiles, nsb):
    seen = {}
    pieces = {}
    for t, st, ch, np_, sb0, sb1 in units(p, n_tiles, nsb):
        assert 0 <= t < n_tiles and 0 <= st < p["n_st"] and sb0 < sb1
        assert np_ <= 15
        if p["tail_k"] and t >= p["full_tiles"]:
            assert sb1 - sb0 >= 4  # tail pieces; uniform chunks may differ by one from nsb/kc
        pieces.setdefault((t, st), set()).add((ch, np_))
        for s in range(sb0, sb1):
            seen[(t, st, s)] = seen.get((t, st, s), 0) + 1
    assert len(seen) == n_tiles * p["n_st"] * nsb and set(seen.values()) == {1}
    for (t, st), ps in pieces.items():  # every tile's pieces are 0..np-1 of one np
        nps = {np_ for _, np_ in ps}
        assert len(nps) == 1 and {c for c, _ in ps} == set(range(nps.pop()))


@pytest.mark.parametrize("model", [LLADA, DREAM])
@pytest.mark.parametrize("M", [32, 128, 160, 1024])
def test_step_shapes_cover_exactly(model, M):
    for n_tiles, K in model.values():
        p = plan(n_tiles, K, M)
        check_cover(p, n_tiles, K // 256)


def test_llada_choices():
    got = {k: plan(*v) for k, v in LLADA.items()}
    assert got["gate_up"]["tail_k"] == 3 and got["gate_up"]["full_tiles"] == 148 and got["gate_up"]["tail_big"] == 16
    assert got["gate_up"]["n_units"] == 2 * SMS  # one whole tile and one piece per SM
    for k in ("qkv", "o", "down", "output"):
        assert got[k]["tail_k"] == 0
    assert got["qkv"]["kc"] == 1 and got["o"]["kc"] == 4 and got["down"]["kc"] == 4 and got["output"]["kc"] == 1


@pytest.mark.parametrize("shape", list(LLADA.values()) + list(DREAM.values()) + [(160, 16384), (200, 8192), (7, 256)])
def test_split_does_not_depend_on_M_or_rows(shape):
    keys = ("kc", "full_tiles", "tail_k", "tail_big")
    ref = {k: plan(*shape, M=128)[k] for k in keys}
    for M, n_rows in ((1, 0), (16, 0), (160, 0), (512, 0), (1024, 0), (160, 32), (1024, 1)):
        p = plan(*shape, M=M, n_rows=n_rows)
        assert {k: p[k] for k in keys} == ref, (M, n_rows)


def test_tail_split_balances_the_sms():
    p = plan(192, 4096)
    per_sm = [0] * SMS
    for u, (_, _, _, _, sb0, sb1) in enumerate(units(p, 192, 16)):
        per_sm[u % SMS] += sb1 - sb0
    assert max(per_sm) <= 22 and min(per_sm) >= 20  # 3072 super-blocks over 148 SMs
    # the uniform split would give 44 SMs two whole tiles (32) and the rest one (16)


def test_workspace_holds_the_partials():
    for n_tiles, K in list(LLADA.values()) + list(DREAM.values()):
        for M in (32, 128, 384):
            p = plan(n_tiles, K, M)
            per_slot = p["mu"] * 128 * 4
            if p["tail_k"]:
                assert p["bytes"] >= SMS * p["n_st"] * per_slot + n_tiles * p["n_st"] * 4
            elif p["kc"] > 1:
                assert p["bytes"] >= n_tiles * p["n_st"] * p["kc"] * per_slot + n_tiles * p["n_st"] * 4
            else:
                assert p["bytes"] == 0


@pytest.mark.parametrize("n_tiles", [1, 5, 100, 149, 150, 200, 250, 295, 297, 400, 1000])
@pytest.mark.parametrize("nsb", [1, 3, 4, 14, 16, 48, 74])
def test_any_shape_covers_exactly(n_tiles, nsb):
    p = plan(n_tiles, nsb * 256)
    check_cover(p, n_tiles, nsb)


def test_bad_arguments():
    with pytest.raises(dllm.DllmError):
        plan(0, 4096)
    with pytest.raises(dllm.DllmError):
        plan(10, 300)
    with pytest.raises(dllm.DllmError):
        plan(10, 4096, n_rows=33)


@pytest.mark.parametrize("Lq,H,sms,want", [
    (1, 1, SMS, 1), (1024, 32, SMS, 2), (1024, 28, SMS, 2), (4096, 32, SMS, 2), (512, 32, SMS, 1),
    (640, 28, SMS, 1), (160, 32, SMS, 1), (128, 148, SMS, 1), (128, 149, SMS, 2), (129, 74, SMS, 1),
    (129, 75, SMS, 2), (1024, 32, 256, 1), (1024, 32, 255, 2),
])
def test_attention_takes_two_tiles_per_cta_beyond_one_wave(Lq, H, sms, want):
    """dllm_attention runs one query tile per CTA while ceil(Lq / 128) * H CTAs fit one
    wave on the SMs, two (ping-pong) beyond that."""
    assert dllm.dllm_debug_attention_tiles(Lq, H, sms) == want


@pytest.mark.parametrize("Lq,H,sms", [(0, 32, SMS), (1024, 0, SMS), (1024, 32, 0), (-5, 1, 1)])
def test_attention_tiles_rejects_bad_arguments(Lq, H, sms):
    with pytest.raises(dllm.DllmError) as e:
        dllm.dllm_debug_attention_tiles(Lq, H, sms)
    assert e.value.code == dllm.DLLM_ERR_ARG
