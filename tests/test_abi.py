"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/la2.h declares, and rejects bad arguments synchronously (before any
CUDA call)."""
import ctypes
import os
import re

import pytest

from causal_linear_attention_la2_b200 import la2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "la2.h")


@pytest.fixture(scope="module")
def lib():
    from causal_linear_attention_la2_b200 import build
    build.build()
    return la2.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(la2_[a-z_]+)\s*\(", text)))


def test_header_declares_the_python_export_list():
    assert _declared_functions() == sorted(la2.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    names = {0: "LA2_OK", 1: "LA2_ERR_INVALID_ARG", 2: "LA2_ERR_UNSUPPORTED",
             3: "LA2_ERR_WORKSPACE", 4: "LA2_ERR_CUDA", 5: "LA2_ERR_TIMEOUT"}
    for code, name in names.items():
        assert la2.la2_status_str(code) == name
    assert la2.la2_status_str(99) == "LA2_UNKNOWN_STATUS"


FAKE = 1 << 20  # a 16-byte aligned non-null value; validation fails before it is used


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, decay=FAKE, out=FAKE, B=1, H=2, T=256, d=128, e=128,
             block=128, dtype=la2.LA2_DTYPE_BF16)
    a.update(kw)
    return la2.la2_fwd_raw(a["q"], a["k"], a["v"], a["decay"], a["out"], a["B"], a["H"], a["T"],
                           a["d"], a["e"], a["block"], a["dtype"])


def _bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, decay=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, H=2,
             T=256, d=128, e=128, block=128, dtype=la2.LA2_DTYPE_BF16)
    a.update(kw)
    return la2.la2_bwd_raw(a["q"], a["k"], a["v"], a["decay"], a["dout"], a["dq"], a["dk"],
                           a["dv"], a["B"], a["H"], a["T"], a["d"], a["e"], a["block"], a["dtype"])


@pytest.mark.parametrize("kw", [dict(block=100), dict(block=0), dict(dtype=7), dict(B=-1),
                                dict(H=-2), dict(T=-5), dict(d=0), dict(e=-1)])
def test_invalid_arguments(lib, kw):
    assert _fwd(**kw) == la2.LA2_ERR_INVALID_ARG
    assert _bwd(**kw) == la2.LA2_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["q", "k", "v", "decay", "out"])
def test_null_pointers_forward(lib, name):
    assert _fwd(**{name: 0}) == la2.LA2_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["q", "k", "v", "decay", "dout", "dq", "dk", "dv"])
def test_null_pointers_backward(lib, name):
    assert _bwd(**{name: 0}) == la2.LA2_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["q", "k", "v", "out"])
def test_misaligned_pointers(lib, name):
    assert _fwd(**{name: FAKE + 8}) == la2.LA2_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(d=96), dict(e=32), dict(d=256)])
def test_bf16_unsupported_shapes(lib, kw):
    assert _fwd(**kw) == la2.LA2_ERR_UNSUPPORTED
    assert _bwd(**kw) == la2.LA2_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(d=129), dict(e=200)])
def test_f32_unsupported_shapes(lib, kw):
    assert _fwd(dtype=la2.LA2_DTYPE_F32, **kw) == la2.LA2_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(T=0)])
def test_empty_problem_is_ok_and_touches_nothing(lib, kw):
    # null pointers are fine for an empty problem: nothing is dereferenced or launched
    assert _fwd(q=0, k=0, v=0, decay=0, out=0, **kw) == la2.LA2_OK
    assert _bwd(q=0, k=0, v=0, decay=0, dout=0, dq=0, dk=0, dv=0, **kw) == la2.LA2_OK
    assert la2.la2_last_launch_count() == 0


@pytest.mark.parametrize("schedule", ["auto", "uniform", "balanced"])
def test_workspace_is_flat_in_T_and_bounded(lib, schedule):
    # the same size for every T, and at most 147 fp32 d x e segment states per
    # group of roles with one (d, e)
    prev = la2.la2_set_schedule(schedule)
    try:
        for B, H in ((1, 16), (1, 1), (3, 7), (64, 64)):
            for d, e in ((64, 64), (128, 128), (64, 128)):
                groups = 1 if d == e else 2
                for is_bwd in (0, 1):
                    sizes = {la2.la2_workspace_bytes(B, H, T, d, e, 128, la2.LA2_DTYPE_BF16, is_bwd)
                             for T in (1, 129, 1024, 65536, 1 << 20)}
                    assert len(sizes) == 1, (B, H, d, e, is_bwd, sizes)
                    n = sizes.pop()
                    assert 0 <= n <= groups * (147 * d * e * 4 + 256), (B, H, d, e, is_bwd, n)
    finally:
        la2.la2_set_schedule(prev)
    assert la2.la2_workspace_bytes(1, 16, 1024, 128, 128, 100, la2.LA2_DTYPE_BF16, 0) == 2 ** 64 - 1


def test_schedule_setting_round_trips(lib):
    prev = la2.la2_set_schedule("balanced")
    try:
        assert la2.la2_set_schedule("uniform") == "balanced"
        assert la2.la2_set_schedule("auto") == "uniform"
        # an unknown value leaves the setting as it is
        assert int(la2.load().la2_set_schedule(7)) == la2.LA2_SCHEDULE_AUTO
        assert la2.la2_set_schedule("auto") == "auto"
    finally:
        la2.la2_set_schedule(prev)


def test_workspace_missing_or_small_is_reported(lib):
    need = la2.la2_workspace_bytes(1, 2, 4096, 128, 128, 128, la2.LA2_DTYPE_BF16, 0)
    assert need > 0  # two sequences: they are cut into segments
    assert _fwd(T=4096) == la2.LA2_ERR_WORKSPACE
    assert la2.la2_fwd_raw(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 4096, 128, 128, 128,
                           la2.LA2_DTYPE_BF16, FAKE, need - 1) == la2.LA2_ERR_WORKSPACE
    assert la2.la2_fwd_raw(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 4096, 128, 128, 128,
                           la2.LA2_DTYPE_BF16, FAKE + 16, need) == la2.LA2_ERR_INVALID_ARG


def test_no_workspace_when_the_grid_is_full(lib):
    # 2 x 40 x 3 backward units >= 148 SMs: no segments, no workspace
    assert la2.la2_workspace_bytes(2, 40, 6144, 128, 128, 128, la2.LA2_DTYPE_BF16, 1) == 0
    assert la2.la2_workspace_bytes(1, 2, 512, 64, 64, 64, la2.LA2_DTYPE_F32, 1) == 0


def test_plan_info(lib):
    prev = la2.la2_set_schedule("uniform")
    try:
        # long-context forward: 16 units of 512 tiles, cut into 9 segments of 57 tiles
        assert la2.la2_plan_info(1, 16, 65536, 128, 128) == [
            {"d": 128, "e": 128, "schedule": "uniform", "units": 16, "segments": 9, "tiles_per_cta": 57,
             "ctas": 144, "prepass_ctas": 128}]
        # its backward: 48 units in 3 segments of 171 tiles
        assert la2.la2_plan_info(1, 16, 65536, 128, 128, is_bwd=True)[0]["segments"] == 3
    finally:
        la2.la2_set_schedule(prev)
    # 15B backward: 240 units fill the GPU, no segments, no pre-pass
    p = la2.la2_plan_info(2, 40, 6144, 128, 128, is_bwd=True)
    assert len(p) == 1 and p[0]["units"] == 240 and p[0]["ctas"] == 240 and p[0]["prepass_ctas"] == 0
    # d != e backward: dq and dk (a, b of width e) in one launch, dv in another
    p = la2.la2_plan_info(2, 3, 1000, 64, 128, is_bwd=True)
    assert [(g["d"], g["e"], g["units"]) for g in p] == [(128, 64, 12), (64, 128, 6)]
    # fp32 inputs and empty problems have no plan; bad arguments are rejected
    assert la2.la2_plan_info(1, 2, 512, 64, 64, 64, la2.LA2_DTYPE_F32) == []
    assert la2.la2_plan_info(0, 2, 512, 64, 64) == []
    with pytest.raises(la2.LA2Error):
        la2.la2_plan_info(1, 2, 512, 64, 64, 100)
    prev = la2.la2_set_schedule("balanced")
    try:
        # 80 units x 48 tiles laid end to end: runs of 26 tiles on 148 CTAs
        assert la2.la2_plan_info(2, 40, 6144, 128, 128) == [
            {"d": 128, "e": 128, "schedule": "balanced", "units": 80, "segments": 0, "tiles_per_cta": 26,
             "ctas": 148, "prepass_ctas": 147}]
    finally:
        la2.la2_set_schedule(prev)


def test_selftest_timeout_rejects_bad_arguments(lib):
    fake = FAKE
    for T, lim in ((0, 100), (257, 100), (100, 0), (100, 2_000_000)):
        assert la2.la2_selftest_timeout_raw(fake, fake, fake, fake, fake, T, 128, 128, lim) == \
            la2.LA2_ERR_INVALID_ARG
    assert la2.la2_selftest_timeout_raw(0, fake, fake, fake, fake, 100, 128, 128, 100) == \
        la2.LA2_ERR_INVALID_ARG
    assert la2.la2_selftest_timeout_raw(fake, fake, fake, fake, fake, 100, 96, 128, 100) == \
        la2.LA2_ERR_UNSUPPORTED


def test_bwd_state_rejects_misaligned_states(lib):
    for pos in range(3):
        st = [0, 0, 0]
        st[pos] = FAKE + 2
        r = la2.load().la2_bwd_state(FAKE, FAKE, FAKE, FAKE, FAKE, st[0], st[1], FAKE, FAKE, FAKE,
                                     st[2], 1, 2, 256, 128, 128, 128, la2.LA2_DTYPE_BF16,
                                     la2.LA2_DTYPE_F32, la2.LA2_LAYOUT_BHTD, 0, 0, 0)
        assert r == la2.LA2_ERR_INVALID_ARG


def test_dlambda_workspace_flat_in_T_and_arguments(lib):
    sizes = {la2.la2_dlambda_workspace_bytes(1, 16, T, 128, 128, la2.LA2_DTYPE_BF16)
             for T in (1000, 65536, 1 << 20)}
    assert len(sizes) == 1 and sizes.pop() > 0
    assert la2.la2_dlambda_workspace_bytes(1, 2, 100, 129, 64, la2.LA2_DTYPE_F32) == 2 ** 64 - 1
    assert la2.la2_dlambda_workspace_bytes(1, 2, 0, 64, 64, la2.LA2_DTYPE_F32) == 0
    f = la2.load().la2_dlambda
    ok = dict(B=1, H=2, T=100, d=64, e=64)
    # misaligned element pointer, NULL input, missing workspace, bad layout
    assert f(FAKE + 1, FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 2, 100, 64, 64, la2.LA2_DTYPE_BF16, 0,
             FAKE, 1 << 30, 0) == la2.LA2_ERR_INVALID_ARG
    assert f(0, FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 2, 100, 64, 64, la2.LA2_DTYPE_BF16, 0,
             FAKE, 1 << 30, 0) == la2.LA2_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 2, 100, 64, 64, la2.LA2_DTYPE_BF16, 0,
             0, 0, 0) == la2.LA2_ERR_WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 2, 100, 64, 64, la2.LA2_DTYPE_BF16, 7,
             FAKE, 1 << 30, 0) == la2.LA2_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 2, 100, 200, 64, la2.LA2_DTYPE_BF16, 0,
             FAKE, 1 << 30, 0) == la2.LA2_ERR_UNSUPPORTED
    del ok


def test_norm_workspace_and_arguments(lib):
    ws = [la2.la2_norm_workspace_bytes(1, 8, T, 128, 128, 128, la2.LA2_DTYPE_BF16, 0)
          for T in (4096, 65536)]
    assert ws[0] == ws[1]                       # the forward's is flat in T
    assert la2.la2_norm_workspace_bytes(1, 8, 64, 129, 64, 128, la2.LA2_DTYPE_F32, 0) == 2 ** 64 - 1
    f = la2.load().la2_fwd_norm
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 128, 128, 128, la2.LA2_DTYPE_BF16, 5,
             FAKE, 1 << 30, 0) == la2.LA2_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, 0, FAKE, 1, 2, 256, 128, 128, 128, la2.LA2_DTYPE_BF16, 0,
             FAKE, 1 << 30, 0) == la2.LA2_ERR_INVALID_ARG
    g = la2.load().la2_bwd_norm
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 128, 128, 128,
             la2.LA2_DTYPE_BF16, 0, 0, 0, 0) == la2.LA2_ERR_WORKSPACE


@pytest.mark.parametrize("block", [64, 256])
def test_bf16_other_blocks_need_no_workspace(lib, block):
    assert la2.la2_workspace_bytes(1, 2, 65536, 128, 128, block, la2.LA2_DTYPE_BF16, 0) == 0
    assert la2.la2_workspace_bytes(1, 2, 65536, 128, 128, block, la2.LA2_DTYPE_BF16, 1) == 0
    plan = la2.la2_plan_info(1, 2, 1000, 128, 64, block, is_bwd=True)
    # one CTA per (sequence, role, 64 value columns), one segment each
    assert [(g["ctas"], g["segments"], g["prepass_ctas"]) for g in plan] == [(8, 1, 0), (2, 1, 0)]


@pytest.mark.parametrize("call", ["fwd_ex", "bwd_ex", "bwd_state"])
def test_out_dtype_arguments(lib, call):
    """An unknown output type is an argument error; bf16 outputs need bf16
    inputs (UNSUPPORTED for fp32 inputs, reported before anything is read)."""
    L = la2.load()
    bf, f32, lay = la2.LA2_DTYPE_BF16, la2.LA2_DTYPE_F32, la2.LA2_LAYOUT_BHTD

    def go(dtype, out_dtype):
        if call == "fwd_ex":
            return L.la2_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, 1, 2, 256, 128, 128, 128, dtype,
                                out_dtype, lay, 0, 0, 0)
        if call == "bwd_ex":
            return L.la2_bwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 128, 128,
                                128, dtype, out_dtype, lay, 0, 0, 0)
        return L.la2_bwd_state(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, FAKE, FAKE, 0, 1, 2, 256,
                               128, 128, 128, dtype, out_dtype, lay, 0, 0, 0)

    assert go(bf, 2) == la2.LA2_ERR_INVALID_ARG
    assert go(bf, -1) == la2.LA2_ERR_INVALID_ARG
    assert go(f32, bf) == la2.LA2_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,H,T,is_bwd,want", [
    (2, 32, 65536, 1, "balanced"),   # 192 units of 512 tiles: uniform's second wave is 44 CTAs
    (3, 50, 16384, 0, "balanced"),   # 150 units of 128 tiles: a second wave of 2 CTAs
    (2, 32, 65536, 0, "uniform"),    # 64 units, cut into 2 segments each
    (1, 16, 65536, 0, "uniform"),    # long forward: 16 units in 9 segments
    (1, 32, 131072, 0, "uniform"),   # 32 units in 4 segments
    (1, 32, 131072, 1, "uniform"),   # 96 units of 1024 tiles, one wave
    (4, 32, 32768, 0, "uniform"),    # 128 units of 256 tiles in one wave
    (4, 32, 32768, 1, "uniform"),    # 384 units, three waves 86% full
    (2, 40, 6144, 0, "uniform"),     # 15B forward: 80 units of only 48 tiles
    (2, 40, 6144, 1, "uniform"),     # 15B backward: 240 units of 48 tiles
    (8, 16, 2048, 1, "uniform"),     # TNL-400M backward
    (128, 32, 1024, 0, "uniform"),   # 4096 short units
])
def test_auto_schedule_choice(lib, B, H, T, is_bwd, want):
    """AUTO takes the balanced plan for >= 148 units of >= 128 tiles whose
    uniform waves leave over a quarter of their SM time idle, the uniform plan
    elsewhere; its workspace covers the plan it takes."""
    prev = la2.la2_set_schedule("auto")
    try:
        p = la2.la2_plan_info(B, H, T, 128, 128, is_bwd=bool(is_bwd))
        assert [g["schedule"] for g in p] == [want]
        if want == "balanced":
            assert p[0]["ctas"] <= 148
            ws = la2.la2_workspace_bytes(B, H, T, 128, 128, 128, la2.LA2_DTYPE_BF16, is_bwd)
            assert ws >= 147 * 128 * 128 * 4
    finally:
        la2.la2_set_schedule(prev)
