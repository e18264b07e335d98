"""CPU-only checks of the C-ABI library: it builds for sm_100a, loads, exports
every symbol include/fa.h declares, and rejects bad arguments synchronously
(these calls return before touching CUDA, so no GPU is needed)."""
import ctypes
import math

import pytest

import io_aware_exact_18_b200 as fa
from io_aware_exact_18_b200 import build as fa_build


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def test_header_declares_the_boundary():
    assert fa.declared_symbols() == ["fa_bwd", "fa_bwd_workspace_bytes",
                                     "fa_fwd", "fa_fwd_fp8", "fa_fwd_gqa", "fa_fwd_kvlen",
                                     "fa_fwd_splitkv", "fa_fwd_splitkv_fp8",
                                     "fa_fwd_splitkv_static",
                                     "fa_last_device_error",
                                     "fa_splitkv_default_splits",
                                     "fa_splitkv_workspace_bytes", "fa_status_string",
                                     "fa_watchdog_selftest"]


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(fa.LIB_PATH)
    for name in fa.declared_symbols():
        assert hasattr(raw, name), name


def test_library_is_built_for_sm100a(lib):
    log = open(fa_build.os.path.join(fa_build.PKG, "build.log")).read()
    assert "arch=compute_100a,code=sm_100a" in log
    assert "fa_fwd_sm100" in log  # ptxas compiled the kernel entry points


def test_status_strings(lib):
    assert fa.fa_status_string(fa.FA_OK) == "FA_OK"
    for s in (fa.FA_ERR_INVALID_ARG, fa.FA_ERR_UNSUPPORTED, fa.FA_ERR_LAUNCH, fa.FA_ERR_TIMEOUT):
        assert fa.fa_status_string(s).startswith("FA_ERR_")
    assert fa.fa_status_string(12345) == "unknown fa status"


# Fake, never-dereferenced device addresses: validation runs before any CUDA call.
P = 1 << 40
GOOD = dict(q=P, k=P + (1 << 30), v=P + (2 << 30), o=P + (3 << 30), lse=P + (4 << 30),
            B=1, H=2, N=256, d=64, scale=0.125, causal=0)


def call(lib, **over):
    a = dict(GOOD, **over)
    return lib.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                      a["d"], a["scale"], a["causal"], None)


@pytest.mark.parametrize("over,status", [
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(H=-3), fa.FA_ERR_INVALID_ARG),
    (dict(N=-1), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-0.1), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=192), fa.FA_ERR_UNSUPPORTED),
    (dict(d=512), fa.FA_ERR_UNSUPPORTED),
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(lse=0), fa.FA_ERR_INVALID_ARG),
    (dict(q=P + 8), fa.FA_ERR_INVALID_ARG),          # not 16-byte aligned
    (dict(o=P + (3 << 30) + 2), fa.FA_ERR_INVALID_ARG),
    (dict(lse=P + (4 << 30) + 1), fa.FA_ERR_INVALID_ARG),
    (dict(o=P), fa.FA_ERR_INVALID_ARG),              # output aliases an input
    (dict(lse=P + (3 << 30) + 64), fa.FA_ERR_INVALID_ARG),  # lse inside o
    (dict(B=1 << 20, H=1 << 12), fa.FA_ERR_INVALID_ARG),    # grid too large
])
def test_argument_errors_are_synchronous(lib, over, status):
    assert call(lib, **over) == status


@pytest.mark.parametrize("over", [dict(B=0), dict(H=0), dict(N=0),
                                  dict(B=0, q=0, k=0, v=0, o=0, lse=0)])
def test_empty_problem_is_a_no_op(lib, over):
    assert call(lib, **over) == fa.FA_OK


def test_kvlen_pointer_alignment(lib):
    a = GOOD
    st = lib.fa_fwd_kvlen(a["q"], a["k"], a["v"], a["o"], a["lse"], 1, 2, 256, 64, 0.125, 0,
                          P + (5 << 30) + 2, None)
    assert st == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("H,H_kv,status", [(8, 0, fa.FA_ERR_INVALID_ARG),
                                            (8, 3, fa.FA_ERR_INVALID_ARG),
                                            (8, 16, fa.FA_ERR_INVALID_ARG),
                                            (8, -1, fa.FA_ERR_INVALID_ARG),
                                            (0, 0, fa.FA_OK)])
def test_gqa_head_arguments(lib, H, H_kv, status):
    a = GOOD
    st = lib.fa_fwd_gqa(a["q"], a["k"], a["v"], a["o"], a["lse"], 1, H, H_kv, 256, 64, 0.125,
                        0, None, None)
    assert st == status


@pytest.mark.parametrize("limit", [0, 999, 5_000_000_001])
def test_watchdog_selftest_rejects_bad_limits(lib, limit):
    assert lib.fa_watchdog_selftest(limit, None) == fa.FA_ERR_INVALID_ARG


def test_python_wrapper_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.attention(x, x, x)
    with pytest.raises(TypeError):
        fa.attention(x.float(), x.float(), x.float())
    assert math.isclose(1 / math.sqrt(64), 0.125)


# ---------------------------------------------------------------- split-KV
WS = P + (6 << 30)
SK = dict(q=P, k=P + (1 << 30), v=P + (2 << 30), o=P + (3 << 30), lse=P + (4 << 30),
          B=2, H=8, H_kv=2, Nq=3, Nk=1000, d=128, scale=0.088, causal=1, kv_len=None,
          splits=4, ws=WS, ws_bytes=1 << 30)


def call_splitkv(lib, **over):
    a = dict(SK, **over)
    return lib.fa_fwd_splitkv(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                              a["H_kv"], a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"],
                              a["kv_len"], a["splits"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("over,status", [
    (dict(Nq=1001), fa.FA_ERR_INVALID_ARG),          # more queries than keys
    (dict(Nq=-1), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=-1, Nq=0), fa.FA_ERR_INVALID_ARG),
    (dict(splits=0), fa.FA_ERR_INVALID_ARG),
    (dict(splits=129), fa.FA_ERR_INVALID_ARG),        # above FA_MAX_SPLITS
    (dict(ws=0), fa.FA_ERR_INVALID_ARG),              # splits > 1 needs a workspace
    (dict(ws_bytes=1000), fa.FA_ERR_INVALID_ARG),     # too small
    (dict(ws=WS + 8), fa.FA_ERR_INVALID_ARG),         # misaligned
    (dict(ws=P + (3 << 30)), fa.FA_ERR_INVALID_ARG),  # overlaps o
    (dict(H_kv=3), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=0), fa.FA_OK),                            # empty: nothing launched
    (dict(B=0, q=0, k=0, v=0, o=0, lse=0, ws=0), fa.FA_OK),
])
def test_splitkv_argument_errors_are_synchronous(lib, over, status):
    assert call_splitkv(lib, **over) == status


def test_splitkv_workspace_bytes(lib):
    B, H, Nq, d = 2, 8, 3, 128
    assert lib.fa_splitkv_workspace_bytes(B, H, Nq, d, 1) == 0
    for s in (2, 7, 128):
        o_bytes = s * B * H * Nq * d * 4
        o_bytes = (o_bytes + 255) // 256 * 256
        assert lib.fa_splitkv_workspace_bytes(B, H, Nq, d, s) == o_bytes + s * B * H * Nq * 4
    assert lib.fa_splitkv_workspace_bytes(B, H, Nq, d, 0) == 0
    assert lib.fa_splitkv_workspace_bytes(B, H, Nq, d, 129) == 0
    assert lib.fa_splitkv_workspace_bytes(-1, H, Nq, d, 2) == 0


def test_splitkv_default_splits_in_range(lib):
    for args in [(1, 32, 8, 1, 8192, 128), (64, 32, 32, 1, 512, 128), (1, 1, 1, 1, 1, 64),
                 (1, 32, 8, 1, 1 << 20, 128)]:
        s = lib.fa_splitkv_default_splits(*args)
        assert 1 <= s <= 128, (args, s)
    assert lib.fa_splitkv_default_splits(0, 32, 8, 1, 8192, 128) == 1


# ---------------------------------------------------------------- backward
BW = dict(q=P, k=P + (1 << 30), v=P + (2 << 30), o=P + (3 << 30), lse=P + (4 << 30),
          do=P + (5 << 30), dq=P + (6 << 30), dk=P + (7 << 30), dv=P + (8 << 30),
          B=2, H=8, H_kv=2, N=300, d=128, scale=0.088, causal=1, kv_len=None,
          ws=P + (9 << 30), ws_bytes=1 << 30)


def call_bwd(lib, **over):
    a = dict(BW, **over)
    return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                      a["dv"], a["B"], a["H"], a["H_kv"], a["N"], a["d"], a["scale"],
                      a["causal"], a["kv_len"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("over,status", [
    (dict(d=256), fa.FA_ERR_UNSUPPORTED),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(N=-1), fa.FA_ERR_INVALID_ARG),
    (dict(H_kv=3), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(ws=0), fa.FA_ERR_INVALID_ARG),
    (dict(ws_bytes=1000), fa.FA_ERR_INVALID_ARG),
    (dict(ws=P + (9 << 30) + 4), fa.FA_ERR_INVALID_ARG),   # misaligned
    (dict(dq=P), fa.FA_ERR_INVALID_ARG),                   # dq is q
    (dict(dk=P + (8 << 30)), fa.FA_ERR_INVALID_ARG),       # dk is dv
    (dict(dv=P + (5 << 30) + 64), fa.FA_ERR_INVALID_ARG),  # dv inside d_o
    (dict(ws=P + (6 << 30)), fa.FA_ERR_INVALID_ARG),       # workspace is dq
    (dict(lse=P + (4 << 30) + 2), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_OK),
    (dict(B=0, q=0, k=0, v=0, o=0, lse=0, do=0, dq=0, dk=0, dv=0, ws=0), fa.FA_OK),
])
def test_bwd_argument_errors_are_synchronous(lib, over, status):
    assert call_bwd(lib, **over) == status


def test_bwd_workspace_bytes(lib):
    assert lib.fa_bwd_workspace_bytes(2, 8, 300) == 2 * 2 * 8 * 384 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 128) == 2 * 128 * 4
    assert lib.fa_bwd_workspace_bytes(-1, 1, 1) == 0


# ---------------------------------------------------------------- e4m3 forward
@pytest.mark.parametrize("over,status", [
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(d=512), fa.FA_ERR_UNSUPPORTED),
    (dict(qs=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(ks=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(vs=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(vs=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(H_kv=3), fa.FA_ERR_INVALID_ARG),
    (dict(o=P), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_OK),
])
def test_fp8_argument_errors_are_synchronous(lib, over, status):
    a = dict(q=P, k=P + (1 << 30), v=P + (2 << 30), o=P + (3 << 30), lse=P + (4 << 30),
             qs=0.01, ks=0.01, vs=0.01, B=1, H=8, H_kv=2, N=300, d=128, scale=0.088,
             causal=1)
    a.update(over)
    st = lib.fa_fwd_fp8(a["q"], a["k"], a["v"], a["qs"], a["ks"], a["vs"], a["o"], a["lse"],
                        a["B"], a["H"], a["H_kv"], a["N"], a["d"], a["scale"], a["causal"],
                        None, None)
    assert st == status


@pytest.mark.parametrize("over,status", [
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(qs=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(vs=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=513), fa.FA_ERR_INVALID_ARG),            # more queries than keys
    (dict(splits=0), fa.FA_ERR_INVALID_ARG),
    (dict(splits=129), fa.FA_ERR_INVALID_ARG),
    (dict(ws=None), fa.FA_ERR_INVALID_ARG),           # splits > 1 needs a workspace
    (dict(ws_bytes=16), fa.FA_ERR_INVALID_ARG),       # too small
    (dict(ws=P + (5 << 30) + 8), fa.FA_ERR_INVALID_ARG),   # misaligned
    (dict(ws=P), fa.FA_ERR_INVALID_ARG),              # overlaps q
    (dict(B=0), fa.FA_OK),
])
def test_fp8_splitkv_argument_errors_are_synchronous(lib, over, status):
    """The e4m3 split-KV entry checks its arguments like fa_fwd_splitkv and
    fa_fwd_fp8, before any CUDA call."""
    a = dict(q=P, k=P + (1 << 30), v=P + (2 << 30), o=P + (3 << 30), lse=P + (4 << 30),
             ws=P + (5 << 30), ws_bytes=1 << 29, qs=0.01, ks=0.01, vs=0.01, B=2, H=8, H_kv=2,
             Nq=4, Nk=512, d=128, scale=0.088, causal=1, splits=3)
    a.update(over)
    st = lib.fa_fwd_splitkv_fp8(a["q"], a["k"], a["v"], a["qs"], a["ks"], a["vs"], a["o"],
                                a["lse"], a["B"], a["H"], a["H_kv"], a["Nq"], a["Nk"], a["d"],
                                a["scale"], a["causal"], None, a["splits"], a["ws"],
                                a["ws_bytes"], None)
    assert st == status



def test_default_splits_rule(lib):
    """fa_splitkv_default_splits keeps units within one wave: at most 128 units
    for shapes the decoding tile takes (d = 128, query heads per K/V head x rows
    <= 8), at most the SM count otherwise (148 here: with no device the count
    falls back to 148), and each range at least four key tiles long."""
    f = lib.fa_splitkv_default_splits
    assert f(1, 32, 8, 1, 131072, 128) == 16        # 8 head groups x 16 = 128 units
    assert f(2, 32, 8, 1, 65536, 128) == 8          # 16 x 8 = 128
    assert f(4, 32, 8, 1, 32768, 128) == 4          # 32 x 4 = 128
    assert f(16, 32, 8, 1, 8192, 128) == 1          # 128 units unsplit
    assert f(1, 32, 8, 1, 131072, 64) == 18         # general kernel: 8 x 18 = 144 <= 148
    assert f(1, 32, 2, 1, 131072, 128) == 74        # 16 heads per group: general kernel, 2 x 74
    assert f(1, 32, 8, 1, 1024, 128) == 2           # 8 key tiles: ranges of >= 4 tiles
    assert f(1, 32, 7, 1, 4096, 128) == 1           # H not a multiple of H_kv: invalid, 1
