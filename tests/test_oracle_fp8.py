"""CPU-only pins of the oracle's e4m3 decoder (oracle/fp8.py).

The decoder is checked against torch's float8_e4m3fn conversion for all 256
codes (a library routine) and against hand-derived codes of the format
(sign, exponent bias 7, 3 mantissa bits, subnormals, one NaN pattern); planted
mistakes in a copy of it must fail those pins. The attention it feeds is the
fp64 oracle, pinned separately.
"""
import math
import os
import types

import numpy as np
import pytest
import torch

from oracle import fp8

HAND = {0x00: 0.0, 0x80: -0.0, 0x38: 1.0, 0xB8: -1.0, 0x7E: 448.0, 0xFE: -448.0,
        0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x40: 2.0, 0x3C: 1.5,
        0x30: 0.5, 0x77: 240.0, 0x78: 256.0}


def decoder_failures(decode):
    out = []
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = decode(codes)
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    if not np.array_equal(nan_ref, nan_got):
        out.append("NaN pattern differs from torch")
    elif not np.array_equal(ref[~nan_ref], got[~nan_got]):
        out.append("values differ from torch float8_e4m3fn")
    for c, v in HAND.items():
        g = float(decode(np.array([c], dtype=np.uint8))[0])
        if not (g == v and math.copysign(1, g) == math.copysign(1, v)):
            out.append(f"code {c:#04x}: {g} != {v}")
    return out


def test_decoder_passes_pins():
    assert decoder_failures(fp8.decode_e4m3) == []


MUTANTS = {
    "bias_8": ("(e - 7)", "(e - 8)"),
    "mantissa_over_16": ("1.0 + m / 8.0", "1.0 + m / 16.0"),
    "subnormal_exponent": ("np.ldexp(m / 8.0, -6)", "np.ldexp(m / 8.0, -7)"),
    "no_nan": ("np.where((e == 15) & ((c & 7) == 7), np.nan, val)", "val"),
    "sign_ignored": ("np.where((c >> 7) & 1, -1.0, 1.0)", "1.0"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_decoder_mutant_is_caught(name):
    src = open(fp8.__file__).read()
    before, after = MUTANTS[name]
    assert src.count(before) == 1, before
    mod = types.ModuleType(f"fp8_{name}")
    mod.__dict__["__file__"] = os.path.join(os.path.dirname(fp8.__file__), f"fp8_{name}.py")
    exec(compile(src.replace(before, after), mod.__file__, "exec"), mod.__dict__)
    assert decoder_failures(mod.decode_e4m3), f"mutant {name} passed every pin"


def test_fp8_attention_is_the_dequantized_attention():
    """With descales that are powers of two the dequantized values are bf16
    values too, so the fp8 route must equal the bf16 oracle route exactly."""
    import oracle
    g = torch.Generator().manual_seed(3)
    x = [torch.randn(1, 2, 40, 16, generator=g).to(torch.float8_e4m3fn) for _ in range(3)]
    o8, l8 = fp8.attention_fp8(*x, 0.5, 2.0, 0.25, 0.3, causal=True)
    bf = [(t.to(torch.float32) * s).to(torch.bfloat16) for t, s in zip(x, (0.5, 2.0, 0.25))]
    ob, lb = oracle.attention(*bf, 0.3, causal=True)
    assert np.array_equal(o8, ob) and np.array_equal(l8, lb)
