"""The tensor-core GEMVs' unpack tables (host data of the CUDA path, checked on
the CPU): every AND of a table must pull exactly the codes it names out of a
128-code segment (kUnpack) or a 32-code unit (kUnit) packed by the oracle's
packer, each code once, in the low byte of its 16-bit half (where bf16 bit
patterns are linear in value)."""
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "quantized_gemm_wq_b200", "csrc", "unpack_tables.h")


def parse_tables(family="kUnpack", n=64):
    text = open(HEADER).read()
    out = {}
    for bits, body in re.findall(family + r"(\d)\[" + str(n) + r"\] = \{(.*?)\};", text, re.S):
        ops = re.findall(r"\{(\d+), 0x([0-9A-F]+)u, (\d+), (\d+), (\d+), (\d+)\}", body)
        out[int(bits)] = [(int(s), int(m, 16), int(a), int(b), int(c), int(d)) for s, m, a, b, c, d in ops]
    return out


def test_header_is_generated():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gen_unpack_tables", os.path.join(ROOT, "quantized_gemm_wq_b200", "gen_unpack_tables.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    assert open(HEADER).read() == gen.render()


@pytest.mark.parametrize("family,nc", [("kUnpack", 128), ("kUnit", 32)])
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_ops_extract_each_code_once(bits, family, nc):
    ops = parse_tables(family, nc // 2)[bits]
    assert len(ops) == nc // 2
    seen = sorted([o[2] for o in ops] + [o[4] for o in ops])
    assert seen == list(range(nc))
    rng = np.random.default_rng(bits)
    for trial in range(20):
        q = rng.integers(0, 1 << bits, size=(1, nc), dtype=np.uint8)
        if trial == 0:
            q[:] = (1 << bits) - 1                      # all bits set: masks must not leak
        words = oracle.pack(q, bits)[0]
        stream = 0
        for i, w in enumerate(words):
            stream |= int(w) << (32 * i)
        for s, m, lo, blo, hi, bhi in ops:
            assert blo + bits <= 8 and bhi + bits <= 8
            assert m == ((((1 << bits) - 1) << blo) | ((((1 << bits) - 1) << bhi) << 16))
            v = ((stream >> s) & 0xFFFFFFFF) & m
            assert v & 0xFFFF == int(q[0, lo]) << blo
            assert v >> 16 == int(q[0, hi]) << bhi


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_bf16_patterns_are_linear(bits):
    """Pattern p < 0x100 in a bf16 is p 2^-133, so code << b reads as q 2^(b-133)."""
    for p in range(256):
        f = np.array([p << 16], dtype=np.uint32).view(np.float32)[0]
        assert float(f) == p * 2.0 ** -133


def test_shift_counts():
    t = parse_tables()
    # windows needing a shift (start not on a word boundary)
    shifts = {b: len({o[0] for o in ops if o[0] % 32}) for b, ops in t.items()}
    assert shifts[2] == 8 and shifts[4] == 16 and shifts[8] == 32
    assert shifts[3] <= 28
    u = parse_tables("kUnit", 16)
    ushifts = {b: len({o[0] for o in ops if o[0] % 32}) for b, ops in u.items()}
    assert ushifts[2] == 2 and ushifts[4] == 4 and ushifts[8] == 8 and ushifts[3] <= 7


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_unit_products_share_one_scale(bits):
    """For every AND of the 32-code unit table: the bf16 pattern of code q at
    offset b times bf16(x 2^(64 - b)) is q x 2^-69 exactly, for every code and
    sampled bf16 activations (the warp-MMA GEMV sums these products in fp32)."""
    ops = parse_tables("kUnit", 16)[bits]
    rng = np.random.default_rng(100 + bits)
    xs = (rng.standard_normal(64) * np.exp2(rng.integers(-20, 20, 64))).astype(np.float32)
    xs = (xs.view(np.uint32) & 0xFFFF0000).view(np.float32)          # bf16-representable
    for s, m, lo, blo, hi, bhi in ops:
        for b in (blo, bhi):
            for q in range(1 << bits):
                a = np.array([(q << b) << 16], dtype=np.uint32).view(np.float32)[0]
                xp = (xs.astype(np.float64) * 2.0 ** (64 - b)).astype(np.float32)
                assert np.all((xp.view(np.uint32) & 0xFFFF) == 0)     # still bf16: scaling is exact
                prod = np.float64(a) * xp.astype(np.float64)
                assert np.array_equal(prod, q * xs.astype(np.float64) * 2.0 ** -69)
