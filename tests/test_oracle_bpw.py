"""Pins for the oracle's bits-per-weight accounting (CPU only)."""
from fractions import Fraction

import pytest

from conftest import read_golden
from oracle.bpw import bpw, linear_bits, rank_for_bpw

# Public Llama-2 architecture constants (model cards): hidden 4096 / 8192, MLP 11008 / 28672,
# 32 / 80 blocks, GQA key/value width 1024 for 70B, vocabulary 32000, untied embedding and head.
LLAMA2_7B = dict(blocks=32, layers=[(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)],
                 hidden=4096)
LLAMA2_70B = dict(blocks=80, layers=[(8192, 8192), (1024, 8192), (1024, 8192), (8192, 8192),
                                     (28672, 8192), (28672, 8192), (8192, 28672)], hidden=8192)
VOCAB = 32000


def _size_gb(arch, bits_per_weight):
    emb_bytes = 2 * VOCAB * arch["hidden"] * 2           # embedding + LM head kept at 16 bit
    if bits_per_weight == 16:
        lin = arch["blocks"] * sum(m * n for m, n in arch["layers"]) * 2
        norms = (arch["blocks"] * 2 * arch["hidden"] + arch["hidden"]) * 2
        return (lin + emb_bytes + norms) / 1e9
    bits = arch["blocks"] * linear_bits(arch["layers"], bits_per_weight)
    return (bits / 8 + emb_bytes) / 1e9


@pytest.mark.parametrize("row", read_golden("model_sizes.txt"), ids=lambda r: f"{r[0]}@{r[1]}")
def test_model_sizes_match_pages(row):
    model, b, size = row[0], float(row[1]), float(row[2])
    arch = LLAMA2_7B if model == "llama2-7b" else LLAMA2_70B
    got = _size_gb(arch, b)
    assert abs(got - size) < 0.005 + 1e-9, (model, b, got, size)


def test_bpw_closed_form_exact_values():
    # 8192^2 at r = 4080: ((16384*4080) + 16*16384) / 8192^2 = 16384*4096/8192^2 = 1 exactly.
    assert bpw(8192, 8192, 4080) == 1
    assert bpw(256, 512, 16) == Fraction(768 * 16 + 16 * 768, 256 * 512)
    assert bpw(4, 4, 0) == Fraction(16 * 8, 16)


@pytest.mark.parametrize("m,n,target", [(4096, 4096, 1.0), (4096, 4096, 0.8), (11008, 4096, 0.8),
                                        (4096, 11008, 0.8), (8192, 8192, 0.55), (1024, 8192, 0.55),
                                        (28672, 8192, 0.55), (8192, 28672, 0.55), (256, 512, 0.1875),
                                        (8192, 8192, 1.0), (17, 33, 3.0)])
def test_rank_for_bpw_is_the_floor(m, n, target):
    r = rank_for_bpw(m, n, target)
    t = Fraction(repr(target))
    assert bpw(m, n, r) <= t or r == 0
    assert bpw(m, n, r + 1) > t


def test_rank_for_bpw_clamps_at_zero():
    # the 16-bit scales alone cost 16(m+n)/(mn) = 8 BPW on a 4x4 layer
    assert rank_for_bpw(4, 4, 1.0) == 0
