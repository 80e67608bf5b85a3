"""The seeded end-to-end cases and their stored oracle values (no GPU).

Every case of synth.cases has a row in tests/golden/e2e_oracle.txt with the case's own
shape, rank and iteration count, and each rank is the one the bits-per-weight rule gives
for its configuration's BPW (or the rank the configuration states).
"""
import pytest

from conftest import read_golden
from oracle.bpw import rank_for_bpw
from synth.cases import CASES

ROWS = {row[0]: row for row in read_golden("e2e_oracle.txt")}
BPW = {"c2_q_proj": 1.0, "c3_q_proj": 0.8, "c3_gate_proj": 0.8, "c3_down_proj": 0.8,
       "c4_k_proj": 0.55}


def test_every_case_has_an_oracle_value():
    assert set(ROWS) == set(CASES)


@pytest.mark.parametrize("name", sorted(CASES))
def test_stored_row_matches_the_case(name):
    c, row = CASES[name], ROWS[name]
    assert (int(row[1]), int(row[2]), int(row[3]), int(row[4])) == (c.m, c.n, c.r, c.iters)
    e = float(row[5])
    assert 0.0 < e < 1.0


@pytest.mark.parametrize("name", sorted(BPW))
def test_case_rank_follows_the_bpw_rule(name):
    c = CASES[name]
    assert rank_for_bpw(c.m, c.n, BPW[name]) == c.r


def test_stated_ranks():
    assert CASES["target_gate_proj"].r == 1000
    assert sorted(CASES[n].r for n in CASES if n.startswith("c5_")) == [16, 256, 1024, 4080]
