"""The CPU reading of the routing-record invariants (tests/routing_checks.py)
that the device checker's verdicts are compared with, pinned without a GPU:
records the oracle builds pass; every single host-side corruption breaks
exactly the invariants it is built to break; and a second, independently
written statement of the dispatch invariants (helpers.check_dispatch_properties)
agrees on which records are valid."""
import pytest
import torch

import routing_checks as RC
from helpers import check_dispatch_properties

SHAPES = [(1, 16, 1, 0), (37, 16, 4, 0), (300, 64, 8, 0), (200, 64, 8, 8), (64, 1024, 16, 0), (33, 32, 2, 2)]


@pytest.mark.parametrize("T,E,k,hot", SHAPES)
def test_oracle_records_are_valid(T, E, k, hot):
    rec = RC.oracle_record(T, E, k, seed=7 + T, hot=hot)
    assert RC.record_faults(rec, T, E, k) == 0
    check_dispatch_properties(rec, T, E, k)
    if hot:
        # every token on experts 0..hot-1: one long segment each, the rest empty
        assert torch.all(rec["counts"][:hot] == T) and int(rec["counts"][hot:].sum()) == 0


@pytest.mark.parametrize("kind", RC.KINDS)
@pytest.mark.parametrize("T,E,k,hot", [(37, 16, 4, 0), (300, 64, 8, 0), (200, 64, 8, 8)])
def test_each_corruption_breaks_exactly_its_invariants(kind, T, E, k, hot):
    rec = RC.oracle_record(T, E, k, seed=11 + T, hot=hot)
    bad, want = RC.corrupt(rec, kind, T, E, k)
    assert RC.record_faults(bad, T, E, k) == want, kind
    # the untouched record is still valid (corrupt() works on a copy)
    assert RC.record_faults(rec, T, E, k) == 0
    if not kind.startswith("weight"):
        with pytest.raises(AssertionError):
            check_dispatch_properties(bad, T, E, k)


def test_weight_check_skipped_without_weights():
    T, E, k = 37, 16, 4
    bad, _ = RC.corrupt(RC.oracle_record(T, E, k, seed=3), "weight_nan", T, E, k)
    del bad["topk_w"]
    assert RC.record_faults(bad, T, E, k) == 0
