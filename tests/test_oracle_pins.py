"""The CPU oracle against hand-worked cases, exact search, closed forms, invariants
and library routines (no GPU)."""
import pytest

import oracle
from tests import oracle_pins as P


@pytest.fixture(scope="module")
def O():
    return oracle.lib()


@pytest.mark.parametrize("check", P.QUANT_CHECKS, ids=lambda f: f.__name__)
def test_quantization_pins(O, check):
    check(O)


@pytest.mark.parametrize("check", P.ATTN_CHECKS, ids=lambda f: f.__name__)
def test_attention_pins(O, check):
    check(O)


@pytest.mark.parametrize("check", P.DRAFT_CHECKS, ids=lambda f: f.__name__)
def test_drafting_pins(O, check):
    check(O)
