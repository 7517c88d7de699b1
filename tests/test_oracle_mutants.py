"""Pin sensitivity: every planted mistake in the oracle fails at least one pin.

The oracle's C file lists its planted mistakes (an off-by-one exponent, ties the
wrong way, a transposed rotation, Lambda multiplying instead of dividing, a
swapped nibble order, ...).  A normal build contains none of them.  Here the
oracle is rebuilt once per mistake (``-DMXQ_MUTANT=k``) and the CPU pins run
against that build: if none of them failed, the pins could not tell that
oracle from the right one.  The pins stop at the first failure, cheapest
first, so the whole sweep takes well under a minute.
"""
import inspect

import pytest

import oracle
from tests import test_oracle_block_pins as block_pins
from tests import test_oracle_gemm_pins as gemm_pins
from tests import test_oracle_nvfp4_pins as nvfp4_pins
from tests import test_oracle_pins as pins
from tests import test_oracle_search_pins as search_pins

N_MUTANTS = 22


def _calls():
    """Every pin of the oracle as a no-argument callable (parametrised pins take their
    first parameter set), in module order."""
    out = []
    for mod in (pins, block_pins, gemm_pins, nvfp4_pins, search_pins):
        for name, f in inspect.getmembers(mod, inspect.isfunction):
            if not name.startswith("test_") or f.__module__ != mod.__name__:
                continue
            marks = [m for m in getattr(f, "pytestmark", []) if m.name == "parametrize"]
            kwargs = {}
            for m in marks:
                names = [n.strip() for n in m.args[0].split(",")]
                first = m.args[1][0]
                vals = first if len(names) > 1 else (first,)
                kwargs.update(zip(names, vals))
            out.append((f"{mod.__name__.split('.')[-1]}::{name}", f, kwargs))
    return out


PINS = _calls()


def test_normal_build_passes_every_pin():
    for name, f, kwargs in PINS:
        f(**kwargs)


@pytest.mark.parametrize("mutant", range(1, N_MUTANTS + 1))
def test_planted_mistake_fails_a_pin(mutant):
    path = oracle.build_variant(mutant)
    caught = None
    with oracle.use_library(path):
        for name, f, kwargs in PINS:
            try:
                f(**kwargs)
            except Exception:   # an assertion, or an oracle error the pin provoked
                caught = name
                break
    assert caught is not None, f"no pin fails with planted mistake {mutant}"
