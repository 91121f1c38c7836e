"""Each planted mistake in the oracle must be caught by at least one pin.

The mutants live behind ``-DORACLE_MUTANT=<n>`` in ``oracle/ssa_oracle.c``:
 1 scoring without the 1/sqrt(d) scale      2 attention without the scale
 3 ties broken towards the higher index    4 selected chunks keep their gists
 5 tail tokens dropped                      6 only the group's first head scores
 7 tail starts one token late               8 query head -> KV head map wrong
10 gist rows indexed token-major           11 selection not re-sorted by index
12 per-head union keeps head 0 only        13 selected-only context drops the gists
14 t levels: remainder units never candidates
15 adaptive top-k without the +1           16 adaptive top-k ignores J (L_eff = L)
17 prefill: earlier chunks' raw tokens seen 18 prefill: a gist hides its own chunk's gists
19 prefill: gists placed before their chunk 20 prefill attention without the scale
21 block mask: a block whose columns run past the end counted full
(mutants 15-21 live in ``oracle/prefill_oracle.c``)
"""
import pytest

from oracle import ssa_oracle
from oracle_pins import ALL_PINS

MUTANTS = [1, 2, 3, 4, 5, 6, 7, 8, 10, 11, 12, 13, 14, 15, 16, 17, 18, 19, 20, 21]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(tmp_path, mutant):
    orc = ssa_oracle.Oracle(ssa_oracle.build(mutant, out_dir=str(tmp_path)))
    assert orc.mutant == mutant
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception as e:  # a crash on bad indexing also counts as caught
            caught.append(f"{pin.__name__}:{type(e).__name__}")
    assert caught, f"mutant {mutant} passed every pin"
