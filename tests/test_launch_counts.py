"""The host-side mirrors of how sf_masked_dw splits a call into launches (CPU). They feed the
launch count that bench.py reports, so they follow the library's packing rules: groups of
consecutive problems reading the same input (at most 8), main launches packed by kernel-parameter
bytes and at most 96 problems, and one row-gather launch per 192 groups / 384 problems."""
import os
import re

from masked_optimizer_step_b200 import binding as sf
from masked_optimizer_step_b200.model import (INPUT_OF, LLAMA_7B_LAYER, dw_gather_launch_count,
                                              dw_launch_count, mask_launch_count)


def _keys(layers):
    return [((l, INPUT_OF[n]), C) for l in range(layers) for n, _, C in LLAMA_7B_LAYER]


def test_7b_step_is_one_gather_and_three_main_launches():
    keys = _keys(32)
    assert dw_gather_launch_count(keys) == 1           # 128 groups, 224 problems
    assert dw_launch_count(keys) == 3                  # 32 KB of parameters per launch


def test_small_calls_take_one_launch_each():
    assert dw_gather_launch_count(_keys(1)) == 1
    assert dw_launch_count(_keys(1)) == 1
    assert dw_gather_launch_count([("x", 512)]) == 1


def test_gather_packs_by_group_and_problem_limits():
    singles = [(i, 256) for i in range(200)]           # 200 one-problem groups: 192 + 8
    assert dw_gather_launch_count(singles) == 2
    eights = [(i // 8, 256) for i in range(8 * 50)]    # 50 groups of 8: 48 fit in 384 problems
    assert dw_gather_launch_count(eights) == 2
    nines = [("same", 256)] * 9                        # a run of 9 splits into groups of 8 and 1
    assert dw_gather_launch_count(nines) == 1


def test_mask_calls_split_the_finalize_for_large_masks():
    # the conductor of a 32,000-row vocabulary: accumulate, busiest row, charges, lists
    assert mask_launch_count([32000]) == 4
    # the 224 trackers of the 7B step (4,096 and 11,008 rows): accumulate, one-launch finalize
    rows = [R for _ in range(32) for _, R, _ in LLAMA_7B_LAYER]
    assert mask_launch_count(rows) == 2
    # both in one call: the batch holds the large mask, so all of it takes the split finalize
    assert mask_launch_count([32000] + rows) == 4
    # more masks than one launch takes: each batch decides on its own
    assert mask_launch_count([4096] * 240 + [32000]) == 2 + 4
    assert mask_launch_count([sf.SF_MASK_SPLIT_ROWS - 32]) == 2
    assert mask_launch_count([sf.SF_MASK_SPLIT_ROWS]) == 4


def test_binding_constants_match_the_header():
    # every numeric #define of the C header that the binding also names carries the same value
    header = open(os.path.join(os.path.dirname(__file__), "..", "include", "sf.h")).read()
    defs = {m.group(1): int(m.group(2), 0)
            for m in re.finditer(r"#define\s+(SF_\w+)\s+(-?(?:0x[0-9a-fA-F]+|\d+))u?\b", header)}
    shared = [n for n in defs if hasattr(sf, n)]
    assert {"SF_MASK_SPLIT_ROWS", "SF_DW_MAX_PER_LAUNCH", "SF_STATUS_WAIT_TIMEOUT",
            "SF_SRC_WORDS", "SF_PHASE_SECOND"} <= set(shared)
    for n in shared:
        assert getattr(sf, n) == defs[n], n
