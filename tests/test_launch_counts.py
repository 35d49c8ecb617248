"""The host-side mirrors of how sf_masked_dw splits a call into launches (CPU). They feed the
launch count that bench.py reports, so they follow the library's packing rules: groups of
consecutive problems reading the same input (at most 8), main launches packed by kernel-parameter
bytes and at most 96 problems, and one row-gather launch per 192 groups / 384 problems."""
from masked_optimizer_step_b200.model import (INPUT_OF, LLAMA_7B_LAYER, dw_gather_launch_count,
                                              dw_launch_count)


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
