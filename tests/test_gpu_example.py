"""The usage example the README shows (masked_optimizer_step_b200/example.py) runs (GPU)."""
import pytest

pytestmark = pytest.mark.gpu


def test_usage_example_runs(sf):
    from masked_optimizer_step_b200 import example
    assert example.main() == 41      # exactly the rows given the signal turn active
