"""Host-side logic of the refinement step that needs no GPU: the stream schedules RefinementStep
accepts, and the benchmark's description of each of them."""
import pytest

import bench
from denoiser_attention_b200 import api


def test_schedules_are_the_documented_ones():
    assert api.RefinementStep.SCHEDULES == ("branches", "attn_then_unmask", "unmask_then_attn", "serial")
    assert set(bench.SCHEDULE_TEXT) == set(api.RefinementStep.SCHEDULES)


def test_schedule_selection():
    assert api.RefinementStep({}, gamma=0.8).schedule == "branches"
    assert api.RefinementStep({}, gamma=0.8, schedule="unmask_then_attn").schedule == "unmask_then_attn"
    # concurrent=False keeps its meaning: everything on the caller's stream
    assert api.RefinementStep({}, gamma=0.8, concurrent=False, schedule="branches").schedule == "serial"


def test_unknown_schedule_is_rejected():
    with pytest.raises(ValueError):
        api.RefinementStep({}, gamma=0.8, schedule="interleaved")
