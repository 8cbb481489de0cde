"""Host-side balance telemetry (no GPU): MaxVio bands and per-step statistics.

The bands follow "Arcee Halts 400B Blackwell Model Collapse With Dynamic
Router Biases", "The MaxVio Metric and the Day-4 Crisis": at most 3 between
the most- and least-routed expert is healthy, about 6 passable late in
training, above that an alarm; an expert with no load makes the ratio +inf.
"""
import math

import torch

from expert_bias_load_b200 import telemetry


def test_maxvio_bands():
    assert telemetry.maxvio_level(1.0) == "healthy"
    assert telemetry.maxvio_level(3.0) == "healthy"
    assert telemetry.maxvio_level(3.01) == "passable"
    assert telemetry.maxvio_level(6.0) == "passable"
    assert telemetry.maxvio_level(6.5) == "alarm"
    assert telemetry.maxvio_level(math.inf) == "alarm"
    assert telemetry.maxvio_level(math.nan) == "alarm"


def test_step_stats_from_loads():
    counts = torch.tensor([200, 50, 100, 50], dtype=torch.int32)
    bias = torch.tensor([-0.002, 0.001, 0.0, 0.001])
    prev = torch.tensor([-0.001, 0.0005, 0.0, 0.0005])
    mom = torch.tensor([-0.001, 0.0005, 0.0, 0.0005])
    st = telemetry.step_stats(counts, bias, momentum=mom, prev_bias=prev)
    assert st["maxvio"] == 4.0 and st["level"] == "passable"                  # 200 / 50, no device scalar given
    assert (st["max_load"], st["min_load"], st["total_load"]) == (200, 50, 400)
    assert abs(st["bias_sum"]) < 1e-9
    assert abs(st["bias_absmax"] - 0.002) < 1e-9 and abs(st["momentum_absmax"] - 0.001) < 1e-9
    assert abs(st["bias_step_absmax"] - 0.001) < 1e-9
    # a dead expert: +inf, an alarm
    st = telemetry.step_stats(torch.tensor([5, 0, 5, 6], dtype=torch.int32), bias)
    assert st["maxvio"] == math.inf and st["level"] == "alarm"
    # the update's own MaxVio scalar takes precedence when given
    st = telemetry.step_stats(counts, bias, maxvio=torch.tensor([2.5]))
    assert st["maxvio"] == 2.5 and st["level"] == "healthy"
