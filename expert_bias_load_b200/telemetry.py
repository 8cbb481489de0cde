"""Per-step balance telemetry of the router.

MaxVio is read from the device scalar smebu_step / sign_update_step write.  The
thresholds follow "Arcee Halts 400B Blackwell Model Collapse With Dynamic
Router Biases", "The MaxVio Metric and the Day-4 Crisis": a ratio of at most 3
between the most- and least-routed expert is healthy, about 6 is passable late
in training, and above 6 signals routing pathology (or, during fine-tuning,
data the model has not seen: readings of 12, 15, 17).

Only small host-side reductions happen here (one device-to-host copy per
call); nothing of the router step itself.
"""
from __future__ import annotations

import math

import torch

MAXVIO_HEALTHY = 3.0
MAXVIO_ALARM = 6.0


def maxvio_level(maxvio: float) -> str:
    """'healthy' (<= 3), 'passable' (<= 6) or 'alarm' (> 6, dead experts included)."""
    if math.isnan(maxvio) or maxvio > MAXVIO_ALARM:
        return "alarm"
    return "healthy" if maxvio <= MAXVIO_HEALTHY else "passable"


def step_stats(counts: torch.Tensor, bias: torch.Tensor, momentum: torch.Tensor = None,
               maxvio: torch.Tensor = None, prev_bias: torch.Tensor = None) -> dict:
    """Balance statistics of one step as plain floats (one synchronising copy).

    counts: int32 [N_r] loads of the step (read before a reset); bias, momentum:
    fp32 [N_r] after the update; maxvio: fp32 [1] from the update; prev_bias:
    bias before the update (for the step norm)."""
    vals = [counts.max().to(torch.float64), counts.min().to(torch.float64), counts.sum().to(torch.float64),
            bias.to(torch.float64).sum(), bias.abs().max().to(torch.float64)]
    vals.append(momentum.abs().max().to(torch.float64) if momentum is not None else torch.zeros((), dtype=torch.float64, device=bias.device))
    vals.append((bias - prev_bias).abs().max().to(torch.float64) if prev_bias is not None else torch.zeros((), dtype=torch.float64, device=bias.device))
    vals.append(maxvio.to(torch.float64).reshape(()) if maxvio is not None else torch.full((), float("nan"), dtype=torch.float64, device=bias.device))
    v = torch.stack([x.reshape(()) for x in vals]).cpu().tolist()
    mx, mn, total, bsum, bmax, mmax, step, mv = v
    if math.isnan(mv):
        mv = math.inf if mn == 0 else mx / mn
    return {"maxvio": mv, "level": maxvio_level(mv), "max_load": int(mx), "min_load": int(mn),
            "total_load": int(total), "bias_sum": bsum, "bias_absmax": bmax, "momentum_absmax": mmax,
            "bias_step_absmax": step}
