"""The SkipGS backward gate against the worked example its paper notes print
(tests/golden/skipgs_worked_example.json) and the rules of "key design" 1-3."""
import json
import math
import os

from gaussian_splatting_differentiable_dgs_b200.skipgs import BackwardGate

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "skipgs_worked_example.json")))


def test_constants_are_the_notes():
    c = GOLD["constants"]
    g = BackwardGate()
    assert (g.warmup, g.beta, g.rho_lo, g.eps) == (c["warmup_W"], c["beta"], c["rho_lo"], c["eps"])


def test_calibration_of_the_budget_floor():
    # a warm-up whose scored steps rise above their baseline 30 % of the time
    g = BackwardGate(warmup=11)
    losses = [1.0] + [0.9, 0.8, 2.0, 0.7, 0.6, 3.0, 0.5, 0.4, 4.0, 0.3]
    for x in losses:
        assert g.decide("v", x) is True          # warm-up: always backward
    assert g.warm_scored == 10
    assert g.warm_rise / g.warm_scored == GOLD["calibration"]["rho_hat_W"]
    g.decide("v", 0.0)                          # first gated step calibrates
    assert abs(g.rho_min - GOLD["calibration"]["rho_min"]) <= 1e-12


def _gated(rho_min, t_minus_1, b):
    g = BackwardGate(warmup=0)
    g.rho_min = rho_min
    g.t, g.b = t_minus_1, b
    return g


def test_skip_allowed_by_the_budget():
    e = GOLD["skip_allowed"]
    g = _gated(GOLD["calibration"]["rho_min"], 2500, 1700)
    assert abs(g.rho_cum() - e["rho_cum"]) <= 1e-12
    g.ema["A"] = e["ema_A"]
    assert g.decide("A", e["loss_A"]) is False
    s, proposed, forced, backward = g.last
    assert round(s, 3) == e["s_printed"] and not proposed and not forced and not backward
    # the baseline still follows the forward loss
    assert abs(g.ema["A"] - (0.95 * e["ema_A"] + 0.05 * e["loss_A"])) <= 1e-15
    assert g.b == 1700


def test_budget_overrides_a_skip():
    e = GOLD["budget_override"]
    g = _gated(GOLD["calibration"]["rho_min"], 1000, 648)
    assert abs(g.rho_cum() - e["rho_cum"]) <= 1e-12
    g.ema["B"] = 1.0
    assert g.decide("B", e["s"]) is True
    s, proposed, forced, backward = g.last
    assert abs(s - e["s"]) <= 1e-7 and not proposed and forced and backward
    assert g.b == 649


def test_rise_and_first_visit_run_the_backward():
    g = _gated(0.5, 100, 100)
    assert g.decide("new", 0.3) is True and g.last[0] == math.inf
    g.ema["x"] = 0.1
    assert g.decide("x", 0.2) is True and g.last[1] and not g.last[2]
