"""Backward gate of SkipGS (SkipGS paper notes, "key design" 1-3): after
densification, every step renders its view and scores the loss against that
view's own running baseline; the backward and the Adam update run only when
the loss rose above it, unless the cumulative share of backward steps would
fall below a floor calibrated during a warm-up.

- Score (key design 1): s = L(t) / (EMA_v(t-1) + eps), eps = 1e-8; a view
  seen for the first time scores +inf, so it always runs the backward.
- Proposal (key design 2): backward iff s > 1.  The view's baseline is
  updated after scoring, whatever the decision:
  EMA_v(t) = beta EMA_v(t-1) + (1 - beta) L(t), beta = 0.95 (the first
  sample starts the baseline at L).
- Budget (key design 3): the first W = 500 steps always run the backward
  and record the share of proposals s > 1 among the steps whose view had a
  baseline; at step W + 1 the floor becomes
  rho_min = rho_lo + (1 - rho_lo) share, rho_lo = 0.5.  After that a
  proposed skip is overridden when rho_cum = b / max(t - 1, 1) < rho_min,
  b the number of backward steps so far.

The gate is host-side bookkeeping: `Stepper.run_view(..., gate=g.decide_for(v))`
asks it once per step with the view's forward loss.
"""
from __future__ import annotations

import math


class BackwardGate:
    def __init__(self, warmup: int = 500, beta: float = 0.95, rho_lo: float = 0.5,
                 eps: float = 1e-8):
        self.warmup = int(warmup)
        self.beta = float(beta)
        self.rho_lo = float(rho_lo)
        self.eps = float(eps)
        self.ema = {}          # view -> loss baseline
        self.t = 0             # steps so far
        self.b = 0             # backward steps so far
        self.warm_scored = 0   # warm-up steps whose view had a baseline
        self.warm_rise = 0     # ... of which proposed a backward (s > 1)
        self.rho_min = None    # set at step warmup + 1
        self.last = None       # (s, proposed, forced, backward) of the last step

    def rho_cum(self) -> float:
        """Share of backward steps among the steps taken so far (at step t:
        b / max(t - 1, 1))."""
        return self.b / max(self.t, 1)

    def decide(self, view, loss: float) -> bool:
        """One step of `view` with forward loss `loss`; True = run the
        backward and the update."""
        rho_prev = self.rho_cum()
        self.t += 1
        base = self.ema.get(view)
        s = math.inf if base is None else loss / (base + self.eps)
        proposed = s > 1.0
        # the baseline follows every forward, whatever the decision
        self.ema[view] = loss if base is None else self.beta * base + (1.0 - self.beta) * loss
        forced = False
        if self.t <= self.warmup:
            if base is not None:
                self.warm_scored += 1
                self.warm_rise += int(proposed)
            backward = True
        else:
            if self.rho_min is None:
                share = self.warm_rise / self.warm_scored if self.warm_scored else 1.0
                self.rho_min = self.rho_lo + (1.0 - self.rho_lo) * share
            backward = proposed
            if not backward and rho_prev < self.rho_min:
                backward = forced = True
        if backward:
            self.b += 1
        self.last = (s, proposed, forced, backward)
        return backward

    def decide_for(self, view):
        """The gate for one step of `view`, as run_view's `gate` callback."""
        return lambda loss: self.decide(view, loss)
