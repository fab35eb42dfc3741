"""Host logic of the chained layer driver (CPU): the tau calibration that the
benchmark and the chained parity tests use.  A stand-in pipe maps tau to a
kept-block fraction with the same monotone staircase shape the real mask has
(more budget never keeps fewer blocks), so the bisection can be checked
without a GPU."""
import math

from entropy_adaptive_radius_b200.pipeline import calibrate_tau


class StairPipe:
    """kept(tau) = floor + (1 - floor) * (1 - exp(-tau / scale)), quantized to
    `levels` steps (a block mask's fraction moves in steps of 1 / blocks)."""

    def __init__(self, floor=0.0665, scale=0.01, levels=591 * 591):
        self.floor, self.scale, self.levels = floor, scale, levels
        self.calls = []
        self.f = None

    def mask(self, tau):
        self.calls.append(tau)
        raw = self.floor + (1.0 - self.floor) * (1.0 - math.exp(-tau / self.scale))
        self.f = math.floor(raw * self.levels) / self.levels

    def kept_fraction(self):
        return self.f


def kept_at(pipe, tau):
    pipe.mask(tau)
    return pipe.kept_fraction()


def test_calibration_reaches_reachable_targets():
    for target in (0.09, 0.12, 0.19, 0.40, 0.90):
        pipe = StairPipe()
        tau = calibrate_tau(pipe, target)
        assert abs(kept_at(pipe, tau) - target) < 0.002, target
        assert len(pipe.calls) <= 31


def test_calibration_below_the_floor_returns_the_nearest_fraction():
    """Targets under the r = 0 floor (the density sweep's 5% point at the
    21x45x80 grid) end at the smallest tau tried, whose fraction is the floor."""
    pipe = StairPipe(floor=0.0665)
    tau = calibrate_tau(pipe, 0.05)
    assert abs(kept_at(pipe, tau) - 0.0665) < 1e-3
    assert tau < 1e-4


def test_calibration_reports_through_the_log():
    lines = []
    pipe = StairPipe()
    calibrate_tau(pipe, 0.12, lines.append)
    assert len(lines) == 1 and "tau calibrated" in lines[0]
