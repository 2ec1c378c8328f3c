"""Adapters that feed generated workload inputs (exactly widened to float64) to the oracle."""
from __future__ import annotations

import numpy as np

import synth


class Source:
    """q/k/v of a workload as float64 token ranges: src.q(t0, n) -> [n, H, d]."""

    def __init__(self, w: synth.Workload):
        self.w = w

    def q(self, t0: int, n: int) -> np.ndarray:
        return synth.to_f64(synth.gen_chunk(self.w, t0, n, "q")[0])

    def k(self, t0: int, n: int) -> np.ndarray:
        return synth.to_f64(synth.gen_chunk(self.w, t0, n, "k")[1])

    def v(self, t0: int, n: int) -> np.ndarray:
        return synth.to_f64(synth.gen_chunk(self.w, t0, n, "v")[2])


def oracle_cfg(w: synth.Workload) -> dict:
    return w.as_config()
