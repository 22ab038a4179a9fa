"""Input side of a multi-step decode trajectory (the drifting workload).

Holds no attention arithmetic.  Between decode steps (outside any timed region) it advances
every sequence by one token: kv_len grows by one, each layer's appended k and v are generated
on the device at the new position, and every `drift_every` steps the planted salient keys move
by `drift_shift` tokens (the old positions get their generator values back).
"""
from __future__ import annotations

import numpy as np
import torch

from .case import Case
from .gpu import DeviceCase


class Trajectory:
    def __init__(self, cfg, device="cuda"):
        self.cfg = cfg
        self.case0 = Case(cfg, step=0)
        self.dc = DeviceCase(self.case0, device=device, prefill="append")
        self.base = torch.from_numpy(np.array(cfg.contexts(0), dtype=np.int32)).to(self.dc.device)
        self.step = 0

    def case_at(self, step: int) -> Case:
        """Host view of the workload at a step (context lengths and planted positions of that step)."""
        return Case(self.cfg, step=step)

    def prepare(self, step: int) -> None:
        """Set the device inputs of decode step `step` (kv_len, appended tokens, planted keys)."""
        dc = self.dc
        dc.kv_len.copy_(self.base + step)
        dc.fill_new_tokens(dc.kv_len - 1)
        if step > 0 and self.cfg.drift_every and step % self.cfg.drift_every == 0:
            dc.replant(step)
        self.step = step
