"""How many requests fit in a fixed KV budget: reserve-the-maximum vs paging.

Host-side arithmetic behind the measurement in "What vLLM Is and Why It
Exists" (section "Code"): a fixed budget of KV token slots, a stream of
requests of known length, and two policies.

* Reserve-the-maximum gives every request ``max_tokens`` slots, so
  ``capacity // max_tokens`` requests fit whatever their real length.
* Paging gives a request only ``ceil(n / block_size)`` blocks; requests are
  admitted in arrival order until the next one's blocks no longer fit.

The waste of paging is the rounding of each request up to whole blocks,
``(slots held - tokens stored) / slots held``, at most ``block_size - 1``
slots per request.
"""
from __future__ import annotations

import dataclasses
from typing import Sequence

import numpy as np


@dataclasses.dataclass
class CapacityResult:
    reserved_fit: int        # requests that fit when each reserves max_tokens
    paged_fit: int           # requests admitted under paging
    slots_held: int          # block-rounded slots held by the admitted requests
    tokens_stored: int       # their actual tokens

    @property
    def improvement(self) -> float:
        return self.paged_fit / self.reserved_fit

    @property
    def waste_fraction(self) -> float:
        return (self.slots_held - self.tokens_stored) / self.slots_held if self.slots_held else 0.0


def compare_policies(lengths: Sequence[int], capacity: int, block_size: int,
                     max_tokens: int) -> CapacityResult:
    lens = np.minimum(np.asarray(lengths, dtype=np.int64), max_tokens)
    held = -(-lens // block_size) * block_size          # slots per request, rounded up
    cum = np.cumsum(held)
    fit = int(np.searchsorted(cum, capacity, side="right"))   # first prefix that overflows
    return CapacityResult(reserved_fit=capacity // max_tokens, paged_fit=fit,
                          slots_held=int(cum[fit - 1]) if fit else 0,
                          tokens_stored=int(lens[:fit].sum()))


def skewed_lengths(rng: np.random.Generator, count: int = 4000, base: int = 100,
                   mean: float = 400.0, cap: int = 4096) -> np.ndarray:
    """Mostly short, a few long: ``min(cap, base + floor(Exp(mean)))``."""
    return np.minimum(cap, base + np.floor(rng.exponential(mean, size=count)).astype(np.int64))
