"""Mixed-precision policy: which bit width each linear of a model gets.

The method keeps most linears at 4 bits and those whose output scales the
residual stream at 8, and rates a policy by the cosine of the model's output
against the dense one and by its size against dense (stable-diffusion.rs
README, introduction). This module chooses such policies from measurements:
given, for every linear, its dense output and its output at each candidate
bit width (computed by the caller, for example with ``qgemm`` on representative
inputs), it finds the assignments that trade size against accuracy best.

The accuracy measure is the cosine of all the linears' outputs taken together
(concatenated) against the dense outputs, as the block measurement in the
bench reports it. With d_l a layer's dense output and e_l = q_l - d_l its
quantisation error, that cosine is an exact function of three sums of
per-layer terms:

    D = sum ||d_l||^2,  A = sum <e_l, d_l>,  B = sum ||e_l||^2
    cos = (D + A) / sqrt(D (D + 2A + B))

so a layer's contribution can be measured once per bit width and any
assignment scored without recomputing outputs. With 16 linears or fewer the
search enumerates every assignment, so its front is exact in the cosine
itself. Beyond that it minimises the output error energy B for each size (a
multiple-choice knapsack, exact when sizes are not bucketed; B and the cosine
move together up to the small cross term A), then scores every point with the
exact cosine. Host-side only; nothing here launches a kernel.
"""
from __future__ import annotations

import dataclasses
import itertools
import math
from typing import Dict, List, Mapping, Optional, Sequence

import numpy as np

EXHAUSTIVE_MAX_LAYERS = 16


@dataclasses.dataclass(frozen=True)
class Option:
    """One bit width for one linear: its packed bytes and its output error
    terms against the dense output (A = <e, d>, B = ||e||^2)."""
    bits: int
    nbytes: int
    cross: float
    err: float


@dataclasses.dataclass(frozen=True)
class LayerStats:
    name: str
    dense_energy: float            # ||d||^2
    options: Mapping[int, Option]  # bits -> Option


@dataclasses.dataclass(frozen=True)
class Policy:
    bits: Dict[str, int]   # layer name -> bits
    nbytes: int
    cosine: float
    err: float             # output error energy B


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):      # a torch tensor, on any device
        a = a.detach().double().cpu().numpy()
    return np.asarray(a, dtype=np.float64).ravel()


def layer_stats(name: str, dense_out, quant_outs: Mapping[int, object], nbytes: Mapping[int, int]) -> LayerStats:
    """The terms of one linear: `dense_out` is its output with dense weights,
    `quant_outs[bits]` its output with the weights at `bits`, `nbytes[bits]`
    the packed size. Outputs may be numpy arrays or torch tensors; the sums
    are taken in fp64."""
    d = _f64(dense_out)
    opts = {}
    for bits, q in quant_outs.items():
        e = _f64(q) - d
        if e.shape != d.shape:
            raise ValueError(f"{name}: output at {bits} bits has {e.size} elements, dense {d.size}")
        opts[int(bits)] = Option(int(bits), int(nbytes[bits]), float(e @ d), float(e @ e))
    if not opts:
        raise ValueError(f"{name}: no quantised outputs")
    return LayerStats(name, float(d @ d), opts)


def cosine(layers: Sequence[LayerStats], assignment: Mapping[str, int]) -> float:
    """Exact cosine of the concatenated outputs under `assignment` (layer name -> bits)."""
    D = sum(l.dense_energy for l in layers)
    A = sum(l.options[assignment[l.name]].cross for l in layers)
    B = sum(l.options[assignment[l.name]].err for l in layers)
    den = D * (D + 2 * A + B)
    if D <= 0 or den <= 0:
        raise ValueError("the dense outputs, or the quantised ones, are all zero")
    return (D + A) / math.sqrt(den)


def _policy(layers, choice) -> Policy:
    a = {l.name: b for l, b in zip(layers, choice)}
    return Policy(a, sum(l.options[b].nbytes for l, b in zip(layers, choice)), cosine(layers, a),
                  sum(l.options[b].err for l, b in zip(layers, choice)))


def _front(points: List[Policy], better) -> List[Policy]:
    """Points no other point beats: smaller or equal size and better or equal
    accuracy, strictly in one. Sorted by size."""
    pts = sorted(points, key=lambda p: (p.nbytes, -better(p)))
    out, best = [], -math.inf
    for p in pts:
        if better(p) > best:
            out.append(p)
            best = better(p)
    return out


def frontier(layers: Sequence[LayerStats], exhaustive_max: int = EXHAUSTIVE_MAX_LAYERS,
             resolution_bytes: Optional[int] = None) -> List[Policy]:
    """The size / accuracy front, smallest first.

    Up to `exhaustive_max` linears: every assignment is scored and the front
    is the exact one in (size, cosine). Beyond: the front in (size, output
    error energy) by dynamic programming over the linears, with sizes grouped
    in buckets of `resolution_bytes` (default: 1/20000 of the largest total;
    1 makes the programme exact), each bucket keeping its smallest error;
    every point of that front is then scored with its exact cosine and the
    front re-filtered on it."""
    layers = list(layers)
    if not layers:
        return []
    names = [l.name for l in layers]
    if len(set(names)) != len(names):
        raise ValueError("layer names must be unique")
    if len(layers) <= exhaustive_max:
        pts = [_policy(layers, c) for c in itertools.product(*[sorted(l.options) for l in layers])]
        return _front(pts, lambda p: p.cosine)
    if resolution_bytes is None:
        largest = sum(max(o.nbytes for o in l.options.values()) for l in layers)
        resolution_bytes = max(1, largest // 20000)
    # bucket -> (bytes, err, choice); Pareto-minimal in (bytes, err) after every layer
    states = {0: (0, 0.0, ())}
    for l in layers:
        nxt = {}
        for nb, err, ch in states.values():
            for b in sorted(l.options):
                o = l.options[b]
                cand = (nb + o.nbytes, err + o.err, ch + (b,))
                k = cand[0] // resolution_bytes
                if k not in nxt or cand[1] < nxt[k][1]:
                    nxt[k] = cand
        states, best = {}, math.inf
        for k in sorted(nxt):
            if nxt[k][1] < best:
                states[k] = nxt[k]
                best = nxt[k][1]
    return _front([_policy(layers, ch) for _, _, ch in states.values()], lambda p: p.cosine)


def cheapest(layers: Sequence[LayerStats], min_cosine: float, **search) -> Optional[Policy]:
    """The smallest policy on the front whose cosine reaches `min_cosine`
    (None if none does). `search`: frontier()'s keyword arguments."""
    for p in frontier(layers, **search):
        if p.cosine >= min_cosine:
            return p
    return None


def most_accurate(layers: Sequence[LayerStats], max_bytes: int, **search) -> Optional[Policy]:
    """The most accurate policy on the front within `max_bytes` (None if even
    the smallest is larger). `search`: frontier()'s keyword arguments."""
    best = None
    for p in frontier(layers, **search):
        if p.nbytes <= max_bytes and (best is None or p.cosine > best.cosine):
            best = p
    return best
