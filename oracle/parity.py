"""Comparison of a routing result with the oracle's -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module (as the rest of ``oracle``). It holds no arithmetic of the method: it
calls ``zha_oracle.route`` and compares kept sets.

Each level of one query head is compared with the oracle's own top-p selection
at that level, the oracle being steered by the compared result's kept set one
level up (``route(..., forced_kept=...)``), so that one tie cannot cascade. A
node on which the two kept sets disagree is a *tie* when its oracle score lies
within ``TIE_TOL`` of the score at the oracle's cut, or when the cumulative mass
at the cut lies within ``TIE_TOL`` of p; every other disagreement is *hard*.
Ties are counted and reported, hard disagreements fail. [ZHA: 전제와 한계] fixes
the rule being compared: softmax over the candidates, sorted by score, the
minimal prefix holding mass p.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import zha_oracle as O

TIE_TOL = 1e-5


@dataclass
class RouteReport:
    heads: int = 0
    levels_compared: int = 0
    ties: int = 0
    hard: list = field(default_factory=list)
    exact_heads: set = field(default_factory=set)

    def summary(self) -> dict:
        return {"heads": self.heads, "levels_compared": self.levels_compared, "ties": self.ties,
                "hard": len(self.hard), "exact_heads": len(self.exact_heads)}


def _level_mass(p, level):
    """The top-p mass of `level` under a number, a {level: p} dict or a
    RoutePolicy; None for a fixed-budget (top-K) level."""
    if isinstance(p, O.RoutePolicy):
        return p.at(level) if p.mode == "top_p" else None
    if isinstance(p, dict):
        return p[level]
    return p


def compare_route_head(q, otree, p, kept_by_level: dict, report: RouteReport, key,
                       route_fn=None) -> None:
    """Compare one query head's kept sets {level: node ids} with the oracle,
    level by level (each level conditioned on the compared kept set one level
    up). ``p`` is what ``zha_oracle.route`` takes: a mass, a {level: p} dict or a
    RoutePolicy (for top-K levels only score ties count). ``route_fn`` replaces
    ``zha_oracle.route`` (same signature) for routing variants."""
    route = route_fn if route_fn is not None else O.route
    forced = {lvl: ids for lvl, ids in kept_by_level.items()}
    tr = route(q, otree, p, forced_kept=forced)
    exact = True
    for lvl, lt in tr.levels.items():
        report.levels_compared += 1
        own = set(lt.topp.kept.tolist())
        got = set(np.asarray(kept_by_level[lvl]).tolist())
        if own == got:
            continue
        exact = False
        cand_pos = {int(n): i for i, n in enumerate(lt.candidates)}
        sel = lt.topp
        m = sel.m
        sigma_cut = lt.sigma[sel.order[m - 1]] if m > 0 else math.inf
        p_lvl = _level_mass(p, lvl)
        near_mass = p_lvl is not None and (
            (m >= 1 and abs(sel.cum[m - 1] - p_lvl) <= TIE_TOL) or
            (m >= 2 and abs(sel.cum[m - 2] - p_lvl) <= TIE_TOL))
        for node in own ^ got:
            if node not in cand_pos:
                report.hard.append((key, lvl, node, "not a candidate"))
                continue
            if abs(lt.sigma[cand_pos[node]] - sigma_cut) <= TIE_TOL or near_mass:
                report.ties += 1
            else:
                report.hard.append((key, lvl, node, float(lt.sigma[cand_pos[node]]), float(sigma_cut)))
    report.heads += 1
    if exact:
        report.exact_heads.add(key)
