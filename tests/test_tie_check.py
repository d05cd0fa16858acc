"""The near-tie rule of the parity tests, on the CPU.

Routing decisions closer than 1e-5 may go either way (a reading of the router
bullet of "Show HN: 遅いコンピュータで GLM 5.2 を実行する", section
実装済みの主な機能, which names a group-limited noaux_tc top-k but fixes no
tie rule).  valid_tie_choice must accept exactly the selections that some
resolution of the near ties produces, and reject a wrong expert, a wrong
group, duplicates or a short list.  The accepted alternatives are derived
here by brute force over every perturbation of the tied values.
"""
import itertools

import numpy as np

from tests.parity_util import MARGIN, valid_tie_choice


def _exact_select(c, G, gk, k):
    """Group-limited top-k with ties to the lower index (brute force)."""
    E = c.shape[0]
    per = E // G
    gs = [max(c[g * per + a] + c[g * per + b] for a, b in itertools.combinations(range(per), 2))
          for g in range(G)]
    groups = max(itertools.combinations(range(G), gk),
                 key=lambda gg: (sum(gs[g] for g in gg), [-g for g in gg]))
    cand = [e for g in groups for e in range(g * per, (g + 1) * per)]
    return set(max(itertools.combinations(cand, k),
                   key=lambda es: (sum(c[e] for e in es), [-e for e in es])))


def test_decidable_choice_is_the_only_valid_one():
    rng = np.random.default_rng(1)
    E, G, gk, k = 16, 4, 2, 3
    for _ in range(50):
        c = rng.uniform(0.0, 1.0, E)
        sel = _exact_select(c, G, gk, k)
        assert valid_tie_choice(sorted(sel), c, G, gk, k)
        per = E // G
        kept = {e // per for e in sel}
        # swapping any selected expert for any other expert is invalid when
        # every gap is far above the margin
        gaps = np.diff(np.sort(c))
        if gaps.min() < 10 * MARGIN:
            continue
        for out in sel:
            for inn in range(E):
                if inn in sel:
                    continue
                alt = sorted((sel - {out}) | {inn})
                assert not valid_tie_choice(alt, c, G, gk, k), (sel, out, inn, kept)


def test_expert_ties_admit_either_expert():
    E, G, gk, k = 8, 1, 1, 2
    c = np.array([0.9, 0.5, 0.7, 0.7 - MARGIN / 2, 0.1, 0.2, 0.3, 0.0])
    assert valid_tie_choice([0, 2], c, G, gk, k)
    assert valid_tie_choice([0, 3], c, G, gk, k)
    assert not valid_tie_choice([0, 1], c, G, gk, k)       # 0.5 is clearly below 0.7
    assert not valid_tie_choice([2, 3], c, G, gk, k)       # drops the clear winner 0
    assert not valid_tie_choice([0, 0], c, G, gk, k)       # duplicate
    assert not valid_tie_choice([0], c, G, gk, k)          # short
    assert not valid_tie_choice([0, 8], c, G, gk, k)       # out of range


def test_group_ties_admit_either_group():
    # groups {0,1}, {2,3}, {4,5}, {6,7}; groups 1 and 2 tie for the second
    # place (scores 1.1 and 1.1 + margin/4), and the third pick comes from it
    E, G, gk, k = 8, 4, 2, 3
    c = np.array([0.9, 0.8, 0.6, 0.5, 0.6 + MARGIN / 4, 0.5, 0.1, 0.0])
    assert valid_tie_choice([0, 1, 4], c, G, gk, k)        # group 2 kept (exact answer)
    assert valid_tie_choice([0, 1, 2], c, G, gk, k)        # group 1 kept
    assert not valid_tie_choice([0, 1, 6], c, G, gk, k)    # group 3 is clearly out
    assert not valid_tie_choice([0, 1, 3], c, G, gk, k)    # 0.5 is clearly below 0.6
    assert not valid_tie_choice([0, 2, 4], c, G, gk, k)    # two groups beside group 0,
    assert not valid_tie_choice([1, 2, 4], c, G, gk, k)    # or without expert 0


def test_brute_force_over_tie_resolutions():
    """On small random routers with values snapped to a coarse grid (many
    exact ties), every selection produced by resolving the ties differently
    (tiny perturbations, below the margin) is accepted, and every k-subset
    that no resolution produces is rejected."""
    rng = np.random.default_rng(2)
    E, G, gk, k = 8, 4, 2, 2
    for _ in range(25):
        c = np.round(rng.uniform(0, 1, E) * 4) / 4.0
        produced = set()
        for _ in range(200):
            eps = rng.uniform(-MARGIN / 10, MARGIN / 10, E)
            produced.add(tuple(sorted(_exact_select(c + eps, G, gk, k))))
        for sel in itertools.combinations(range(E), k):
            ok = valid_tie_choice(list(sel), c, G, gk, k)
            if sel in produced:
                assert ok, (c, sel)
            elif ok:
                # accepted but not seen: must be producible by some resolution
                # of the ties -- check exhaustively over sign patterns
                ties = [e for e in range(E) if np.sum(np.abs(c - c[e]) <= MARGIN) > 1]
                found = False
                for signs in itertools.product((-1, 1), repeat=len(ties)):
                    cc = c.copy()
                    for e, sg in zip(ties, signs):
                        cc[e] += sg * MARGIN / 10 * (1 + e / 100)
                    if tuple(sorted(_exact_select(cc, G, gk, k))) == sel:
                        found = True
                        break
                assert found, (c, sel)
