"""Write the SwiGLU fixtures of this folder from exact arithmetic.

    python tests/golden/make_swiglu.py      # rewrites swiglu_cases.txt, swiglu_expert.txt

Nothing here imports the oracle or the CUDA library.  Every expected value is
the exact real result of the defining formula, evaluated with Python's
decimal module at 60 significant digits (exp) or with exact fractions, then
rounded once to the nearest fp32 (ties to even) by `f32`, below.

What the formulas are (pages by title and section):
  "Show HN: 遅いコンピュータで GLM 5.2 を実行する" (ja.news.hada.io/topic?id=31297),
  section 実装済みの主な機能 -- integer-dot bullet (Q8_0-style int8
  activations, blocks of 32 with one scale each) and quantisation bullet
  (packed int4 weights with per-row scales, dequantised on use); an expert is
  gate, up and down matrices ("Comment exécuter un réseau de neurones de 744
  milliards de paramètres sur un ordinateur ordinaire", devtrends.cc, "Comment
  fonctionne le moteur"); the activation between them is SwiGLU:
      h = SiLU(g) * u,   SiLU(g) = g * sigmoid(g) = g / (1 + e^-g),
  with g the gate projection and u the up projection.

swiglu_cases.txt: one (g, u, h) per line, g and u fp32 values spanning
|g| in [0.1, 4] of both signs (where sigmoid(g) is far from 0 and 1, so that
dropping it, moving it to u, or replacing SiLU by ReLU changes h), plus a few
saturated and zero cases.  A case is kept only if its exact h lies at least
1e-9 (relative) away from every fp32 rounding boundary, so that any
evaluation accurate to fp64 rounds to the same fp32 h.

swiglu_expert.txt: one expert (hidden 32, intermediate 32, int4, power-of-two
row scales) on one token, chosen so that g and u are exact fp32 values with
|g| < 4; the expected Q8_0(h) codes and scale, the expert output e (a dense
layer's output) and the layer output y.
"""
import os
import random
from decimal import Decimal, getcontext
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
getcontext().prec = 60


# ----------------------------------------------------------------- fp32 rounding
def _rne(q):
    """Fraction -> nearest integer, ties to even."""
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl + (fl & 1)


def _exp2(e):
    return Fraction(2) ** e


def _binade(a):
    """e with 2^e <= a < 2^(e+1), a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while _exp2(e) > a:
        e -= 1
    while _exp2(e + 1) <= a:
        e += 1
    return e


def f32(q):
    """Exact rational -> the nearest fp32 value (ties to even), as a Fraction."""
    q = Fraction(q)
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    ulp = _exp2(max(_binade(a), -126) - 23)
    n = _rne(a / ulp)
    r = n * ulp
    assert r < _exp2(128), "overflow"
    return sign * r


def boundary_distance(q):
    """Relative distance of q from the nearest fp32 rounding boundary (a
    midpoint between two neighbouring fp32 values)."""
    q = Fraction(q)
    if q == 0:
        return 1.0
    a = abs(q)
    ulp = _exp2(max(_binade(a), -126) - 23)
    m = a / ulp
    frac = m - (m.numerator // m.denominator)
    return float(abs(frac - Fraction(1, 2)) * ulp / a)


def fmt(q):
    """An fp32 value as a decimal string that parses back to exactly it."""
    v = float(q)
    assert Fraction(v) == q
    return repr(v)


# ------------------------------------------------------------------ SwiGLU exact
def swiglu_exact(g, u):
    """SiLU(g) * u as a Fraction accurate to ~1e-55 relative (g, u Fractions)."""
    gd = Decimal(g.numerator) / Decimal(g.denominator)
    ud = Decimal(u.numerator) / Decimal(u.denominator)
    hd = gd / (Decimal(1) + (-gd).exp()) * ud
    return Fraction(hd)


def f32_of_float(x):
    return f32(Fraction(x))


def make_cases():
    rnd = random.Random(20261203)
    cases = []
    # hand-chosen: both signs, |g| in [0.1, 4], g != u, plus zero and saturation
    hand = [(0.5, 3.0), (-0.5, 3.0), (2.0, -1.25), (-2.0, -1.25), (1.0, 1.0), (-1.0, 2.0),
            (0.125, 7.0), (-0.125, 7.0), (3.75, 0.5), (-3.75, 0.5), (0.0, 5.0), (1.5, 0.0),
            (12.0, 1.0), (-12.0, 1.0), (30.0, -2.0), (-30.0, -2.0)]
    for g, u in hand:
        cases.append((f32_of_float(g), f32_of_float(u)))
    while len(cases) < 80:
        g = f32_of_float(rnd.uniform(0.1, 4.0) * rnd.choice((-1, 1)))
        u = f32_of_float(rnd.gauss(0.0, 2.0))
        if g == u:
            continue
        cases.append((g, u))
    out = []
    for g, u in cases:
        h_exact = swiglu_exact(g, u)
        if h_exact != 0 and boundary_distance(h_exact) < 1e-9:
            continue
        out.append((g, u, f32(h_exact)))
    return out


# ------------------------------------------------------- one expert, one token
def q8_block(h):
    """Q8_0 of one block of 32 fp32 values (Fractions): d = fp32(amax / 127)
    (IEEE division), q = clamp(rne(fp32(h / d)), -127, 127)."""
    amax = max(abs(v) for v in h)
    d = f32(amax / 127)
    if d == 0:
        return [0] * len(h), d
    q = [max(-127, min(127, _rne(f32(v / d)))) for v in h]
    return q, d


def make_expert():
    """hidden H = 32, intermediate I = 32, int4 weights, one routed expert
    (top-1, one group, router weights 0 so w = routed_scaling_factor), no
    shared expert.  x = [127, 0, ..., 0]: Q8_0 scale 1, code 127 at element 0.
    Gate row r holds c_r * 2^-k_r at element 0 and 7 * 2^-k_r at element 31,
    so its int4 scale is 2^-k_r (exact) and its code at element 0 is c_r;
    hence g_r = 127 * c_r * 2^-k_r exactly.  Up rows likewise.  Down row r
    holds codes dc[r][i] * 2^-kd_r with one of them +-7, so scale 2^-kd_r."""
    rnd = random.Random(7)
    H = I = 32
    x = [Fraction(0)] * H
    x[0] = Fraction(127)
    gate = [[Fraction(0)] * H for _ in range(I)]
    up = [[Fraction(0)] * H for _ in range(I)]
    g = []
    u = []
    for r in range(I):
        while True:
            cg, kg = rnd.randint(-7, 7), rnd.choice((7, 8, 9, 10))
            cu, ku = rnd.randint(-7, 7), rnd.choice((6, 7, 8, 9))
            gv = Fraction(127 * cg) / _exp2(kg)
            uv = Fraction(127 * cu) / _exp2(ku)
            if cg != 0 and cu != 0 and gv != uv and abs(gv) < 4:
                break
        gate[r][0], gate[r][31] = Fraction(cg) / _exp2(kg), Fraction(7) / _exp2(kg)
        up[r][0], up[r][31] = Fraction(cu) / _exp2(ku), Fraction(7) / _exp2(ku)
        g.append(gv)
        u.append(uv)
    h = []
    for r in range(I):
        he = swiglu_exact(g[r], u[r])
        assert boundary_distance(he) > 1e-9, r
        h.append(f32(he))
    hq, hd = q8_block(h)
    down = [[Fraction(0)] * I for _ in range(H)]
    y = []
    ev = []
    rsf = Fraction(3, 2)
    for r in range(H):
        kd = rnd.choice((4, 5, 6))
        codes = [rnd.randint(-7, 7) for _ in range(I)]
        codes[rnd.randrange(I)] = rnd.choice((-7, 7))
        for i in range(I):
            down[r][i] = Fraction(codes[i]) / _exp2(kd)
        S = sum(codes[i] * hq[i] for i in range(I))
        e = f32(S * hd / _exp2(kd))           # one block: S * d_h * row scale
        ev.append(e)
        y.append(f32(rsf * e))                 # combine: w = rsf * s / s
    return dict(H=H, I=I, x=x, gate=gate, up=up, down=down, g=g, u=u, h=h, hq=hq, hd=hd,
                y=y, e=ev, rsf=rsf)


def write():
    src = ('# Sources: "Show HN: 遅いコンピュータで GLM 5.2 を実行する" (ja.news.hada.io/topic?id=31297),\n'
           '# section 実装済みの主な機能 (integer-dot and quantisation bullets; SwiGLU experts).\n'
           '# Written by tests/golden/make_swiglu.py from exact arithmetic (no oracle call).\n')
    with open(os.path.join(HERE, "swiglu_cases.txt"), "w") as f:
        f.write("# h = SiLU(g) * u = g / (1 + exp(-g)) * u, exact value rounded once to fp32.\n")
        f.write(src)
        f.write("# g | u | h\n")
        for g, u, h in make_cases():
            f.write("%s | %s | %s\n" % (fmt(g), fmt(u), fmt(h)))
    ex = make_expert()
    with open(os.path.join(HERE, "swiglu_expert.txt"), "w") as f:
        f.write("# One int4 expert, hidden 32, intermediate 32, one token, no shared expert;\n")
        f.write("# router weights 0 (w = routed_scaling_factor = 1.5), top-1 of 1 routed expert.\n")
        f.write(src)
        f.write("rsf: %s\n" % fmt(ex["rsf"]))
        f.write("x: %s\n" % " ".join(fmt(v) for v in ex["x"]))
        for name in ("gate", "up", "down"):
            for r, row in enumerate(ex[name]):
                f.write("%s %d: %s\n" % (name, r, " ".join(fmt(v) for v in row)))
        f.write("g: %s\n" % " ".join(fmt(v) for v in ex["g"]))
        f.write("u: %s\n" % " ".join(fmt(v) for v in ex["u"]))
        f.write("h: %s\n" % " ".join(fmt(v) for v in ex["h"]))
        f.write("hq: %s\n" % " ".join(str(v) for v in ex["hq"]))
        f.write("hd: %s\n" % fmt(ex["hd"]))
        f.write("y: %s\n" % " ".join(fmt(v) for v in ex["y"]))
        f.write("# e: the expert's output before the combine (a dense layer's output)\n")
        f.write("e: %s\n" % " ".join(fmt(v) for v in ex["e"]))


if __name__ == "__main__":
    write()
