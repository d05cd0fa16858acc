"""Pins of the C oracle against what the pages and the mathematics fix.

No test here re-types the oracle's formulas: each checks hand-computed values
(tests/golden), exact rational arithmetic, brute-force enumeration on tiny
inputs, invariants, or a special case that reduces to a library routine.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import golden

RNG = np.random.default_rng(12345)


# ----------------------------------------------------------------------------- Q8_0
def test_q8_hand_values():
    for x, d, q in golden.q8_blocks():
        qq, dd = oracle.quant_q8(x[None])
        assert dd[0, 0] == d, (x[:6], dd[0, 0], d)
        np.testing.assert_array_equal(qq[0], q)


def test_q8_roundtrip_and_extremes():
    x = RNG.standard_normal((64, 256)).astype(np.float32) * 3.0
    x[5, 32:64] = 0.0  # an all-zero block
    q, d = oracle.quant_q8(x)
    dq = q.astype(np.float64) * np.repeat(d.astype(np.float64), 32, axis=1)
    bound = np.repeat(d.astype(np.float64), 32, axis=1) * (0.5 + 1e-6)
    assert np.all(np.abs(x - dq) <= bound)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    # the largest element of every non-zero block maps to +-127
    xb = x.reshape(64, -1, 32)
    qb = q.reshape(64, -1, 32)
    arg = np.abs(xb).argmax(axis=2)
    top = np.take_along_axis(qb, arg[..., None], axis=2)[..., 0].astype(np.int32)
    nz = d > 0
    assert np.all(np.abs(top[nz]) == 127)
    assert np.all(q[5, 32:64] == 0) and d[5, 1] == 0.0


def test_q8_power_of_two_equivariance():
    x = RNG.standard_normal((8, 128)).astype(np.float32)
    q0, d0 = oracle.quant_q8(x)
    for k in (-7, 3, 11):
        q1, d1 = oracle.quant_q8(x * np.float32(2.0 ** k))
        np.testing.assert_array_equal(q0, q1)
        np.testing.assert_array_equal(d0 * np.float32(2.0 ** k), d1)


# --------------------------------------------------------------- weight formats
def test_weight_hand_values():
    for bits, w, s, q, by in golden.weight_rows():
        codes, scales = oracle.quant_weights(w[None], bits)
        assert scales[0] == s, (bits, scales[0], s)
        np.testing.assert_array_equal(codes[0], by)
        np.testing.assert_array_equal(oracle.unpack_weights(codes, 32, bits)[0], q)


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_unpack_is_a_bijection_on_bytes(bits):
    """Every byte value decodes to a distinct tuple of in-range codes, and each
    code value appears in every field position (all 256/16/4 values)."""
    per = 8 // bits
    allb = np.arange(256, dtype=np.uint8)[:, None]
    vals = oracle.unpack_weights(allb, per, bits)  # one byte per row
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    assert vals.min() >= lo and vals.max() <= hi
    assert len({tuple(v) for v in vals}) == 256
    for pos in range(per):
        assert set(vals[:, pos].tolist()) == set(range(lo, hi + 1))


@pytest.mark.parametrize("bits,qmax,lo,hi", [(8, 127, -127, 127), (4, 7, -8, 7), (2, 2, -2, 1)])
def test_weight_roundtrip(bits, qmax, lo, hi):
    w = (RNG.standard_normal((16, 256)) * 0.02).astype(np.float32)
    codes, s = oracle.quant_weights(w, bits)
    q = oracle.unpack_weights(codes, 256, bits).astype(np.float64)
    assert q.min() >= lo and q.max() <= hi
    amax = np.abs(w).max(axis=1)
    np.testing.assert_array_equal(s, (amax / np.float32(qmax)).astype(np.float32))
    err = np.abs(w - q * s[:, None].astype(np.float64))
    sat = q == hi  # int2 saturates +amax to +1
    assert np.all(err[~sat] <= s[:, None].repeat(256, 1)[~sat] * (0.5 + 1e-6))
    # codes of the amax element
    i = np.abs(w).argmax(axis=1)
    top = q[np.arange(16), i]
    expect = np.clip(np.sign(w[np.arange(16), i]) * qmax, lo, hi)
    np.testing.assert_array_equal(top, expect)


# ------------------------------------------------------ FP8 checkpoint weights
def test_fp8_e4m3_hand_values():
    for code, value in golden.fp8_e4m3():
        got = oracle.fp8_e4m3(code)
        if math.isnan(value):
            assert math.isnan(got), hex(code)
        else:
            assert got == value and math.copysign(1.0, got) == math.copysign(1.0, value), hex(code)


def test_fp8_e4m3_all_codes_match_torch():
    """Every one of the 256 codes decodes as torch's own float8_e4m3fn does."""
    import torch
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = np.array([oracle.fp8_e4m3(c) for c in range(256)], np.float32)
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(nan, np.isnan(got))
    np.testing.assert_array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_dequant_fp8_block_grid_on_ragged_shapes():
    """Block (r // 128, k // 128) scales element (r, k), ragged last blocks
    included: with every code 1.0 the output is the scale grid, block by block."""
    rows, K = 130, 224
    codes = np.full((rows, K), 0x38, np.uint8)          # 1.0
    scale = np.array([[0.5, 2.0], [4.0, 0.25]], np.float32)
    w = oracle.dequant_fp8(codes, scale, block=128)
    assert np.all(w[:128, :128] == 0.5) and np.all(w[:128, 128:] == 2.0)
    assert np.all(w[128:, :128] == 4.0) and np.all(w[128:, 128:] == 0.25)
    # one code per block, negative and subnormal values
    codes[0, 0], codes[129, 223], codes[5, 130] = 0xB8, 0x01, 0x7E
    w = oracle.dequant_fp8(codes, scale, block=128)
    assert w[0, 0] == -0.5 and w[129, 223] == np.float32(0.25 * 2.0 ** -9) and w[5, 130] == 896.0


def test_requant_fp8_on_hand_rows():
    """FP8 codes of the hand-computed weight rows (encoded by torch) with a
    block scale of 1 requantise to the hand-computed per-row codes."""
    import torch
    tested = 0
    for bits, w, s, q, by in golden.weight_rows():
        enc = torch.from_numpy(w).to(torch.float8_e4m3fn)
        if not torch.equal(enc.to(torch.float32), torch.from_numpy(w)):
            continue  # a row e4m3 cannot hold exactly (e.g. 127)
        codes = enc.view(torch.uint8).numpy()[None]
        c, sc = oracle.requant_fp8(codes, np.ones((1, 1), np.float32), bits, block=128)
        assert sc[0] == s
        np.testing.assert_array_equal(c[0], by)
        tested += 1
    assert tested >= 2


# -------------------------------------------------------------------- int dot
def _rand_q8(K):
    x = RNG.standard_normal(K).astype(np.float32) * RNG.uniform(0.1, 5.0)
    return oracle.quant_q8(x[None])


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_block_sums_match_integer_matmul(bits):
    K = 256
    w = (RNG.standard_normal((24, K)) * 0.02).astype(np.float32)
    codes, _ = oracle.quant_weights(w, bits)
    q = oracle.unpack_weights(codes, K, bits).astype(np.int64)
    xq, _ = _rand_q8(K)
    S = oracle.block_sums(codes, bits, K, xq)
    ref = np.einsum("rbk,bk->rb", q.reshape(24, -1, 32), xq.reshape(-1, 32).astype(np.int64))
    np.testing.assert_array_equal(S, ref)


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_int_dot_within_one_rounding_of_exact(bits):
    """out_r equals the exact rational dequantised dot rounded once to fp32
    (allowing the fp64 stage: <= 1 ulp of fp32)."""
    K = 192
    w = (RNG.standard_normal((12, K)) * 0.02).astype(np.float32)
    codes, s = oracle.quant_weights(w, bits)
    q = oracle.unpack_weights(codes, K, bits)
    xq, xd = _rand_q8(K)
    out = oracle.int_dot(codes, s, bits, K, xq, xd)
    for r in range(12):
        exact = Fraction(0)
        for k in range(K):
            exact += Fraction(int(q[r, k])) * Fraction(int(xq[0, k])) * Fraction(float(xd[0, k // 32]))
        exact *= Fraction(float(s[r]))
        ulp = np.spacing(np.float32(abs(float(exact))))
        assert abs(Fraction(float(out[r])) - exact) <= Fraction(float(ulp)), r


def test_int_dot_power_of_two_scales_equal_float_dot():
    """With power-of-two scales every partial is exact, so the int path equals a
    plain numpy float dot of the dequantised values bit for bit."""
    K, bits = 128, 4
    codes = RNG.integers(0, 256, size=(10, K // 2), dtype=np.uint8)
    s = np.float32(2.0) ** RNG.integers(-8, 2, size=10).astype(np.float32)
    xq = RNG.integers(-127, 128, size=(1, K)).astype(np.int8)
    xd = (np.float32(2.0) ** RNG.integers(-6, 3, size=K // 32)).astype(np.float32)
    out = oracle.int_dot(codes, s, bits, K, xq, xd)
    q = oracle.unpack_weights(codes, K, bits).astype(np.float64)
    xv = xq[0].astype(np.float64) * np.repeat(xd.astype(np.float64), 32)
    ref = ((q * s[:, None].astype(np.float64)) @ xv).astype(np.float32)
    np.testing.assert_array_equal(out, ref)


# -------------------------------------------------------------------- routing
def _exact_scores(x, Wr, bias):
    """l = exact sum of fp32 products (math.fsum), s = sigmoid, c = s + b."""
    E = Wr.shape[0]
    s = np.empty(E)
    for e in range(E):
        l = math.fsum(float(a) * float(b) for a, b in zip(x, Wr[e]))
        s[e] = 1.0 / (1.0 + math.exp(-l))
    return s, s + bias.astype(np.float64)


def _brute_force_route(c, E, G, gk, k):
    per = E // G
    gscore = []
    for g in range(G):
        cs = c[g * per:(g + 1) * per]
        if per == 1:
            gscore.append(cs[0])
        else:
            gscore.append(max(cs[a] + cs[b] for a, b in itertools.combinations(range(per), 2)))
    best_groups = max(itertools.combinations(range(G), gk), key=lambda gs: sum(gscore[g] for g in gs))
    cand = [e for g in best_groups for e in range(g * per, (g + 1) * per)]
    best = max(itertools.combinations(cand, k), key=lambda es: sum(c[e] for e in es))
    return set(best)


@pytest.mark.parametrize("E,G,gk,k", [(8, 1, 1, 2), (8, 4, 2, 3), (12, 3, 2, 4), (16, 4, 1, 3),
                                      (16, 8, 4, 5), (6, 6, 3, 3)])
def test_route_matches_brute_force(E, G, gk, k):
    H = 64
    for trial in range(12):
        x = RNG.standard_normal(H).astype(np.float32)
        Wr = (RNG.standard_normal((E, H)) / 8.0).astype(np.float32)
        b = RNG.uniform(-0.1, 0.1, E).astype(np.float32)
        r = oracle.route(x, Wr, b, k, G, gk, 2.5)
        s, c = _exact_scores(x, Wr, b)
        assert set(r["idx"][0].tolist()) == _brute_force_route(c, E, G, gk, k)
        # sorted by descending choice score
        cs = c[r["idx"][0]]
        assert np.all(np.diff(cs) <= 0)
        # weights: renormalised sigmoid scores times the scaling factor (bias excluded)
        sel = s[r["idx"][0]]
        np.testing.assert_allclose(r["w"][0], sel / sel.sum() * 2.5, rtol=1e-6)
        assert abs(float(r["w"][0].astype(np.float64).sum()) - 2.5) < 1e-5


@pytest.mark.parametrize("E,G,gk,k", [(8, 1, 1, 4), (16, 4, 2, 5), (12, 3, 2, 6)])
@pytest.mark.parametrize("p", [0.3, 0.5, 0.7, 0.9])
def test_top_p_keeps_a_smallest_subset_reaching_p(E, G, gk, k, p):
    """Adaptive expert top-p, checked by brute force over subsets: the kept
    experts are a smallest subset of the top-k whose scores reach p of the
    top-k's score sum, they are the largest scores, at least one is kept,
    dropped slots read -1 / 0, and the weights renormalise over the kept."""
    H = 64
    for trial in range(10):
        x = RNG.standard_normal(H).astype(np.float32)
        Wr = (RNG.standard_normal((E, H)) / 8.0).astype(np.float32)
        b = RNG.uniform(-0.1, 0.1, E).astype(np.float32)
        full = oracle.route(x, Wr, b, k, G, gk, 2.5)
        r = oracle.route(x, Wr, b, k, G, gk, 2.5, top_p=p)
        s, c = _exact_scores(x, Wr, b)
        sel = full["idx"][0].tolist()
        kept = [e for e in r["idx"][0].tolist() if e >= 0]
        assert set(kept) <= set(sel) and len(kept) >= 1
        for j, e in enumerate(r["idx"][0].tolist()):       # slots keep their places
            assert e == -1 or e == sel[j]
        if r["pmargin"][0] < 1e-9:
            continue                                       # a cut on the boundary itself
        total = sum(s[e] for e in sel)
        m = min(n for n in range(1, k + 1)
                if any(sum(s[e] for e in sub) >= p * total
                       for sub in itertools.combinations(sel, n)))
        assert len(kept) == m
        top = sorted(sel, key=lambda e: -s[e])[:m]
        assert sorted(kept) == sorted(top)
        w = r["w"][0]
        assert np.all(w[r["idx"][0] < 0] == 0)
        ks = np.array([s[e] for e in kept])
        np.testing.assert_allclose(w[r["idx"][0] >= 0], ks / ks.sum() * 2.5, rtol=1e-6)


def test_top_p_off_values_and_one_kept():
    E, H, k = 16, 64, 4
    x = RNG.standard_normal((6, H)).astype(np.float32)
    Wr = (RNG.standard_normal((E, H)) / 8.0).astype(np.float32)
    b = RNG.uniform(-0.1, 0.1, E).astype(np.float32)
    base = oracle.route(x, Wr, b, k, 4, 2, 2.5)
    for off in (0.0, 1.0, 1.5):
        r = oracle.route(x, Wr, b, k, 4, 2, 2.5, top_p=off)
        np.testing.assert_array_equal(r["idx"], base["idx"])
        np.testing.assert_array_equal(r["w"], base["w"])
    r = oracle.route(x, Wr, b, k, 4, 2, 2.5, top_p=1e-6)   # only the largest s survives
    for t in range(6):
        kept = r["idx"][t][r["idx"][t] >= 0]
        assert len(kept) == 1
        assert kept[0] == max(base["idx"][t], key=lambda e: base["s"][t][e])
        assert r["w"][t][r["idx"][t] >= 0][0] == np.float32(2.5)


def test_top_p_exact_boundary_and_ties():
    """Zero router weights make every score exactly 0.5 (the bias alone
    orders the choice): with k = 4 and p = 1/2 the first two slots reach
    exactly half the sum, so the cut falls after them -- reaching p stops the
    keeping -- and equal scores keep the earlier slots."""
    E, H, k = 8, 32, 4
    x = RNG.standard_normal((1, H)).astype(np.float32)
    Wr = np.zeros((E, H), np.float32)
    b = np.array([0.01, 0.05, 0.02, 0.07, 0.03, 0.0, 0.06, 0.04], np.float32)
    r = oracle.route(x, Wr, b, k, 1, 1, 2.0, top_p=0.5)
    assert r["idx"][0].tolist() == [3, 6, -1, -1]   # slots by c: 3, 6, 1, 7
    np.testing.assert_array_equal(r["w"][0], np.array([1.0, 1.0, 0.0, 0.0], np.float32))
    r = oracle.route(x, Wr, b, k, 1, 1, 2.0, top_p=0.75)
    assert r["idx"][0].tolist() == [3, 6, 1, -1]


def test_top_p_layer_with_one_kept_expert():
    """With a single kept expert the layer is e_shared + rsf * e_kept exactly
    (its renormalised weight is rsf: s / s = 1)."""
    rng = np.random.default_rng(31)
    cfg = _cfg(n_routed=8, top_k=3, n_group=4, topk_group=2, expert_top_p=1e-6)
    layer = _layer(cfg, rng)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    res = layer.forward(x)
    xq, xd = oracle.quant_q8(x)
    for t in range(4):
        kept = res["idx"][t][res["idx"][t] >= 0]
        assert len(kept) == 1 and res["w"][t][res["idx"][t] >= 0][0] == np.float32(2.5)
        e_sh = oracle.expert(64, 32, 4, layer.experts[-1], xq[t], xd[t])[0].astype(np.float64)
        e_k = oracle.expert(64, 32, 4, layer.experts[kept[0]], xq[t], xd[t])[0].astype(np.float64)
        np.testing.assert_array_equal(res["out"][t], (e_sh + 2.5 * e_k).astype(np.float32))
        # dropped slots carry no intermediate
        for j in np.nonzero(res["idx"][t] < 0)[0]:
            assert np.all(res["hq"][t, j] == 0) and np.all(res["hd"][t, j] == 0)


def test_route_bias_shift_invariance_and_plain_topk():
    E, H, k = 32, 64, 6
    x = RNG.standard_normal((5, H)).astype(np.float32)
    Wr = (RNG.standard_normal((E, H)) / 8.0).astype(np.float32)
    b = RNG.uniform(-0.1, 0.1, E).astype(np.float32)
    r0 = oracle.route(x, Wr, b, k, 4, 2, 2.5)
    r1 = oracle.route(x, Wr, b + np.float32(0.25), k, 4, 2, 2.5)
    np.testing.assert_array_equal(r0["idx"], r1["idx"])
    np.testing.assert_array_equal(r0["w"], r1["w"])
    # keeping every group is a plain top-k of c
    r2 = oracle.route(x, Wr, b, k, 4, 4, 2.5)
    logits = x.astype(np.float64) @ Wr.astype(np.float64).T
    c = 1.0 / (1.0 + np.exp(-logits)) + b.astype(np.float64)
    ref = np.argsort(-c, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(r2["idx"], ref)
    # no bias: top-k of the logits (sigmoid is monotone)
    r3 = oracle.route(x, Wr, np.zeros(E, np.float32), k, 1, 1, 2.5)
    np.testing.assert_array_equal(r3["idx"], np.argsort(-logits, axis=1, kind="stable")[:, :k])


def test_route_ties_go_to_lower_index():
    """Equal choice scores (duplicated router rows and biases) resolve to the
    lower expert index, and equal group scores to the lower group."""
    E, H = 8, 32
    x = RNG.standard_normal((1, H)).astype(np.float32)
    Wr = (RNG.standard_normal((E, H)) / 6.0).astype(np.float32)
    b = RNG.uniform(-0.1, 0.1, E).astype(np.float32)
    # make experts 5 and 2 the two best, exactly tied
    Wr[2] = Wr[5] = np.abs(x[0]) * np.sign(x[0]) / 4.0
    b[2] = b[5] = 0.05
    r = oracle.route(x, Wr, b, 1, 1, 1, 1.0)
    assert r["idx"][0, 0] == 2
    r = oracle.route(x, Wr, b, 2, 1, 1, 1.0)
    assert r["idx"][0].tolist() == [2, 5] and r["kmargin"][0] > 0
    # groups {0,1} and {2,3} of size 2 identical: the lower group wins
    Wr2 = np.concatenate([Wr[:2], Wr[:2], Wr[4:]])
    b2 = np.concatenate([b[:2], b[:2], b[4:]])
    r = oracle.route(x, Wr2, b2, 1, 4, 1, 1.0)
    s, c = _exact_scores(x[0], Wr2, b2)
    gs = [c[2 * g] + c[2 * g + 1] for g in range(4)]
    if max(gs) == gs[0]:
        assert r["idx"][0, 0] in (0, 1) and r["gmargin"][0] == 0.0


def test_route_margins():
    E, H = 16, 32
    x = RNG.standard_normal((20, H)).astype(np.float32)
    Wr = (RNG.standard_normal((E, H)) / 6.0).astype(np.float32)
    b = RNG.uniform(-0.1, 0.1, E).astype(np.float32)
    r = oracle.route(x, Wr, b, 3, 4, 2, 2.5)
    for t in range(20):
        s, c = _exact_scores(x[t], Wr, b)
        per = 4
        gs = sorted((sorted(c[g * per:(g + 1) * per])[-1] + sorted(c[g * per:(g + 1) * per])[-2]
                     for g in range(4)), reverse=True)
        assert abs(r["gmargin"][t] - (gs[1] - gs[2])) < 1e-12
        kept = np.argsort(-np.array(gs))  # noqa: F841  (group order only for the margin)
        cand = sorted([c[e] for e in range(E) if e // per in
                       set(np.argsort([-(sorted(c[g * per:(g + 1) * per])[-1] +
                                         sorted(c[g * per:(g + 1) * per])[-2]) for g in range(4)],
                                      kind="stable")[:2])], reverse=True)
        assert abs(r["kmargin"][t] - (cand[2] - cand[3])) < 1e-12
    r_all = oracle.route(x, Wr, b, E, 1, 1, 2.5)
    assert np.all(np.isinf(r_all["kmargin"])) and np.all(np.isinf(r_all["gmargin"]))


# ------------------------------------------------------------- expert + layer
def _layer(cfg, rng, wscale=0.02):
    H, I, E, S = cfg["hidden"], cfg["inter"], cfg["n_routed"], cfg["n_shared"]
    Wr = (rng.standard_normal((E, H)) / math.sqrt(H)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    experts = []
    for _ in range(E + S):
        g = (rng.standard_normal((I, H)) * wscale).astype(np.float32)
        u = (rng.standard_normal((I, H)) * wscale).astype(np.float32)
        d = (rng.standard_normal((H, I)) * wscale).astype(np.float32)
        experts.append(oracle.QExpert.quantise(g, u, d, cfg["bits"]))
    return oracle.Layer(cfg, Wr, b, experts)


def _cfg(**kw):
    c = dict(hidden=64, inter=32, n_routed=6, n_shared=1, top_k=2, n_group=1, topk_group=1,
             routed_scaling_factor=2.5, bits=4)
    c.update(kw)
    return c


def test_single_expert_hand_computed():
    H, I = 64, 32
    x = np.zeros((1, H), np.float32)
    x[0, 0], x[0, 32] = 127.0, 254.0

    def mats(shared):
        g = np.zeros((I, H), np.float32)
        g[0, 0], g[0, 32], g[0, 63] = 1.0, 1.0, 7.0
        u = np.zeros((I, H), np.float32)
        u[0, 32], u[0, 63] = 0.5, 0.875
        d = np.zeros((H, I), np.float32)
        for r in range(H):
            d[r, 0] = 1.0 if shared else float((r % 15) - 7)
            d[r, 31] = 7.0
        return oracle.QExpert.quantise(g, u, d, 4)

    cfg = _cfg(n_routed=1, top_k=1)
    layer = oracle.Layer(cfg, np.zeros((1, H), np.float32), np.zeros(1, np.float32),
                         [mats(False), mats(True)])
    res = layer.forward(x)
    np.testing.assert_array_equal(res["out"][0], golden.single_expert_y())
    assert res["w"][0, 0] == np.float32(2.5)
    assert res["hq"][0, 0, 0] == 127 and np.all(res["hq"][0, 0, 1:] == 0)
    assert res["hd"][0, 0, 0] == np.float32(381.0)


def test_swiglu_hand_values():
    """h = SiLU(g) * u against its exact value rounded once to fp32
    (tests/golden/make_swiglu.py), for |g| in [0.1, 4] of both signs, g != u,
    and the zero and saturated cases."""
    cases = golden.swiglu_cases()
    g = np.array([c[0] for c in cases], np.float32)
    u = np.array([c[1] for c in cases], np.float32)
    h = np.array([c[2] for c in cases], np.float32)
    np.testing.assert_array_equal(oracle.swiglu(g, u), h)


def test_swiglu_fixture_separates_plausible_mistakes():
    """The fixture has teeth: dropping the sigmoid, gating u instead of g,
    ReLU in place of SiLU and sigmoid(+g) each disagree with it in most of the
    unsaturated cases (so any of them in the oracle fails the pin above)."""
    cases = [c for c in golden.swiglu_cases() if 0.1 <= abs(float(c[0])) <= 4.0
             and float(c[1]) != 0.0]
    assert len(cases) >= 40
    g = np.array([c[0] for c in cases], np.float64)
    u = np.array([c[1] for c in cases], np.float64)
    h = np.array([c[2] for c in cases], np.float32)
    sig = lambda v: 1.0 / (1.0 + np.exp(-v))  # noqa: E731
    wrong = {
        "no sigmoid": g * u,
        "SiLU of u": u * sig(u) * g,
        "ReLU": np.maximum(g, 0.0) * u,
        "sigmoid(+g)": g / (1.0 + np.exp(g)) * u,
    }
    for name, v in wrong.items():
        assert np.mean(v.astype(np.float32) != h) > 0.9, name


def test_swiglu_expert_exact():
    """One int4 expert whose g and u are exact fp32 values with |g| < 4:
    the oracle's g, u, Q8_0(h) codes and scale and output y equal the values
    make_swiglu.py derived by exact arithmetic."""
    ex = golden.swiglu_expert()
    H = I = 32
    q = oracle.QExpert.quantise(ex["gate"], ex["up"], ex["down"], 4)
    xq, xd = oracle.quant_q8(ex["x"])
    np.testing.assert_array_equal(oracle.int_dot(*q.gate, 4, H, xq, xd), ex["g"])
    np.testing.assert_array_equal(oracle.int_dot(*q.up, 4, H, xq, xd), ex["u"])
    e, hq, hd = oracle.expert(H, I, 4, q, xq, xd)
    np.testing.assert_array_equal(hq, ex["hq"])
    assert hd[0] == ex["hd"]
    cfg = _cfg(hidden=H, inter=I, n_routed=1, n_shared=0, top_k=1,
               routed_scaling_factor=ex["rsf"])
    layer = oracle.Layer(cfg, np.zeros((1, H), np.float32), np.zeros(1, np.float32), [q])
    res = layer.forward(ex["x"])
    np.testing.assert_array_equal(res["hq"][0, 0], ex["hq"])
    np.testing.assert_array_equal(res["out"][0], ex["y"])


def test_dense_layer_hand_computed():
    """A dense layer (no router, the expert as its one shared expert, weight 1)
    on the exact unsaturated expert outputs the expert's exact e."""
    ex = golden.swiglu_expert()
    H = I = 32
    q = oracle.QExpert.quantise(ex["gate"], ex["up"], ex["down"], 4)
    cfg = _cfg(hidden=H, inter=I, n_routed=0, n_shared=1, top_k=0)
    layer = oracle.Layer(cfg, np.zeros((0, H), np.float32), np.zeros(0, np.float32), [q])
    res = layer.forward(ex["x"])
    np.testing.assert_array_equal(res["out"][0], ex["e"])
    np.testing.assert_array_equal(res["hq"][0, 0], ex["hq"])


def test_dense_layer_equals_moe_without_routed_weight():
    """Dense layer == the same shared expert inside a MoE layer whose routed
    weights are all zero (routed_scaling_factor 0), bit for bit."""
    rng = np.random.default_rng(21)
    moe = _layer(_cfg(n_routed=4, top_k=2, routed_scaling_factor=0.0), rng)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    dense = oracle.Layer(_cfg(n_routed=0, top_k=0), np.zeros((0, 64), np.float32),
                         np.zeros(0, np.float32), [moe.experts[-1]])
    np.testing.assert_array_equal(dense.forward(x)["out"], moe.forward(x)["out"])


def test_dense_mixture_when_k_equals_E():
    """top_k = E with one group: every expert is used with weight
    rsf * s_i / sum(s), so y = e_shared + rsf * sum_i (s_i / sum s) e_i."""
    rng = np.random.default_rng(7)
    cfg = _cfg(n_routed=5, top_k=5)
    layer = _layer(cfg, rng)
    x = rng.standard_normal((3, 64)).astype(np.float32)
    y = layer.forward(x)["out"]
    xq, xd = oracle.quant_q8(x)
    logits = x.astype(np.float64) @ layer.Wr.astype(np.float64).T
    s = 1.0 / (1.0 + np.exp(-logits))
    for t in range(3):
        es = [oracle.expert(64, 32, 4, ex, xq[t], xd[t])[0].astype(np.float64)
              for ex in layer.experts]
        ref = es[5] + 2.5 * sum(s[t, i] / s[t].sum() * es[i] for i in range(5))
        np.testing.assert_allclose(y[t], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def test_linearity_in_scaling_factor():
    rng = np.random.default_rng(8)
    cfg = _cfg()
    layer = _layer(cfg, rng)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    ys = {}
    for rsf in (0.0, 1.0, 2.5):
        layer.cfg["routed_scaling_factor"] = rsf
        ys[rsf] = layer.forward(x)["out"].astype(np.float64)
    scale = np.abs(ys[2.5]).max()
    np.testing.assert_allclose(ys[2.5] - ys[0.0], 2.5 * (ys[1.0] - ys[0.0]), atol=1e-5 * scale)
    # rsf = 0 leaves only the shared expert
    xq, xd = oracle.quant_q8(x)
    e_sh = oracle.expert(64, 32, 4, layer.experts[-1], xq[0], xd[0])[0]
    np.testing.assert_array_equal(ys[0.0][0].astype(np.float32), e_sh)


def test_relabelling_experts_leaves_output_unchanged():
    rng = np.random.default_rng(9)
    cfg = _cfg(n_routed=8, top_k=3, n_group=4, topk_group=2)
    layer = _layer(cfg, rng)
    x = rng.standard_normal((6, 64)).astype(np.float32)
    base = layer.forward(x)
    # permute groups as blocks and experts inside each group
    gperm = [2, 0, 3, 1]
    perm = []
    for g in gperm:
        inner = [2 * g, 2 * g + 1]
        if g % 2:
            inner.reverse()
        perm += inner
    perm = np.array(perm)
    relab = oracle.Layer(cfg, layer.Wr[perm], layer.bias[perm],
                         [layer.experts[p] for p in perm] + [layer.experts[-1]])
    res = relab.forward(x)
    np.testing.assert_array_equal(res["out"], base["out"])
    np.testing.assert_array_equal(perm[res["idx"]], base["idx"])


def test_overrides_reproduce_own_decisions():
    rng = np.random.default_rng(10)
    cfg = _cfg(n_routed=8, top_k=2)
    layer = _layer(cfg, rng)
    x = rng.standard_normal((3, 64)).astype(np.float32)
    a = layer.forward(x)
    b = layer.forward(x, idx_in=a["idx"], hq_in=a["hq"], hd_in=a["hd"])
    np.testing.assert_array_equal(a["out"], b["out"])
    # a different (valid) choice changes the output
    idx2 = a["idx"].copy()
    idx2[0, 1] = [e for e in range(8) if e not in idx2[0]][0]
    c = layer.forward(x, idx_in=idx2)
    assert not np.array_equal(c["out"][0], a["out"][0])
    np.testing.assert_array_equal(c["out"][1:], a["out"][1:])


def test_missing_expert_is_reported():
    rng = np.random.default_rng(11)
    cfg = _cfg(n_routed=4, top_k=1)
    layer = _layer(cfg, rng)
    x = rng.standard_normal((1, 64)).astype(np.float32)
    e = layer.route(x)["idx"][0, 0]
    layer.experts[e] = None
    with pytest.raises(KeyError):
        layer.forward(x)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(12)
    layer = _layer(_cfg(n_routed=8, top_k=2), rng)
    x = rng.standard_normal((9, 64)).astype(np.float32)
    np.testing.assert_array_equal(layer.forward(x, nthreads=1)["out"],
                                  layer.forward(x, nthreads=4)["out"])
