"""Shared helpers of the GPU parity tests: build one layer on both sides from
the same seeded fp32 tensors, and compare the CUDA path with the oracle.

The CUDA side quantises its weights with its own kernel; the oracle quantises
host copies of the same fp32 tensors with its own C code.  Weight codes are
compared bit for bit wherever both sides have them.
"""
import itertools

import numpy as np
import torch

import oracle
import synth
import quantized_expert_ffn_noaux_b200 as qe

REL_TOL = 2e-4          # ||y - y_ref||_inf <= REL_TOL * ||y_ref||_inf, per token row
MARGIN = 1e-5           # routing decisions closer than this may go either way


class GpuLayer:
    """Weights of one layer generated on the GPU; the handle; lazy oracle copies."""

    def __init__(self, cfg, max_tokens, layer=0, device="cuda", gen_device=None, seed=None):
        self.cfg = dict(cfg)
        self.layer = layer
        self.seed = cfg["seed"] if seed is None else seed
        self.device = device
        self.gen_device = gen_device or device
        E, S, bits = cfg["n_routed"], cfg["n_shared"], cfg["bits"]
        W, b = synth.router(cfg, device=self.gen_device, seed=self.seed, layer=layer)
        self.Wr, self.bias = W.to(device), b.to(device)
        self.experts = []
        for e in range(E + S):
            g, u, d = self.expert_fp32(e)
            self.experts.append(qe.Expert.quantise(g, u, d, bits))
            del g, u, d
        lc = synth.layer_cfg(cfg)
        lc["max_tokens"] = max_tokens
        self.handle = qe.MoELayer(lc, self.Wr, self.bias, self.experts)
        self._oracle_experts = {}

    def expert_fp32(self, e):
        g, u, d = synth.expert_fp32(self.cfg, e, device=self.gen_device, seed=self.seed,
                                    layer=self.layer)
        return g.to(self.device), u.to(self.device), d.to(self.device)

    def oracle_expert(self, e, check_codes=True):
        """QExpert quantised by the oracle from host copies of the fp32 weights;
        also checks the CUDA quantiser produced identical codes and scales."""
        if e not in self._oracle_experts:
            mats = [m.cpu().numpy() for m in self.expert_fp32(e)]
            qx = oracle.QExpert.quantise(*mats, bits=self.cfg["bits"])
            if check_codes:
                gpu = self.experts[e]
                for (oc, os_), (gc, gs) in zip((qx.gate, qx.up, qx.down),
                                               (gpu.gate, gpu.up, gpu.down)):
                    np.testing.assert_array_equal(gc.cpu().numpy(), oc)
                    np.testing.assert_array_equal(gs.cpu().numpy(), os_)
            self._oracle_experts[e] = qx
        return self._oracle_experts[e]

    def oracle_layer(self, experts_needed):
        E, S = self.cfg["n_routed"], self.cfg["n_shared"]
        exs = [None] * (E + S)
        for e in set(experts_needed) | set(range(E, E + S)):
            exs[e] = self.oracle_expert(e)
        return oracle.Layer(synth.layer_cfg(self.cfg), self.Wr.cpu().numpy(),
                            self.bias.cpu().numpy(), exs)

    def close(self):
        self.handle.close()


def decidable(route_res, t):
    ok = route_res["kmargin"][t] > MARGIN and route_res["gmargin"][t] > MARGIN
    if "pmargin" in route_res:  # the adaptive expert top-p's cut
        ok = ok and route_res["pmargin"][t] > MARGIN
    return ok


def _group_scores(c, G):
    """Sum of the two largest choice scores of each group (one if a group has
    a single expert)."""
    per = c.shape[0] // G
    cg = np.sort(c.reshape(G, per), axis=1)[:, ::-1]
    return cg[:, 0] + (cg[:, 1] if per > 1 else 0.0)


def valid_tie_choice(sel, c, G, gk, k, margin=MARGIN):
    """Whether the expert set `sel` is a correct selection for choice scores
    `c` once every comparison closer than `margin` may go either way: some
    set K of gk groups holds every group whose score is clearly above the
    gk-th and none clearly below it, `sel` is k distinct experts of K's
    groups, and every expert of K left out of `sel` is not clearly above any
    expert in it (a valid alternative of the group-limited top-k)."""
    sel = [int(e) for e in sel]
    E = c.shape[0]
    if len(sel) != k or len(set(sel)) != k or min(sel) < 0 or max(sel) >= E:
        return False
    per = E // G
    gs = _group_scores(c, G)
    theta = np.sort(gs)[::-1][gk - 1]
    must = [g for g in range(G) if gs[g] > theta + margin]
    may = [g for g in range(G) if abs(gs[g] - theta) <= margin]
    if not set(e // per for e in sel) <= set(must) | set(may):
        return False
    for fill in itertools.combinations(may, gk - len(must)):
        kept = set(must) | set(fill)
        if not all(e // per in kept for e in sel):
            continue
        rest = [e for e in range(E) if e // per in kept and e not in sel]
        lo = min(c[e] for e in sel)
        if all(c[e] <= lo + margin for e in rest):
            return True
    return False


def check_route(gpu_idx, gpu_w, ref, tokens=None, G=None, gk=None, rsf=None):
    """Bit-exact idx for decidable tokens (as sets, order where the c gap is
    clear); weights within 1e-6 relative of the renormalised sigmoid scores of
    the chosen set.  Undecidable tokens (a routing margin within 1e-5) must
    carry a valid tie alternative (valid_tie_choice) sorted by descending c up
    to the margin.  Returns the undecidable tokens."""
    gpu_idx = np.asarray(gpu_idx)
    gpu_w = np.asarray(gpu_w)
    tokens = range(gpu_idx.shape[0]) if tokens is None else tokens
    loose = []
    for i, t in enumerate(tokens):
        gi, ri = gpu_idx[i], ref["idx"][t]
        c = ref["c"][t]
        if (gi < 0).any() or (ri < 0).any():
            # adaptive expert top-p dropped slots (-1, weight 0; slots keep their places)
            kept = gi[gi >= 0]
            assert len(set(kept.tolist())) == len(kept) and len(kept) >= 1, (t, gi)
            assert np.all(gpu_w[i][gi < 0] == 0), (t, gi, gpu_w[i])
            if decidable(ref, t):
                np.testing.assert_array_equal(gi, ri)
                np.testing.assert_allclose(gpu_w[i], ref["w"][t], rtol=1e-6)
            else:
                s = ref["s"][t][kept]
                scale = float(ref["w"][t].astype(np.float64).sum()) if rsf is None else rsf
                np.testing.assert_allclose(gpu_w[i][gi >= 0], s / s.sum() * scale, rtol=1e-6)
                loose.append(i)
            continue
        if not decidable(ref, t):
            assert G is not None and gk is not None, "check_route needs G, gk for near ties"
            assert valid_tie_choice(gi, c, G, gk, len(ri)), (t, gi, ri)
            for j in range(len(gi) - 1):
                assert c[gi[j]] >= c[gi[j + 1]] - MARGIN, (t, j, gi)
            s = ref["s"][t][gi]
            scale = float(ref["w"][t].astype(np.float64).sum()) if rsf is None else rsf
            np.testing.assert_allclose(gpu_w[i], s / s.sum() * scale, rtol=1e-6)
            loose.append(i)
            continue
        assert set(gi.tolist()) == set(ri.tolist()), (t, gi, ri)
        for j in range(len(ri) - 1):
            if c[ri[j]] - c[ri[j + 1]] > MARGIN:
                assert gi[j] == ri[j], (t, j, gi, ri)
        np.testing.assert_allclose(gpu_w[i], ref["w"][t], rtol=1e-6)
    return loose


def check_out_rows(y, y_ref, what=""):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    for t in range(y.shape[0]):
        scale = np.abs(y_ref[t]).max()
        err = np.abs(y[t] - y_ref[t]).max()
        assert err <= REL_TOL * scale, "%s token %d: err %.3g > %.1e * %.3g" % (what, t, err,
                                                                                 REL_TOL, scale)


def compare_forward(gl, x_dev, tokens=None, check_h=True):
    """Run the CUDA layer on x_dev [T][H]; compare the tokens in `tokens`
    (default all) with the oracle.  Returns (gpu out, oracle result)."""
    T = x_dev.shape[0]
    out = gl.handle.forward(x_dev)
    idx, w, hq, hd = gl.handle.dbg_last_forward(T)
    torch.cuda.synchronize()
    tokens = list(range(T)) if tokens is None else list(tokens)
    x_host = x_dev.cpu().numpy()[tokens]
    out = out.cpu().numpy()[tokens]
    idx, w = idx.cpu().numpy()[tokens], w.cpu().numpy()[tokens]
    hq, hd = hq.cpu().numpy()[tokens], hd.cpu().numpy()[tokens]
    if gl.cfg["n_routed"] == 0:  # a dense layer: no routing to compare
        layer = gl.oracle_layer(set())
        ref = layer.forward(x_host, nthreads=oracle.n_threads_default())
    else:
        # the oracle routes the sampled tokens itself
        probe = oracle.Layer(synth.layer_cfg(gl.cfg), gl.Wr.cpu().numpy(), gl.bias.cpu().numpy(),
                             [None] * (gl.cfg["n_routed"] + gl.cfg["n_shared"]))
        ref_route = probe.route(x_host)
        loose = check_route(idx, w, ref_route, G=gl.cfg["n_group"], gk=gl.cfg["topk_group"],
                            rsf=gl.cfg["routed_scaling_factor"])
        need = set(idx.reshape(-1).tolist()) | set(ref_route["idx"].reshape(-1).tolist())
        need.discard(-1)  # a slot the adaptive expert top-p dropped
        layer = gl.oracle_layer(need)
        # undecidable tokens: the oracle re-runs with the CUDA side's choice, which
        # check_route has confirmed to be a valid tie alternative
        idx_in = ref_route["idx"].copy()
        for i in loose:
            idx_in[i] = idx[i]
        ref = layer.forward(x_host, idx_in=idx_in, nthreads=oracle.n_threads_default())
    if check_h:
        np.testing.assert_array_equal(hq, ref["hq"])
        np.testing.assert_array_equal(hd, ref["hd"])
    check_out_rows(out, ref["out"])
    return out, ref
