"""Readers for the hand-computed fixtures in this folder (plain text, one case per line)."""
import os
from fractions import Fraction

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _lines(name):
    with open(os.path.join(HERE, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


def _f32_of(tok):
    """'a/b' means the fp32 quotient fp32(a) / fp32(b); otherwise fp32(tok)."""
    if "/" in tok:
        a, b = tok.split("/")
        return np.float32(np.float32(float(a)) / np.float32(float(b)))
    return np.float32(float(tok))


def q8_blocks():
    out = []
    for ln in _lines("q8_blocks.txt"):
        parts = dict(p.strip().split(":", 1) for p in ln.split("|"))
        x = np.zeros(32, np.float32)
        xs = [float(v) for v in parts["x"].split()]
        x[:len(xs)] = xs
        q = np.zeros(32, np.int8)
        qs = [int(v) for v in parts["q"].split()]
        q[:len(qs)] = qs
        out.append((x, _f32_of(parts["d"].strip()), q))
    return out


def weight_rows():
    out = []
    for ln in _lines("weight_rows.txt"):
        fields = [p.strip() for p in ln.split("|")]
        bits = int(fields[0])
        kv = dict(p.split(":", 1) for p in fields[1:])
        w = np.zeros(32, np.float32)
        ws = [float(v) for v in kv["w"].split()]
        w[:len(ws)] = ws
        q = np.zeros(32, np.int8)
        qs = [int(v) for v in kv["q"].split()]
        q[:len(qs)] = qs
        nbytes = 32 * bits // 8
        by = np.zeros(nbytes, np.uint8)
        bs = [int(v, 16) for v in kv["bytes"].split()]
        by[:len(bs)] = bs
        out.append((bits, w, _f32_of(kv["s"].strip()), q, by))
    return out


def single_expert_y():
    ys = []
    for ln in _lines("single_expert_exact.txt"):
        assert ln.startswith("y:")
        ys += [float(v) for v in ln[2:].split()]
    return np.array(ys, np.float32)


def swiglu_cases():
    """[(g, u, h)] fp32 triples from swiglu_cases.txt."""
    out = []
    for ln in _lines("swiglu_cases.txt"):
        g, u, h = (np.float32(float(v)) for v in ln.split("|"))
        out.append((g, u, h))
    return out


def swiglu_expert():
    """The one-expert case of swiglu_expert.txt as a dict of numpy arrays:
    x [1][32], gate/up [32][32], down [32][32] fp32; g, u, h [32] fp32;
    hq [32] int8; hd fp32 scalar; y [32] fp32; rsf float."""
    rows = {"gate": {}, "up": {}, "down": {}}
    d = {}
    for ln in _lines("swiglu_expert.txt"):
        key, val = ln.split(":", 1)
        parts = key.split()
        if parts[0] in rows:
            rows[parts[0]][int(parts[1])] = [float(v) for v in val.split()]
        else:
            d[key.strip()] = val.split()
    out = {name: np.array([m[r] for r in range(len(m))], np.float32) for name, m in rows.items()}
    out["x"] = np.array([[float(v) for v in d["x"]]], np.float32)
    for k in ("g", "u", "h", "y", "e"):
        out[k] = np.array([float(v) for v in d[k]], np.float32)
    out["hq"] = np.array([int(v) for v in d["hq"]], np.int8)
    out["hd"] = np.float32(float(d["hd"][0]))
    out["rsf"] = float(d["rsf"][0])
    return out


def fp8_e4m3():
    """[(code, value)] from fp8_e4m3.txt (value a Python float, nan allowed)."""
    out = []
    for ln in _lines("fp8_e4m3.txt"):
        c, v = (t.strip() for t in ln.split("|"))
        out.append((int(c, 16), float(v)))
    return out


__all__ = ["fp8_e4m3", "q8_blocks", "weight_rows", "single_expert_y", "swiglu_cases", "swiglu_expert",
           "Fraction"]
