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


__all__ = ["q8_blocks", "weight_rows", "single_expert_y", "Fraction"]
