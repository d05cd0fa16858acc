"""The seeded generators: shapes, determinism, independence of experts."""
import math

import numpy as np
import torch

import synth


def test_workload_shapes_and_determinism():
    cfg = synth.workload("tiny_h256_e8_t4")
    x = synth.tokens(cfg)
    assert x.shape == (4, 256) and x.dtype == torch.float32
    assert torch.equal(x, synth.tokens(cfg))
    W, b = synth.router(cfg)
    assert W.shape == (8, 256) and b.shape == (8,)
    assert float(b.abs().max()) <= 0.1
    g, u, d = synth.expert_fp32(cfg, 3)
    assert g.shape == (128, 256) and u.shape == (128, 256) and d.shape == (256, 128)
    g2, _, _ = synth.expert_fp32(cfg, 4)
    assert not torch.equal(g, g2)
    assert abs(float(g.std()) - 0.02) < 0.002
    assert abs(float(W.std()) - 1 / math.sqrt(256)) < 0.01


def test_shared_tokens_are_correlated():
    cfg = synth.workload("glm52_verify_int4_t4", hidden=512)
    x = synth.tokens(cfg).numpy().astype(np.float64)
    r01 = np.corrcoef(x[0], x[1])[0, 1]
    r23 = np.corrcoef(x[2], x[3])[0, 1]
    assert r01 > 0.8 and abs(r23) < 0.2
