"""Seeded synthetic inputs shared by the oracle tests and the CUDA path.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no quantisation, routing or expert math).  Every value is
an fp32 tensor drawn from a torch generator seeded from (seed, purpose,
layer, expert, matrix), so any single expert can be regenerated on its own.

Values depend on the device the generator runs on (torch's CPU and CUDA
generators are different streams); a test that compares two sides draws once
and copies the same tensor to both.

Workloads (shapes and distributions of the layer the pages describe: a
GLM-5.2-class MoE layer with hidden 6144, expert intermediate 2048, 256
routed experts + 1 shared, top-8 of 8 groups keeping 4):
  x ~ N(0, 1); router W ~ N(0, 1/H) (std 1/sqrt(H)); correction bias
  ~ U(-0.1, 0.1); expert weights ~ N(0, std 0.02); routed_scaling_factor 2.5.
"""
import hashlib
import math

import torch

GLM52 = dict(hidden=6144, inter=2048, n_routed=256, n_shared=1, top_k=8, n_group=8,
             topk_group=4, routed_scaling_factor=2.5, bits=4)

WORKLOADS = {
    # tiny layer: hidden 256, intermediate 128, 8 routed + 1 shared, top-2, one group
    "tiny_h256_e8_t4": dict(hidden=256, inter=128, n_routed=8, n_shared=1, top_k=2, n_group=1,
                            topk_group=1, routed_scaling_factor=2.5, bits=4, tokens=4, seed=0,
                            x="iid"),
    # single-token decode of the GLM-5.2-shaped layer, int4
    "glm52_decode_int4_t1": dict(GLM52, tokens=1, seed=1, x="iid"),
    # 4-token verification batch whose tokens share experts
    "glm52_verify_int4_t4": dict(GLM52, tokens=4, seed=2, x="shared"),
    # 2048-token batch-union prefill, int4
    "glm52_prefill_int4_t2048": dict(GLM52, tokens=2048, seed=3, x="iid"),
    # weight-precision sweep on the same shapes (bits in 8/4/2, tokens 1/4/512, 8 layers)
    "glm52_sweep": dict(GLM52, tokens=1, seed=4, x="iid", sweep_bits=(8, 4, 2),
                        sweep_tokens=(1, 4, 512), layers=8),
}

ROUTER_BIAS_HALF_WIDTH = 0.1
EXPERT_STD = 0.02
SHARED_X_CORR = 0.9


def workload(name, **over):
    cfg = dict(WORKLOADS[name])
    cfg.update(over)
    cfg["name"] = name
    return cfg


def layer_cfg(cfg):
    """The layer-shape keys only."""
    keys = ("hidden", "inter", "n_routed", "n_shared", "top_k", "n_group", "topk_group",
            "routed_scaling_factor", "bits")
    out = {k: cfg[k] for k in keys}
    if cfg.get("expert_top_p"):
        out["expert_top_p"] = cfg["expert_top_p"]
    return out


def seed_for(*parts):
    h = hashlib.blake2b(repr(parts).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _gen(device, *parts):
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(*parts))
    return g


def randn(shape, std, device, *parts):
    g = _gen(device, *parts)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def uniform(shape, lo, hi, device, *parts):
    g = _gen(device, *parts)
    t = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    return t.mul_(hi - lo).add_(lo)


def tokens(cfg, T=None, device="cpu", seed=None, layer=0, stream=0):
    """Activations x [T][H].  kind "shared": x1 = 0.9*x0 + sqrt(0.19)*n (unit
    variance, so tokens 0 and 1 tend to pick the same experts); other rows iid."""
    T = cfg["tokens"] if T is None else T
    seed = cfg["seed"] if seed is None else seed
    H = cfg["hidden"]
    x = randn((T, H), 1.0, device, seed, "x", layer, stream)
    if cfg.get("x") == "shared" and T >= 2:
        n = randn((H,), 1.0, device, seed, "x-noise", layer, stream)
        x[1] = SHARED_X_CORR * x[0] + math.sqrt(1.0 - SHARED_X_CORR ** 2) * n
    return x


def router(cfg, device="cpu", seed=None, layer=0):
    """(W_r [E][H] ~ N(0, 1/H), bias [E] ~ U(-0.1, 0.1))."""
    seed = cfg["seed"] if seed is None else seed
    E, H = cfg["n_routed"], cfg["hidden"]
    W = randn((E, H), 1.0 / math.sqrt(H), device, seed, "router-w", layer)
    b = uniform((E,), -ROUTER_BIAS_HALF_WIDTH, ROUTER_BIAS_HALF_WIDTH, device, seed,
                "router-b", layer)
    return W, b


def expert_fp32(cfg, e, device="cpu", seed=None, layer=0):
    """Expert e's (gate [I][H], up [I][H], down [H][I]) fp32 weights ~ N(0, 0.02^2).
    Index e == n_routed + i is shared expert i."""
    seed = cfg["seed"] if seed is None else seed
    H, I = cfg["hidden"], cfg["inter"]
    gate = randn((I, H), EXPERT_STD, device, seed, "w", layer, e, "gate")
    up = randn((I, H), EXPERT_STD, device, seed, "w", layer, e, "up")
    down = randn((H, I), EXPERT_STD, device, seed, "w", layer, e, "down")
    return gate, up, down
