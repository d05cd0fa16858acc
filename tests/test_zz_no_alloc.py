"""coli_router_static, the routing entry point that allocates nothing.

Some callers cannot allocate device memory where they route (their memory is
already handed to a caching allocator or a fixed budget, or their loop cannot
take cudaMalloc's implicit synchronisation).  coli_router_static keeps its
scratch in a fixed array inside the library, so it needs no handle.  Its
result must equal the handle-based coli_router's, call after call, even
though every call reuses the same scratch.
"""
import numpy as np
import pytest
import torch

import synth
import quantized_expert_ffn_noaux_b200 as qe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _handle(cfg, W, b, max_tokens):
    lc = synth.layer_cfg(cfg)
    lc.update(max_tokens=max_tokens)
    dummy = qe.Expert(*[(torch.zeros((cfg["inter"], cfg["hidden"] // 2), dtype=torch.uint8,
                                     device=DEV), torch.zeros(cfg["inter"], device=DEV))] * 3)
    return qe.MoELayer(lc, W, b, [dummy] * (cfg["n_routed"] + cfg["n_shared"]))


def test_router_static_matches_router_on_consecutive_calls():
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    h = _handle(cfg, W, b, max_tokens=8)
    for call, T in enumerate((4, 1, 8)):
        x = synth.tokens(cfg, T=T, device=DEV, stream=100 + call)
        idx_ref, w_ref = h.router(x)
        idx, w = qe.router_static(synth.layer_cfg(cfg), W, b, x)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), w_ref.cpu().numpy(), rtol=1e-6)
    h.close()


def test_router_static_rejects_sizes_beyond_its_scratch():
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    x = synth.tokens(cfg, T=9, device=DEV)
    with pytest.raises(qe.ColiError) as ei:
        qe.router_static(synth.layer_cfg(cfg), W, b, x)
    assert ei.value.status == qe.COLI_EINVAL and "T <=" in str(ei.value)
