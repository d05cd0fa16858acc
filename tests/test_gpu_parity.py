"""CUDA path vs the oracle, element by element, through the C ABI.

Bit-exact: Q8_0 codes and scales, weight codes and scales, int32 block sums,
routing indices of decidable tokens, intermediate Q8_0(h) codes.  fp32
outputs: ||y_t - y_ref,t||_inf <= 2e-4 * ||y_ref,t||_inf per token.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_expert_ffn_noaux_b200 as qe
from tests.parity_util import GpuLayer, check_out_rows, check_route, compare_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ quantisers
@pytest.mark.parametrize("rows,n", [(1, 32), (3, 256), (17, 6144), (2048, 6144)])
def test_quant_q8_bitexact(rows, n):
    r = _rng(rows)
    x = (r.standard_normal((rows, n)) * r.uniform(0.01, 50.0, (rows, 1))).astype(np.float32)
    x[0, :32] = 0.0                      # zero block
    if rows > 1:
        x[1, 32:64] = 0.5 * np.sign(x[1, 32:64])   # exact halves -> round half even
    q, d = qe.quant_q8(torch.from_numpy(x).to(DEV))
    qo, do = oracle.quant_q8(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(d.cpu().numpy(), do)


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("rows,K", [(1, 64), (33, 256), (300, 6144), (6144, 2048)])
def test_quant_weights_bitexact(bits, rows, K):
    r = _rng(rows + K + bits)
    w = (r.standard_normal((rows, K)) * 0.02).astype(np.float32)
    w[0, :] = 0.0
    if rows > 2:
        w[2, :8] = [0.5, -0.5, 1.5, 2.5, -7.0, 7.0, 3.5, 1.0]
    c, s = qe.quant_weights(torch.from_numpy(w).to(DEV), bits)
    co, so = oracle.quant_weights(w, bits)
    np.testing.assert_array_equal(c.cpu().numpy(), co)
    np.testing.assert_array_equal(s.cpu().numpy(), so)


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("rows,K,T", [(5, 64, 1), (64, 256, 3), (96, 6144, 2), (200, 2048, 4)])
def test_block_sums_bitexact(bits, rows, K, T):
    r = _rng(rows * K + bits)
    w = (r.standard_normal((rows, K)) * 0.02).astype(np.float32)
    x = r.standard_normal((T, K)).astype(np.float32)
    codes, _ = oracle.quant_weights(w, bits)
    xq, _ = oracle.quant_q8(x)
    S = qe.dbg_block_sums(torch.from_numpy(codes).to(DEV), bits, K,
                          torch.from_numpy(xq).to(DEV)).cpu().numpy()
    for t in range(T):
        np.testing.assert_array_equal(S[t], oracle.block_sums(codes, bits, K, xq[t]))


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("T", [1, 4, 8, 9, 100])
def test_router_glm52_shape(T):
    cfg = synth.workload("glm52_decode_int4_t1")
    W, b = synth.router(cfg, device=DEV)
    x = synth.tokens(cfg, T=T, device=DEV, stream=T)
    lc = synth.layer_cfg(cfg)
    lc.update(max_tokens=max(T, 1))
    # a handle needs experts; one tiny shared set of pointers is enough for routing
    dummy = qe.Expert(*[(torch.zeros((cfg["inter"], cfg["hidden"] // 2), dtype=torch.uint8,
                                     device=DEV), torch.zeros(cfg["inter"], device=DEV))] * 3)
    h = qe.MoELayer(lc, W, b, [dummy] * (cfg["n_routed"] + cfg["n_shared"]))
    idx, w = h.router(x)
    ref = oracle.route(x.cpu().numpy(), W.cpu().numpy(), b.cpu().numpy(), cfg["top_k"],
                       cfg["n_group"], cfg["topk_group"], cfg["routed_scaling_factor"])
    loose = check_route(idx.cpu().numpy(), w.cpu().numpy(), ref, G=cfg["n_group"],
                        gk=cfg["topk_group"], rsf=cfg["routed_scaling_factor"])
    assert len(loose) <= max(1, T // 50)
    h.close()


# ------------------------------------------------------------------ layers
def _small_cfg(**kw):
    c = dict(hidden=256, inter=128, n_routed=8, n_shared=1, top_k=2, n_group=1, topk_group=1,
             routed_scaling_factor=2.5, bits=4, seed=0, x="iid", tokens=4)
    c.update(kw)
    return c


def test_tiny_layer_all_tokens():
    cfg = synth.workload("tiny_h256_e8_t4")
    gl = GpuLayer(cfg, max_tokens=4)
    x = synth.tokens(cfg, device=DEV)
    compare_forward(gl, x)
    gl.close()


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("T", [1, 3, 8, 9, 37])
def test_small_layers_every_path(bits, T):
    """Several tiles and a ragged tail: hidden 384 (12 blocks), inter 320
    (10 row chunks), 16 experts in 4 groups; T spans the few-token path
    (T <= 8) and the grouped path (T > 8)."""
    cfg = _small_cfg(hidden=384, inter=320, n_routed=16, n_group=4, topk_group=2, top_k=3,
                     bits=bits, seed=100 + T)
    if bits == 2:
        cfg.update(hidden=384, inter=384)
    gl = GpuLayer(cfg, max_tokens=max(T, 9))
    x = synth.tokens(cfg, T=T, device=DEV)
    compare_forward(gl, x)
    gl.close()


def test_no_shared_expert_and_dense_topk():
    cfg = _small_cfg(n_shared=0, n_routed=6, top_k=6, seed=5)
    gl = GpuLayer(cfg, max_tokens=5)
    compare_forward(gl, synth.tokens(cfg, T=5, device=DEV))
    gl.close()


def test_two_shared_experts_and_max_tokens():
    cfg = _small_cfg(n_shared=2, seed=6)
    gl = GpuLayer(cfg, max_tokens=12)
    compare_forward(gl, synth.tokens(cfg, T=12, device=DEV))
    gl.close()


def test_repeated_forward_is_bit_identical():
    cfg = _small_cfg(seed=7)
    gl = GpuLayer(cfg, max_tokens=16)
    x = synth.tokens(cfg, T=16, device=DEV)
    a = gl.handle.forward(x).cpu()
    b = gl.handle.forward(x).cpu()
    y = synth.tokens(cfg, T=3, device=DEV, stream=1)
    gl.handle.forward(y)
    c = gl.handle.forward(x).cpu()
    assert torch.equal(a, b) and torch.equal(a, c)
    gl.close()


def test_forward_host_matches_device_path():
    cfg = _small_cfg(seed=8)
    gl = GpuLayer(cfg, max_tokens=8)
    x = synth.tokens(cfg, T=8, device=DEV)
    y_dev = gl.handle.forward(x).cpu()
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    gl.handle.forward_host(xh, yh)
    assert torch.equal(y_dev, yh)
    gl.close()


def test_invalid_arguments_are_rejected():
    cfg = _small_cfg(seed=9)
    gl = GpuLayer(cfg, max_tokens=4)
    x = synth.tokens(cfg, T=4, device=DEV)
    h = gl.handle
    L = qe.lib()
    s = qe._stream()
    out = torch.empty_like(x)
    assert L.coli_moe_forward(h._h, qe._ptr(x), 0, qe._ptr(out), s) == qe.COLI_EINVAL
    assert L.coli_moe_forward(h._h, qe._ptr(x), 5, qe._ptr(out), s) == qe.COLI_EINVAL
    assert L.coli_moe_forward(h._h, None, 4, qe._ptr(out), s) == qe.COLI_EINVAL
    assert L.coli_moe_forward(h._h, qe._ptr(x), 4, qe._ptr(x), s) == qe.COLI_EINVAL
    mis = torch.empty(4 * 256 + 4, device=DEV)[1:1 + 4 * 256].view(4, 256)
    assert L.coli_moe_forward(h._h, qe._ptr(mis), 4, qe._ptr(out), s) == qe.COLI_EINVAL
    assert L.coli_quant_q8(qe._ptr(x), 4, 33, qe._ptr(out), qe._ptr(out), s) == qe.COLI_EINVAL
    assert L.coli_dbg_last_forward(h._h, 3, None, None, None, None, s) == qe.COLI_EINVAL
    torch.cuda.synchronize()
    # the handle still works afterwards
    compare_forward(gl, x)
    gl.close()


def test_bounded_wait_reports_timeout_and_handle_recovers():
    """A device wait that nothing satisfies gives up after about a second and
    is reported as COLI_ETIMEOUT; the handle keeps working afterwards."""
    cfg = _small_cfg(seed=10)
    gl = GpuLayer(cfg, max_tokens=4)
    assert gl.handle.device_status() == qe.COLI_OK
    gl.handle.dbg_wait_probe()
    assert gl.handle.device_status() == qe.COLI_ETIMEOUT
    assert gl.handle.device_status() == qe.COLI_OK
    compare_forward(gl, synth.tokens(cfg, T=4, device=DEV))
    assert gl.handle.device_status() == qe.COLI_OK
    gl.close()


@pytest.mark.parametrize("path", ["decode", "tensor_cores"])
def test_real_kernels_give_up_under_a_short_wait_limit(path):
    """A short per-handle wait limit makes the waits inside the layer's own
    kernels run out (the persistent decode kernel; the tcgen05 grouped GEMMs):
    every forward then either completes or reports COLI_ETIMEOUT -- nothing
    hangs or faults -- at least one reports it, and with the default limit
    back the same handle computes the layer exactly as before."""
    if path == "decode":
        cfg = _small_cfg(hidden=384, inter=320, n_routed=16, n_group=4, topk_group=2, top_k=3,
                         seed=11)
        T = 4
    else:
        cfg = _small_cfg(hidden=512, inter=256, n_routed=16, n_group=4, topk_group=2, top_k=3,
                         seed=12)
        T = 37
    gl = GpuLayer(cfg, max_tokens=T)
    x = synth.tokens(cfg, T=T, device=DEV)
    y0, _ = compare_forward(gl, x)
    seen = []
    for cycles in (100, 1000, 10000, 100000):
        gl.handle.dbg_set_wait_limit(cycles)
        gl.handle.forward(x)
        seen.append(gl.handle.device_status())
    gl.handle.dbg_set_wait_limit(0)
    assert set(seen) <= {qe.COLI_OK, qe.COLI_ETIMEOUT}, seen
    assert qe.COLI_ETIMEOUT in seen, seen
    assert gl.handle.device_status() == qe.COLI_OK
    y1, _ = compare_forward(gl, x)
    np.testing.assert_array_equal(y0, y1)
    gl.close()


# ------------------------------------------------------- full-size workloads
@pytest.fixture(scope="module")
def glm52_layer():
    cfg = synth.workload("glm52_decode_int4_t1")
    gl = GpuLayer(cfg, max_tokens=2048)
    yield gl
    gl.close()
    torch.cuda.empty_cache()


def test_glm52_decode_t1(glm52_layer):
    cfg = synth.workload("glm52_decode_int4_t1")
    x = synth.tokens(cfg, device=DEV)
    compare_forward(glm52_layer, x)
    for s in range(1, 4):  # more single tokens through the same handle
        compare_forward(glm52_layer, synth.tokens(cfg, device=DEV, stream=s))


def test_glm52_verify_t4_shares_experts(glm52_layer):
    cfg = synth.workload("glm52_verify_int4_t4")
    x = synth.tokens(cfg, device=DEV)
    _, ref = compare_forward(glm52_layer, x)
    a, b = set(ref["idx"][0].tolist()), set(ref["idx"][1].tolist())
    assert len(a & b) >= 1, "tokens 0 and 1 share no expert"


def _compare_on_tensor_cores(gl, x):
    """compare_forward on every token, asserting that the forward ran the
    tcgen05 grouped GEMMs (not the CUDA-core grouped kernels)."""
    gl.handle.profile(True)
    compare_forward(gl, x)
    names = gl.handle.profile_read()
    gl.handle.profile(False)
    assert "gateup_tc" in names and "down_tc" in names, sorted(names)


def test_glm52_prefill_t2048_every_token(glm52_layer):
    """Batch-union prefill of 2048 tokens: every token's routing, Q8_0(h)
    codes of all 9 slots and output row against the oracle, on the tensor-core
    path (every one of the 257 experts is active)."""
    cfg = synth.workload("glm52_prefill_int4_t2048")
    x = synth.tokens(cfg, device=DEV)
    _compare_on_tensor_cores(glm52_layer, x)


@pytest.mark.parametrize("bits", [8, 2])
@pytest.mark.parametrize("T", [1, 4, 512])
def test_glm52_sweep_formats(bits, T):
    cfg = synth.workload("glm52_sweep", bits=bits)
    gl = GpuLayer(cfg, max_tokens=T)
    x = synth.tokens(cfg, T=T, device=DEV)
    if T > 8:
        _compare_on_tensor_cores(gl, x)
    else:
        compare_forward(gl, x)
    gl.close()
    torch.cuda.empty_cache()
