"""The C-ABI library loads and exports every entry point include/coli_moe.h
declares; host-side argument checks work without a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

import quantized_expert_ffn_noaux_b200 as qe
from quantized_expert_ffn_noaux_b200 import build as qbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "coli_moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b(coli_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    return qe.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("coli_moe_create", "coli_router", "coli_quant_q8", "coli_moe_forward",
                 "coli_moe_destroy", "coli_quant_weights", "coli_moe_forward_host"):
        assert need in names


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert L.coli_abi_version() == 2


def test_status_strings(L):
    assert L.coli_status_str(0) == b"COLI_OK"
    assert L.coli_status_str(1) == b"COLI_EINVAL"


def _cfg(**kw):
    c = dict(hidden=256, inter=128, n_routed=8, n_shared=1, top_k=2, n_group=1, topk_group=1,
             routed_scaling_factor=2.5, wfmt=4, max_tokens=4)
    c.update(kw)
    return qe._Config(c["hidden"], c["inter"], c["n_routed"], c["n_shared"], c["top_k"],
                      c["n_group"], c["topk_group"], c["routed_scaling_factor"], c["wfmt"],
                      c["max_tokens"], c.get("expert_top_p", 0.0))


@pytest.mark.parametrize("bad", [dict(hidden=250), dict(inter=0), dict(wfmt=3),
                                 dict(n_group=3), dict(topk_group=2), dict(top_k=9),
                                 dict(top_k=0), dict(max_tokens=0), dict(n_shared=5),
                                 dict(wfmt=2, hidden=288), dict(expert_top_p=float("nan")),
                                 dict(n_routed=0, top_k=1), dict(n_routed=0, top_k=0, n_shared=0)])
def test_invalid_configs_are_rejected_on_the_host(L, bad):
    c = _cfg(**bad)
    assert L.coli_moe_workspace_bytes(ctypes.byref(c)) == 0
    h = ctypes.c_void_p(1)
    fake = ctypes.c_void_p(4096)
    st = L.coli_moe_create(ctypes.byref(c), fake, fake, fake, ctypes.byref(h))
    assert st == qe.COLI_EINVAL and not h.value
    assert L.coli_last_error()


def test_workspace_size_grows_with_tokens(L):
    a = L.coli_moe_workspace_bytes(ctypes.byref(_cfg(max_tokens=1)))
    b = L.coli_moe_workspace_bytes(ctypes.byref(_cfg(max_tokens=64)))
    assert 0 < a < b


def test_argument_errors_need_no_device(L):
    fake = ctypes.c_void_p(4096)
    # len not a multiple of 32
    assert L.coli_quant_q8(fake, 1, 33, fake, fake, None) == qe.COLI_EINVAL
    # misaligned pointer
    assert L.coli_quant_q8(ctypes.c_void_p(4100), 1, 32, fake, fake, None) == qe.COLI_EINVAL
    assert L.coli_quant_weights(fake, 1, 32, 5, fake, fake, None) == qe.COLI_EINVAL
    assert L.coli_quant_weights(fake, 1, 32, 2, fake, fake, None) == qe.COLI_EINVAL  # K % 64
    assert L.coli_router(None, fake, 1, fake, fake, None) == qe.COLI_EINVAL
    assert L.coli_moe_forward(None, fake, 1, fake, None) == qe.COLI_EINVAL
    assert L.coli_dbg_block_sums(fake, 4, 1, 31, fake, 1, fake, None) == qe.COLI_EINVAL
    assert L.coli_dbg_set_wait_limit(None, 100, None) == qe.COLI_EINVAL
    L.coli_moe_destroy(None)


def test_injected_allocation_failure(L, monkeypatch):
    monkeypatch.setenv("COLI_FAULT", "alloc")
    c = _cfg()
    experts = (qe._Expert * 9)()
    for i in range(9):
        for m in ("gate", "up", "down"):
            setattr(experts[i], m, qe._QMat(4096, 8192))
    h = ctypes.c_void_p()
    st = L.coli_moe_create(ctypes.byref(c), ctypes.c_void_p(4096), ctypes.c_void_p(4096),
                           experts, ctypes.byref(h))
    assert st == qe.COLI_ENOMEM and not h.value
    assert b"COLI_FAULT" in L.coli_last_error()
