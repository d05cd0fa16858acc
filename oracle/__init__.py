"""Test infrastructure: numpy/ctypes front end of the scalar C oracle.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does, and this package imports nothing from it.

Every function below calls the C oracle in ``oracle.c`` (built by
``oracle/build.py``); see that file for the page passages each step follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

QBLK = 32
_LIB = None


class _QMat(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_routed", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("top_k", ctypes.c_int), ("n_group", ctypes.c_int),
                ("topk_group", ctypes.c_int), ("bits", ctypes.c_int),
                ("routed_scaling_factor", ctypes.c_float), ("expert_top_p", ctypes.c_float)]


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        _LIB = ctypes.CDLL(path)
        vp, i64, ci, cf = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        _LIB.oracle_quant_q8.argtypes = [vp, i64, i64, vp, vp]
        _LIB.oracle_quant_q8.restype = None
        _LIB.oracle_quant_weights.argtypes = [vp, i64, i64, ci, vp, vp]
        _LIB.oracle_quant_weights.restype = ci
        _LIB.oracle_unpack_weights.argtypes = [vp, i64, i64, ci, vp]
        _LIB.oracle_unpack_weights.restype = ci
        _LIB.oracle_block_sums.argtypes = [vp, ci, i64, i64, vp, vp]
        _LIB.oracle_block_sums.restype = None
        _LIB.oracle_int_dot.argtypes = [vp, vp, ci, i64, i64, vp, vp, vp]
        _LIB.oracle_int_dot.restype = None
        _LIB.oracle_route.argtypes = [vp, i64, i64, vp, vp, ci, ci, ci, ci, cf, cf, vp, vp, vp, vp,
                                      vp, vp, vp]
        _LIB.oracle_route.restype = ci
        _LIB.oracle_fp8_e4m3.argtypes = [ctypes.c_uint8]
        _LIB.oracle_fp8_e4m3.restype = cf
        _LIB.oracle_dequant_fp8.argtypes = [vp, vp, i64, i64, i64, vp]
        _LIB.oracle_dequant_fp8.restype = None
        _LIB.oracle_requant_fp8.argtypes = [vp, vp, i64, i64, i64, ci, vp, vp]
        _LIB.oracle_requant_fp8.restype = ci
        _LIB.oracle_swiglu.argtypes = [vp, vp, i64, vp]
        _LIB.oracle_swiglu.restype = None
        _LIB.oracle_expert.argtypes = [i64, i64, ci, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        _LIB.oracle_expert.restype = ci
        _LIB.oracle_moe_forward.argtypes = [vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp,
                                            vp, vp, ci]
        _LIB.oracle_moe_forward.restype = ci
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def row_bytes(K, bits):
    return K * bits // 8


def quant_q8(x):
    """Q8_0 of a [rows][len] fp32 array -> (codes int8 [rows][len], d fp32 [rows][len/32])."""
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None]
    rows, n = x.shape
    assert n % QBLK == 0
    q = np.empty((rows, n), np.int8)
    d = np.empty((rows, n // QBLK), np.float32)
    lib().oracle_quant_q8(_p(x), rows, n, _p(q), _p(d))
    return q, d


def quant_weights(w, bits):
    """Per-row quantisation -> (packed codes uint8 [rows][K*bits/8], scales fp32 [rows])."""
    w = _c(w, np.float32)
    rows, K = w.shape
    codes = np.empty((rows, row_bytes(K, bits)), np.uint8)
    scales = np.empty(rows, np.float32)
    rc = lib().oracle_quant_weights(_p(w), rows, K, bits, _p(codes), _p(scales))
    if rc != 0:
        raise ValueError("oracle_quant_weights rejected bits=%d K=%d" % (bits, K))
    return codes, scales


def unpack_weights(codes, K, bits):
    codes = _c(codes, np.uint8)
    rows = codes.shape[0]
    out = np.empty((rows, K), np.int8)
    rc = lib().oracle_unpack_weights(_p(codes), rows, K, bits, _p(out))
    if rc != 0:
        raise ValueError("bad bits")
    return out


def block_sums(codes, bits, K, xq):
    codes = _c(codes, np.uint8)
    xq = _c(xq, np.int8).reshape(-1)
    rows = codes.shape[0]
    S = np.empty((rows, K // QBLK), np.int32)
    lib().oracle_block_sums(_p(codes), bits, rows, K, _p(xq), _p(S))
    return S


def int_dot(codes, scales, bits, K, xq, xd):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    xq = _c(xq, np.int8).reshape(-1)
    xd = _c(xd, np.float32).reshape(-1)
    rows = codes.shape[0]
    out = np.empty(rows, np.float32)
    lib().oracle_int_dot(_p(codes), _p(scales), bits, rows, K, _p(xq), _p(xd), _p(out))
    return out


def route(x, Wr, bias, top_k, n_group, topk_group, rsf, top_p=0.0):
    """Route tokens -> dict(idx, w, s, c, kmargin, gmargin, pmargin).  top_p in
    (0, 1): adaptive expert top-p (dropped slots idx -1, w 0)."""
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None]
    Wr = _c(Wr, np.float32)
    bias = _c(bias, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    s = np.empty((T, E), np.float64)
    c = np.empty((T, E), np.float64)
    km = np.empty(T, np.float64)
    gm = np.empty(T, np.float64)
    pm = np.empty(T, np.float64)
    rc = lib().oracle_route(_p(x), T, H, _p(Wr), _p(bias), E, n_group, topk_group, top_k,
                            float(rsf), float(top_p), _p(idx), _p(w), _p(s), _p(c), _p(km),
                            _p(gm), _p(pm))
    if rc != 0:
        raise ValueError("oracle_route rejected E=%d G=%d gk=%d k=%d" % (E, n_group, topk_group,
                                                                        top_k))
    return dict(idx=idx, w=w, s=s, c=c, kmargin=km, gmargin=gm, pmargin=pm)


def fp8_e4m3(code):
    """Value of one FP8 e4m3 code (fp32; NaN for S.1111.111)."""
    return float(lib().oracle_fp8_e4m3(int(code) & 0xFF))


def dequant_fp8(codes, scale, block=128):
    """FP8 codes [rows][K] (uint8) with block scales [ceil(rows/B)][ceil(K/B)]
    -> fp32 weights [rows][K]."""
    codes = _c(codes, np.uint8)
    scale = _c(scale, np.float32)
    rows, K = codes.shape
    assert scale.shape == (-(-rows // block), -(-K // block))
    out = np.empty((rows, K), np.float32)
    lib().oracle_dequant_fp8(_p(codes), _p(scale), rows, K, block, _p(out))
    return out


def requant_fp8(codes, scale, bits, block=128):
    """The converter step: FP8 + block scales -> per-row (codes, scales)."""
    codes = _c(codes, np.uint8)
    scale = _c(scale, np.float32)
    rows, K = codes.shape
    assert scale.shape == (-(-rows // block), -(-K // block))
    out = np.empty((rows, row_bytes(K, bits)), np.uint8)
    sc = np.empty(rows, np.float32)
    rc = lib().oracle_requant_fp8(_p(codes), _p(scale), rows, K, block, bits, _p(out), _p(sc))
    if rc != 0:
        raise ValueError("oracle_requant_fp8 rc=%d" % rc)
    return out, sc


def swiglu(g, u):
    """SwiGLU of fp32 gate/up outputs -> h fp32 (same shape)."""
    g = _c(g, np.float32).reshape(-1)
    u = _c(u, np.float32).reshape(-1)
    assert g.shape == u.shape
    h = np.empty_like(g)
    lib().oracle_swiglu(_p(g), _p(u), g.size, _p(h))
    return h


class QExpert:
    """One expert's three quantised matrices (host numpy arrays)."""

    def __init__(self, gate, up, down):
        self.gate, self.up, self.down = gate, up, down  # each (codes, scales)

    @staticmethod
    def quantise(gate_w, up_w, down_w, bits):
        return QExpert(quant_weights(gate_w, bits), quant_weights(up_w, bits),
                       quant_weights(down_w, bits))


def _qmat(cs):
    codes, scales = cs
    return _QMat(codes.ctypes.data, scales.ctypes.data)


def expert(H, I, bits, ex, xq, xd, hq_in=None, hd_in=None):
    """One expert on one token's Q8_0 activations -> (e [H], hq [I], hd [I/32])."""
    xq = _c(xq, np.int8).reshape(-1)
    xd = _c(xd, np.float32).reshape(-1)
    hq = np.empty(I, np.int8)
    hd = np.empty(I // QBLK, np.float32)
    e = np.empty(H, np.float32)
    g, u, d = _qmat(ex.gate), _qmat(ex.up), _qmat(ex.down)
    if hq_in is not None:
        hq_in = _c(hq_in, np.int8)
        hd_in = _c(hd_in, np.float32)
    rc = lib().oracle_expert(H, I, bits, ctypes.byref(g), ctypes.byref(u), ctypes.byref(d),
                             _p(xq), _p(xd), _p(hq_in), _p(hd_in), _p(hq), _p(hd), _p(e))
    if rc != 0:
        raise ValueError("oracle_expert rc=%d" % rc)
    return e, hq, hd


class Layer:
    """Host copy of one layer for the oracle.

    cfg: dict with hidden, inter, n_routed, n_shared, top_k, n_group, topk_group,
    routed_scaling_factor, bits.  experts: list of length n_routed + n_shared of
    QExpert or None (None = not needed; shared experts last).
    """

    def __init__(self, cfg, Wr, bias, experts):
        self.cfg = dict(cfg)
        self.Wr = _c(Wr, np.float32)
        self.bias = _c(bias, np.float32)
        self.experts = list(experts)
        assert len(self.experts) == cfg["n_routed"] + cfg["n_shared"]

    def _ccfg(self):
        c = self.cfg
        return _Cfg(c["hidden"], c["inter"], c["n_routed"], c["n_shared"], c["top_k"],
                    c["n_group"], c["topk_group"], c["bits"], c["routed_scaling_factor"],
                    c.get("expert_top_p", 0.0))

    def route(self, x):
        c = self.cfg
        return route(x, self.Wr, self.bias, c["top_k"], c["n_group"], c["topk_group"],
                     c["routed_scaling_factor"], c.get("expert_top_p", 0.0))

    def forward(self, x, idx_in=None, hq_in=None, hd_in=None, nthreads=1):
        """-> dict(out [T][H], idx, w, hq [T][k+S][I], hd [T][k+S][I/32])."""
        c = self.cfg
        x = _c(x, np.float32)
        if x.ndim == 1:
            x = x[None]
        T, H = x.shape
        I, k, S = c["inter"], c["top_k"], c["n_shared"]
        n = c["n_routed"] + S
        mats = (_QMat * (3 * n))()
        keep = []
        for e, ex in enumerate(self.experts):
            if ex is None:
                continue
            for m, cs in enumerate((ex.gate, ex.up, ex.down)):
                codes = _c(cs[0], np.uint8)
                scales = _c(cs[1], np.float32)
                keep += [codes, scales]
                mats[3 * e + m] = _QMat(codes.ctypes.data, scales.ctypes.data)
        out = np.empty((T, H), np.float32)
        idx = np.empty((T, k), np.int32)
        w = np.empty((T, k), np.float32)
        hq = np.empty((T, k + S, I), np.int8)
        hd = np.empty((T, k + S, I // QBLK), np.float32)
        if idx_in is not None:
            idx_in = _c(idx_in, np.int32)
        if hq_in is not None:
            hq_in = _c(hq_in, np.int8)
            hd_in = _c(hd_in, np.float32)
        cc = self._ccfg()
        rc = lib().oracle_moe_forward(ctypes.byref(cc), _p(self.Wr), _p(self.bias), mats, _p(x),
                                      T, _p(idx_in), _p(hq_in), _p(hd_in), _p(idx), _p(w),
                                      _p(hq), _p(hd), _p(out), int(nthreads))
        if rc == -3:
            raise KeyError("oracle_moe_forward: a selected expert was not provided")
        if rc != 0:
            raise ValueError("oracle_moe_forward rc=%d" % rc)
        del keep
        return dict(out=out, idx=idx, w=w, hq=hq, hd=hd)


def n_threads_default():
    return os.cpu_count() or 1
