"""B200 (sm_100a) quantised Mixture-of-Experts layer: thin Python binding.

Every function here marshals arguments into the C ABI of ``libcoli_moe.so``
(declared in ``include/coli_moe.h``) and nothing else: every step of the
layer runs in the library's CUDA kernels.  torch is used only to hold device
memory and to name the current stream.  If the library is missing or fails to
load, importing the binding's functions raises immediately; there is no
fallback.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcoli_moe.so")

COLI_OK, COLI_EINVAL, COLI_ENOMEM, COLI_ECUDA, COLI_EUNSUPPORTED, COLI_ETIMEOUT = range(6)
WFMT = {8: 8, 4: 4, 2: 2}


class ColiError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (_status_name(status), msg))
        self.status = status


def _status_name(s):
    return ["COLI_OK", "COLI_EINVAL", "COLI_ENOMEM", "COLI_ECUDA", "COLI_EUNSUPPORTED",
            "COLI_ETIMEOUT"][s] if 0 <= s < 6 else "COLI_%d" % s


class _QMat(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class _Expert(ctypes.Structure):
    _fields_ = [("gate", _QMat), ("up", _QMat), ("down", _QMat)]


class _Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_routed", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("top_k", ctypes.c_int), ("n_group", ctypes.c_int),
                ("topk_group", ctypes.c_int), ("routed_scaling_factor", ctypes.c_float),
                ("wfmt", ctypes.c_int), ("max_tokens", ctypes.c_int),
                ("expert_top_p", ctypes.c_float)]


class _KTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int), ("ms", ctypes.c_double)]


_lib = None


def lib():
    """Load the CUDA library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libcoli_moe.so is not built (run python -m "
                          "quantized_expert_ffn_noaux_b200.build): %s" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, ci, cf = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    sigs = {
        "coli_status_str": ([ci], ctypes.c_char_p),
        "coli_last_error": ([], ctypes.c_char_p),
        "coli_abi_version": ([], ci),
        "coli_launch_count": ([], ctypes.c_uint64),
        "coli_quant_q8": ([vp, i64, i64, vp, vp, vp], ci),
        "coli_quant_weights": ([vp, i64, i64, ci, vp, vp, vp], ci),
        "coli_requant_fp8": ([vp, vp, i64, i64, i64, ci, vp, vp, vp], ci),
        "coli_moe_create": ([vp, vp, vp, vp, ctypes.POINTER(vp)], ci),
        "coli_router": ([vp, vp, ci, vp, vp, vp], ci),
        "coli_moe_forward": ([vp, vp, ci, vp, vp], ci),
        "coli_moe_forward_host": ([vp, vp, ci, vp, vp], ci),
        "coli_moe_set_experts": ([vp, ci, ci, ci], ci),
        "coli_moe_forward_partial": ([vp, vp, ci, vp, vp], ci),
        "coli_combine_partials": ([vp, ci, i64, vp, vp], ci),
        "coli_moe_destroy": ([vp], None),
        "coli_moe_workspace_bytes": ([vp], ctypes.c_size_t),
        "coli_moe_profile": ([vp, ci], ci),
        "coli_moe_profile_read": ([vp, vp, ci, ctypes.POINTER(ci)], ci),
        "coli_dbg_block_sums": ([vp, ci, i64, i64, vp, ci, vp, vp], ci),
        "coli_dbg_last_forward": ([vp, ci, vp, vp, vp, vp, vp], ci),
        "coli_dbg_wait_probe": ([vp, vp], ci),
        "coli_dbg_set_wait_limit": ([vp, ctypes.c_longlong, vp], ci),
        "coli_moe_device_status": ([vp, vp], ci),
        "coli_router_static": ([vp, vp, vp, vp, ci, vp, vp, vp], ci),
    }
    for name, (args, res) in sigs.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(status):
    if status != COLI_OK:
        raise ColiError(status, lib().coli_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def launch_count():
    return int(lib().coli_launch_count())


def row_bytes(K, bits):
    return K * bits // 8


# ---------------------------------------------------------------- functions
def quant_q8(x, q=None, d=None, stream=None):
    """Q8_0 of fp32 rows x [rows][len] (device) -> (q int8, d fp32)."""
    rows, n = x.shape
    q = torch.empty((rows, n), dtype=torch.int8, device=x.device) if q is None else q
    d = torch.empty((rows, n // 32), dtype=torch.float32, device=x.device) if d is None else d
    _check(lib().coli_quant_q8(_ptr(x), rows, n, _ptr(q), _ptr(d), _stream(stream)))
    return q, d


def quant_weights(w, bits, codes=None, scales=None, stream=None):
    """Per-row quantisation of fp32 w [rows][K] (device) -> (codes uint8, scales fp32)."""
    rows, K = w.shape
    if codes is None:
        codes = torch.empty((rows, row_bytes(K, bits)), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=w.device)
    _check(lib().coli_quant_weights(_ptr(w), rows, K, bits, _ptr(codes), _ptr(scales),
                                    _stream(stream)))
    return codes, scales


def requant_fp8(w_fp8, block_scale, bits, block=128, codes=None, scales=None, stream=None):
    """FP8 e4m3 codes w_fp8 [rows][K] (uint8, device) with block scales
    [ceil(rows/block)][ceil(K/block)] fp32 -> per-row (codes uint8, scales fp32)."""
    rows, K = w_fp8.shape
    if codes is None:
        codes = torch.empty((rows, row_bytes(K, bits)), dtype=torch.uint8, device=w_fp8.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=w_fp8.device)
    _check(lib().coli_requant_fp8(_ptr(w_fp8), _ptr(block_scale), rows, K, block, bits,
                                  _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def dbg_block_sums(codes, bits, K, xq, stream=None):
    """int32 block sums [T][rows][K/32] of one matrix against T Q8_0 vectors."""
    rows = codes.shape[0]
    T = xq.shape[0]
    S = torch.empty((T, rows, K // 32), dtype=torch.int32, device=codes.device)
    _check(lib().coli_dbg_block_sums(_ptr(codes), bits, rows, K, _ptr(xq), T, _ptr(S),
                                     _stream(stream)))
    return S


def _config(cfg, max_tokens=None):
    return _Config(cfg["hidden"], cfg["inter"], cfg["n_routed"], cfg["n_shared"], cfg["top_k"],
                   cfg["n_group"], cfg["topk_group"], cfg["routed_scaling_factor"], cfg["bits"],
                   cfg.get("max_tokens", 1) if max_tokens is None else max_tokens,
                   cfg.get("expert_top_p", 0.0))


def router_static(cfg, router_w, bias, x, idx=None, w=None, stream=None):
    """coli_router_static: routing without a handle and without any device
    allocation inside the library (T <= 8, n_routed <= 1024)."""
    T = x.shape[0]
    k = cfg["top_k"]
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx is None else idx
    w = torch.empty((T, k), dtype=torch.float32, device=x.device) if w is None else w
    c = _config(cfg, max_tokens=max(T, 1))
    _check(lib().coli_router_static(ctypes.byref(c), _ptr(router_w), _ptr(bias), _ptr(x), T,
                                    _ptr(idx), _ptr(w), _stream(stream)))
    return idx, w


class Expert:
    """Device tensors of one expert: (codes, scales) for gate, up, down."""

    def __init__(self, gate, up, down):
        self.gate, self.up, self.down = gate, up, down

    @staticmethod
    def quantise(gate_w, up_w, down_w, bits, stream=None):
        return Expert(quant_weights(gate_w, bits, stream=stream),
                      quant_weights(up_w, bits, stream=stream),
                      quant_weights(down_w, bits, stream=stream))

    def nbytes(self):
        return sum(int(c.numel()) + 4 * int(s.numel()) for c, s in (self.gate, self.up, self.down))


class MoELayer:
    """Handle of one quantised MoE layer (coli_moe_create).

    cfg keys: hidden, inter, n_routed, n_shared, top_k, n_group, topk_group,
    routed_scaling_factor, bits, max_tokens.  router_w [E][H] and bias [E] are
    fp32 device tensors; experts is a list of E + S Expert (shared last).  The
    handle borrows all of them; this object keeps references so they outlive it.
    A dense layer is n_routed = 0 with top_k = 0 (router_w and bias may be
    None or empty): every token through the shared experts only.
    """

    def __init__(self, cfg, router_w, bias, experts):
        self.cfg = dict(cfg)
        self._keep = (router_w, bias, list(experts))
        c = _Config(cfg["hidden"], cfg["inter"], cfg["n_routed"], cfg["n_shared"], cfg["top_k"],
                    cfg["n_group"], cfg["topk_group"], cfg["routed_scaling_factor"], cfg["bits"],
                    cfg["max_tokens"], cfg.get("expert_top_p", 0.0))
        arr = (_Expert * len(experts))()
        for i, ex in enumerate(experts):
            arr[i] = _Expert(*(_QMat(m[0].data_ptr(), m[1].data_ptr())
                               for m in (ex.gate, ex.up, ex.down)))
        h = ctypes.c_void_p()
        _check(lib().coli_moe_create(ctypes.byref(c), _ptr(router_w), _ptr(bias), arr,
                                     ctypes.byref(h)))
        self._h = h
        self.device = router_w.device if router_w is not None else experts[0].gate[0].device

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            lib().coli_moe_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self):
        c = self.cfg
        cc = _config(c)
        return int(lib().coli_moe_workspace_bytes(ctypes.byref(cc)))

    def router(self, x, idx=None, w=None, stream=None):
        T = x.shape[0]
        k = self.cfg["top_k"]
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx is None else idx
        w = torch.empty((T, k), dtype=torch.float32, device=x.device) if w is None else w
        _check(lib().coli_router(self._h, _ptr(x), T, _ptr(idx), _ptr(w), _stream(stream)))
        return idx, w

    def forward(self, x, out=None, stream=None):
        T = x.shape[0]
        out = torch.empty_like(x) if out is None else out
        _check(lib().coli_moe_forward(self._h, _ptr(x), T, _ptr(out), _stream(stream)))
        return out

    def set_experts(self, e_lo, e_hi, own_shared=True):
        """Compute only routed experts [e_lo, e_hi) (and the shared ones if own_shared)."""
        _check(lib().coli_moe_set_experts(self._h, int(e_lo), int(e_hi), 1 if own_shared else 0))

    def forward_partial(self, x, out=None, stream=None):
        """fp64 [T][H]: the unrounded sum over this handle's experts' slots."""
        T = x.shape[0]
        if out is None:
            out = torch.empty(x.shape, dtype=torch.float64, device=x.device)
        _check(lib().coli_moe_forward_partial(self._h, _ptr(x), T, _ptr(out), _stream(stream)))
        return out

    def forward_host(self, x_host, out_host, stream=None):
        """x_host, out_host: CPU fp32 tensors (pinned for async copies)."""
        T = x_host.shape[0]
        _check(lib().coli_moe_forward_host(self._h, _ptr(x_host), T, _ptr(out_host),
                                           _stream(stream)))
        return out_host

    def profile(self, enable=True):
        _check(lib().coli_moe_profile(self._h, 1 if enable else 0))

    def profile_read(self):
        arr = (_KTime * 32)()
        n = ctypes.c_int()
        _check(lib().coli_moe_profile_read(self._h, arr, 32, ctypes.byref(n)))
        return {arr[i].name.decode(): (arr[i].launches, arr[i].ms) for i in range(min(n.value, 32))}

    def device_status(self, stream=None):
        """Synchronise and return the device-side status (COLI_OK or COLI_ETIMEOUT)."""
        return int(lib().coli_moe_device_status(self._h, _stream(stream)))

    def dbg_wait_probe(self, stream=None):
        _check(lib().coli_dbg_wait_probe(self._h, _stream(stream)))

    def dbg_set_wait_limit(self, cycles, stream=None):
        """Cycles a kernel wait on progress may last (<= 0: the default)."""
        _check(lib().coli_dbg_set_wait_limit(self._h, int(cycles), _stream(stream)))

    def dbg_last_forward(self, T, stream=None):
        c = self.cfg
        k, S, I = c["top_k"], c["n_shared"], c["inter"]
        dev = self.device
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        hq = torch.empty((T, k + S, I), dtype=torch.int8, device=dev)
        hd = torch.empty((T, k + S, I // 32), dtype=torch.float32, device=dev)
        _check(lib().coli_dbg_last_forward(self._h, T, _ptr(idx), _ptr(w), _ptr(hq), _ptr(hd),
                                           _stream(stream)))
        return idx, w, hq, hd


# ---------------------------------------------------------- expert parallelism
def combine_partials(parts, out=None, stream=None):
    """parts: fp64 [R][...] (device, part order) -> fp32 [...] = fp32(sum in part order)."""
    n = parts[0].numel()
    if out is None:
        out = torch.empty(parts.shape[1:], dtype=torch.float32, device=parts.device)
    _check(lib().coli_combine_partials(_ptr(parts), parts.shape[0], n, _ptr(out), _stream(stream)))
    return out


def expert_range(n_routed, rank, world):
    """Contiguous routed-expert range [lo, hi) of `rank` among `world` GPUs,
    sizes differing by at most one."""
    base, rem = divmod(n_routed, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def gather_partials(part, group=None):
    """All ranks' partial outputs, stacked in rank order ([R][...]), on every rank."""
    dist = torch.distributed
    world = dist.get_world_size(group)
    parts = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(parts, part.contiguous(), group=group)
    return torch.stack(parts)


class ExpertParallelLayer:
    """This GPU's share of an expert-parallel layer: the router (replicated),
    routed experts expert_range(E, rank, world) and, on rank 0, the shared
    experts.  forward() computes the fp64 partial over this rank's (token,
    expert) pairs, all-gathers the partials over `group` (NCCL between GPUs)
    and sums them in rank order on every rank: the same output on every rank,
    deterministic from call to call.

    experts: list of E + S Expert objects; those this rank does not own may be
    None (a placeholder is passed; its weights are never read)."""

    def __init__(self, cfg, router_w, bias, experts, rank, world, group=None):
        self.rank, self.world, self.group = rank, world, group
        self.e_lo, self.e_hi = expert_range(cfg["n_routed"], rank, world)
        E = cfg["n_routed"]
        dev = router_w.device
        ph = None
        full = []
        for e, ex in enumerate(experts):
            owned = (self.e_lo <= e < self.e_hi) if e < E else rank == 0
            if ex is None:
                if owned:
                    raise ValueError("expert %d is owned by rank %d but not given" % (e, rank))
                if ph is None:
                    z = torch.zeros(16, dtype=torch.uint8, device=dev)
                    sc = torch.zeros(4, dtype=torch.float32, device=dev)
                    ph = Expert((z, sc), (z, sc), (z, sc))
                ex = ph
            full.append(ex)
        self.layer = MoELayer(cfg, router_w, bias, full)
        self.layer.set_experts(self.e_lo, self.e_hi, own_shared=(rank == 0))

    def forward(self, x, stream=None):
        part = self.layer.forward_partial(x, stream=stream)
        return combine_partials(gather_partials(part, self.group), stream=stream)

    def close(self):
        self.layer.close()
