"""CRISP sparse-prefill attention on B200 (sm_100a): thin Python binding.

Every stage runs in the CUDA kernels of ``libcrisp.so`` behind the C ABI of
``include/crisp.h``; this module only marshals arguments. Tensors are torch
CUDA tensors (torch supplies device memory and streams), passed as raw device
pointers. There is no CPU fallback: if the library is missing, every call
raises.

Entry points (same names as the C ABI): ``route``, ``select``, ``attend``,
``prefill``, ``dense_attention``, plus ``workspace_size``, ``index_dims``,
``device_status`` and the ``Config`` / ``IndexBuffers`` helpers.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

__all__ = [
    "Config", "IndexBuffers", "CrispError", "lib", "library_path", "workspace_size", "index_dims",
    "route", "route_noalloc", "select", "attend", "prefill", "dense_attention", "device_status", "status_string",
    "BF16", "FP32", "ROUTE_AUTO", "ROUTE_VS", "ROUTE_PE", "SYMBOLS",
]

BF16, FP32 = 0, 1
ROUTE_AUTO, ROUTE_VS, ROUTE_PE = -1, 0, 1
STATUS_NAMES = {
    0: "CRISP_OK", 1: "CRISP_ERR_INVALID_ARG", 2: "CRISP_ERR_SHAPE", 3: "CRISP_ERR_DTYPE",
    4: "CRISP_ERR_ALIGN", 5: "CRISP_ERR_WORKSPACE", 6: "CRISP_ERR_UNSUPPORTED", 7: "CRISP_ERR_CUDA",
    8: "CRISP_ERR_CAPACITY", 9: "CRISP_ERR_TIMEOUT", 10: "CRISP_ERR_NONFINITE", 11: "CRISP_ERR_TOO_LARGE",
}
# every function include/crisp.h declares
SYMBOLS = ["crisp_cfg_init", "crisp_workspace_size", "crisp_index_dims", "crisp_route", "crisp_select",
           "crisp_attend", "crisp_prefill", "crisp_dense_attention", "crisp_device_status",
           "crisp_status_string", "crisp_version", "crisp_route_noalloc", "crisp_exp2_selftest",
           "crisp_prefill_batch", "crisp_workspace_size_batch", "crisp_prefill_varlen",
           "crisp_prefill_host", "crisp_workspace_size_host", "crisp_wait_selftest",
           "crisp_diag_select_simt", "crisp_diag_attend_simt"]


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcrisp.so")


class CrispError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32), ("d", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("block", ctypes.c_int32), ("last_q", ctypes.c_int32),
        ("w_sink", ctypes.c_int32), ("w_local", ctypes.c_int32), ("tau_proxy", ctypes.c_float),
        ("alpha", ctypes.c_float), ("gamma", ctypes.c_float), ("sm_scale", ctypes.c_float),
        ("force_route", ctypes.c_int32), ("reserved", ctypes.c_int32), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
    ]


_INDEX_FIELDS = ["route", "c_struct", "p_v", "p_s", "mu", "vs_mask", "v_idx", "s_idx", "nv", "ns",
                 "pe_mask", "pe_count", "pe_cut"]


class _Index(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _INDEX_FIELDS]


_LIB = None


def lib() -> ctypes.CDLL:
    """Load libcrisp.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m long_context_prefill_last_b200.build`")
        L = ctypes.CDLL(path)
        vp, cfgp = ctypes.c_void_p, ctypes.POINTER(_Cfg)
        L.crisp_cfg_init.argtypes = [cfgp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32]
        L.crisp_workspace_size.argtypes = [cfgp, ctypes.POINTER(ctypes.c_size_t)]
        L.crisp_index_dims.argtypes = [cfgp, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
        L.crisp_route.argtypes = [vp, vp, cfgp, vp, vp, vp]
        L.crisp_route_noalloc.argtypes = [vp, vp, cfgp, vp, vp, vp]
        L.crisp_exp2_selftest.argtypes = [vp, vp, vp, vp, ctypes.c_int32, vp]
        L.crisp_wait_selftest.argtypes = [ctypes.c_int64, vp, vp]
        L.crisp_select.argtypes = [vp, vp, cfgp, ctypes.POINTER(_Index), vp]
        L.crisp_attend.argtypes = [vp, vp, vp, vp, cfgp, ctypes.POINTER(_Index), vp]
        L.crisp_prefill.argtypes = [vp, vp, vp, vp, cfgp, vp]
        L.crisp_prefill_batch.argtypes = [vp, vp, vp, vp, cfgp, ctypes.c_int32, vp]
        L.crisp_prefill_host.argtypes = [vp, vp, vp, vp, cfgp, vp, vp]
        L.crisp_workspace_size_host.argtypes = [cfgp, ctypes.POINTER(ctypes.c_size_t)]
        L.crisp_workspace_size_batch.argtypes = [cfgp, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
        L.crisp_prefill_varlen.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                           ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                           cfgp, vp]
        L.crisp_dense_attention.argtypes = [vp, vp, vp, vp, cfgp, vp]
        L.crisp_diag_select_simt.argtypes = [vp, vp, cfgp, ctypes.POINTER(_Index), vp]
        L.crisp_diag_attend_simt.argtypes = [vp, vp, vp, vp, cfgp, ctypes.POINTER(_Index), ctypes.c_int32, vp]
        L.crisp_device_status.argtypes = [cfgp, vp, ctypes.POINTER(ctypes.c_int32)]
        L.crisp_status_string.argtypes = [ctypes.c_int]
        L.crisp_status_string.restype = ctypes.c_char_p
        L.crisp_version.restype = ctypes.c_int32
        for name in SYMBOLS:
            if name not in ("crisp_status_string", "crisp_version"):
                getattr(L, name).restype = ctypes.c_int
        _LIB = L
    return _LIB


def status_string(code: int) -> str:
    return lib().crisp_status_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != 0:
        raise CrispError(code, where)


@dataclasses.dataclass
class Config:
    """Layer shape and knobs (mirrors crisp_cfg; defaults as crisp_cfg_init)."""
    n: int
    h_q: int
    h_kv: int
    d: int = 128
    dtype: int = BF16
    block: int = 128
    last_q: int = 64
    w_sink: int = 128
    w_local: int = 128
    tau_proxy: float = 0.10
    alpha: float = 1.0
    gamma: float = 0.95
    sm_scale: float = 0.0
    force_route: int = ROUTE_AUTO
    workspace: Optional[object] = None     # torch.uint8 CUDA tensor
    reserved: int = 0

    @property
    def n_blocks(self) -> int:
        return self.n // self.block

    @property
    def words(self) -> int:
        return (self.n_blocks + 31) // 32

    def _c(self) -> _Cfg:
        c = _Cfg()
        for f, _ in _Cfg._fields_:
            if f in ("workspace", "workspace_bytes"):
                continue
            setattr(c, f, getattr(self, f))
        if self.workspace is not None:
            c.workspace = self.workspace.data_ptr()
            c.workspace_bytes = self.workspace.numel() * self.workspace.element_size()
        return c

    def allocate_workspace(self, device="cuda", batch: int = 1, max_n: Optional[int] = None, host: bool = False):
        """Device workspace for this shape; `batch` sequences (crisp_prefill_batch),
        sequences up to `max_n` tokens (crisp_prefill_varlen) or a layer in host
        memory (crisp_prefill_host)."""
        import torch
        c = dataclasses.replace(self, n=max_n) if max_n is not None else self
        if host:
            nbytes = workspace_size_host(c)
        else:
            nbytes = workspace_size(c) if batch == 1 else workspace_size_batch(c, batch)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        return self.workspace


def workspace_size(cfg: Config) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().crisp_workspace_size(ctypes.byref(cfg._c()), ctypes.byref(out)), "crisp_workspace_size")
    return out.value


def workspace_size_batch(cfg: Config, batch: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().crisp_workspace_size_batch(ctypes.byref(cfg._c()), int(batch), ctypes.byref(out)),
           "crisp_workspace_size_batch")
    return out.value


def workspace_size_host(cfg: Config) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().crisp_workspace_size_host(ctypes.byref(cfg._c()), ctypes.byref(out)), "crisp_workspace_size_host")
    return out.value


def index_dims(cfg: Config):
    nb, w = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib().crisp_index_dims(ctypes.byref(cfg._c()), ctypes.byref(nb), ctypes.byref(w)), "crisp_index_dims")
    return nb.value, w.value


class IndexBuffers:
    """Device buffers for a crisp_index (torch tensors, allocated once)."""

    def __init__(self, cfg: Config, device="cuda"):
        import torch
        nb, w = index_dims(cfg)
        h = cfg.h_q
        i32, f32, u32 = torch.int32, torch.float32, torch.int32
        self.route = torch.zeros(h, dtype=i32, device=device)
        self.c_struct = torch.zeros(h, dtype=f32, device=device)
        self.p_v = torch.zeros(h, nb, dtype=f32, device=device)
        self.p_s = torch.zeros(h, nb, dtype=f32, device=device)
        self.mu = torch.zeros(h, 2, dtype=f32, device=device)
        self.vs_mask = torch.zeros(h, 2, w, dtype=u32, device=device)
        self.v_idx = torch.zeros(h, nb, dtype=i32, device=device)
        self.s_idx = torch.zeros(h, nb, dtype=i32, device=device)
        self.nv = torch.zeros(h, dtype=i32, device=device)
        self.ns = torch.zeros(h, dtype=i32, device=device)
        self.pe_mask = torch.zeros(h, nb, w, dtype=u32, device=device)
        self.pe_count = torch.zeros(h, dtype=torch.int64, device=device)
        self.pe_cut = torch.zeros(h, dtype=f32, device=device)

    def _c(self) -> _Index:
        ix = _Index()
        for f in _INDEX_FIELDS:
            setattr(ix, f, getattr(self, f).data_ptr())
        return ix


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def route(q, k, cfg: Config, route_out, c_struct_out, stream=None) -> None:
    _check(lib().crisp_route(_ptr(q), _ptr(k), ctypes.byref(cfg._c()), _ptr(route_out), _ptr(c_struct_out),
                             _stream(stream)), "crisp_route")


def route_noalloc(q, k, cfg: Config, route_out, c_struct_out, stream=None) -> None:
    """crisp_route with the library's static scratch array instead of a workspace
    (cfg.workspace is ignored). For callers that cannot give the library device
    memory; concurrent calls race on the shared array. A device-side failure
    shows as route -1 and C_struct NaN on every head."""
    _check(lib().crisp_route_noalloc(_ptr(q), _ptr(k), ctypes.byref(cfg._c()), _ptr(route_out),
                                     _ptr(c_struct_out), _stream(stream)), "crisp_route_noalloc")


def select(q, k, cfg: Config, index: IndexBuffers, stream=None) -> None:
    _check(lib().crisp_select(_ptr(q), _ptr(k), ctypes.byref(cfg._c()), ctypes.byref(index._c()), _stream(stream)),
           "crisp_select")


def attend(q, k, v, out, cfg: Config, index: IndexBuffers, stream=None) -> None:
    _check(lib().crisp_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(cfg._c()),
                              ctypes.byref(index._c()), _stream(stream)), "crisp_attend")


def prefill(q, k, v, out, cfg: Config, stream=None) -> None:
    _check(lib().crisp_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(cfg._c()), _stream(stream)),
           "crisp_prefill")


def prefill_batch(q, k, v, out, cfg: Config, stream=None) -> None:
    """crisp_prefill_batch: q/out [batch, h_q, n, d], k/v [batch, h_kv, n, d]; cfg is one sequence's."""
    _check(lib().crisp_prefill_batch(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(cfg._c()), int(q.shape[0]),
                                     _stream(stream)), "crisp_prefill_batch")


_COPY_STREAMS = {}


def prefill_host(q, k, v, out, cfg: Config, stream=None, copy_stream=None) -> None:
    """crisp_prefill_host: q/out [h_q, n, d] and k/v [h_kv, n, d] in page-locked
    host memory; copies run on `copy_stream` (one per device by default) and
    overlap the kernels on `stream`. Completes with `stream`."""
    import torch
    if copy_stream is None:
        dev = torch.cuda.current_device()
        if dev not in _COPY_STREAMS:
            _COPY_STREAMS[dev] = torch.cuda.Stream(device=dev)
        copy_stream = _COPY_STREAMS[dev]
    _check(lib().crisp_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(cfg._c()), _stream(stream),
                                    _stream(copy_stream)), "crisp_prefill_host")


def prefill_varlen(qs, ks, vs, outs, cfg: Config, stream=None) -> None:
    """crisp_prefill_varlen: per-sequence tensors qs[i] [h_q, n_i, d], ks/vs[i] [h_kv, n_i, d]."""
    cnt = len(qs)
    if not (len(ks) == len(vs) == len(outs) == cnt):
        raise ValueError("q, k, v and out lists differ in length")
    arr = ctypes.c_void_p * cnt
    n = (ctypes.c_int32 * cnt)(*[int(t.shape[1]) for t in qs])
    _check(lib().crisp_prefill_varlen(arr(*[_ptr(t) for t in qs]), arr(*[_ptr(t) for t in ks]),
                                      arr(*[_ptr(t) for t in vs]), arr(*[_ptr(t) for t in outs]), n, cnt,
                                      ctypes.byref(cfg._c()), _stream(stream)), "crisp_prefill_varlen")


def dense_attention(q, k, v, out, cfg: Config, stream=None) -> None:
    _check(lib().crisp_dense_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(cfg._c()),
                                       _stream(stream)), "crisp_dense_attention")


def diag_select_simt(q, k, cfg: Config, index: IndexBuffers, stream=None) -> None:
    """crisp_select with the proxy map on the CUDA-core kernel (a test cross-check)."""
    _check(lib().crisp_diag_select_simt(_ptr(q), _ptr(k), ctypes.byref(cfg._c()), ctypes.byref(index._c()),
                                        _stream(stream)), "crisp_diag_select_simt")


def diag_attend_simt(q, k, v, out, cfg: Config, index: Optional[IndexBuffers], dense: bool = False,
                     stream=None) -> None:
    """crisp_attend (or dense attention) on the CUDA-core kernel (a test cross-check)."""
    ix = ctypes.byref(index._c()) if index is not None else None
    _check(lib().crisp_diag_attend_simt(_ptr(q), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(cfg._c()), ix,
                                        1 if dense else 0, _stream(stream)), "crisp_diag_attend_simt")


def exp2_selftest(x, stream=None):
    """(poly3, poly5, exp2f) of a float32 CUDA tensor, evaluated on the device."""
    import torch
    outs = [torch.empty_like(x) for _ in range(3)]
    _check(lib().crisp_exp2_selftest(_ptr(x), _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), x.numel(),
                                     _stream(stream)), "crisp_exp2_selftest")
    return tuple(outs)


def wait_selftest(limit_cycles: int, status, stream=None) -> None:
    """Run the bounded mbarrier wait against a barrier nothing arrives on;
    `status` (int32[8] CUDA tensor, zeroed) receives CRISP_ERR_TIMEOUT and site 99."""
    _check(lib().crisp_wait_selftest(int(limit_cycles), _ptr(status), _stream(stream)), "crisp_wait_selftest")


def device_status(cfg: Config, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status code."""
    st = ctypes.c_int32(0)
    _check(lib().crisp_device_status(ctypes.byref(cfg._c()), _stream(stream), ctypes.byref(st)),
           "crisp_device_status")
    return st.value


def raise_on_device_status(cfg: Config, stream=None, where: str = "device") -> None:
    code = device_status(cfg, stream)
    if code != 0:
        raise CrispError(code, where)
