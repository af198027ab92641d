"""Python binding of libkvb, the sm_100a KV-bank library (argument marshalling only).

Every function here has the name of the C entry point it calls (include/kvb.h)
and only converts arguments: torch tensors become device pointers, a torch
stream (or None = torch's current stream) becomes a cudaStream_t, a non-OK status
becomes a ``KvbError``.  All computation happens in the library's CUDA kernels;
importing this package fails if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "KvbError", "kvb_config", "kvb_admit_stats", "make_config", "lib", "LIB_PATH", "Bank", "PAGES_PRESET",
    "KVB_BF16", "KVB_F32", "KVB_DENSITYKV", "KVB_FORCINGKV",
    "KVB_ORDER_DISTURBANCE", "KVB_ORDER_SOURCE", "KVB_BASELINES_FIXED", "KVB_BASELINES_REFRESH",
    "KVB_EVICT_THRESHOLD_RATIO", "KVB_EVICT_DENSEST", "KVB_EVICT_THRESHOLD_SOURCE",
    "KVB_BOTTOMK_FRAME", "KVB_BOTTOMK_CALL", "KVB_SIM_PER_LAYER", "KVB_SIM_FIRST_LAYER",
    "KVB_STORE_NATIVE", "KVB_STORE_FP8_E4M3",
    "kvb_workspace_size", "kvb_bank_create", "kvb_bank_destroy", "kvb_admit", "kvb_prune_hybrid",
    "kvb_attend", "kvb_read_stats", "kvb_bank_export", "kvb_bank_import", "kvb_device_status",
    "kvb_status_string", "kvb_launch_count", "kvb_trace_enable", "kvb_trace_read", "kvb_density_workspace_size", "kvb_density", "kvb_density_noalloc", "kvb_segment_cosine",
    "kvb_selftest_timeout", "kvb_admit_begin", "kvb_admit_finish",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvb.so")

KVB_BF16, KVB_F32 = 0, 1
KVB_DENSITYKV, KVB_FORCINGKV = 0, 1
KVB_ORDER_DISTURBANCE, KVB_ORDER_SOURCE = 0, 1
KVB_BASELINES_FIXED, KVB_BASELINES_REFRESH = 0, 1
KVB_EVICT_THRESHOLD_RATIO, KVB_EVICT_DENSEST, KVB_EVICT_THRESHOLD_SOURCE = 0, 1, 2
KVB_BOTTOMK_FRAME, KVB_BOTTOMK_CALL = 0, 1
KVB_SIM_PER_LAYER, KVB_SIM_FIRST_LAYER = 0, 1
KVB_STORE_NATIVE, KVB_STORE_FP8_E4M3 = 0, 1

# The Soft-Riesz parameters the DensityKV pages select (§4 parameter sensitivity,
# App. E parameter sweeps: width sigma = 8, decay p = 2, regulariser eps fixed
# at 1) in this library's form phi = (||a - b||^2 / h + eps)^(-s/2): h = sigma^2.
# make_config(**PAGES_PRESET) uses them instead of the defaults (h = d, eps 1e-3).
PAGES_PRESET = dict(dist_scale=64.0, eps=1.0, s=2.0)

STATUS = {0: "KVB_OK", 1: "KVB_E_INVAL", 2: "KVB_E_WORKSPACE", 3: "KVB_E_CUDA", 4: "KVB_E_DEVICE_TIMEOUT",
          5: "KVB_E_DEVICE_BOUNDS", 6: "KVB_E_STATE", 7: "KVB_E_UNSUPPORTED"}


class KvbError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({kvb_status_string(status)})")


class kvb_config(ctypes.Structure):
    _fields_ = [
        ("method", ctypes.c_int), ("dtype", ctypes.c_int),
        ("layers", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("capacity", ctypes.c_int32), ("max_candidates", ctypes.c_int32),
        ("tau", ctypes.c_float), ("eps", ctypes.c_float), ("s", ctypes.c_float), ("dist_scale", ctypes.c_float),
        ("sync_heads", ctypes.c_int32),
        ("frame_h", ctypes.c_int32), ("frame_w", ctypes.c_int32), ("seg_h", ctypes.c_int32),
        ("seg_w", ctypes.c_int32), ("hist_frames", ctypes.c_int32), ("max_new_frames", ctypes.c_int32),
        ("retention", ctypes.c_float), ("max_queries", ctypes.c_int32),
        ("cand_order", ctypes.c_int32), ("baselines", ctypes.c_int32), ("evict_order", ctypes.c_int32),
        ("bottomk_scope", ctypes.c_int32), ("sim_source", ctypes.c_int32), ("storage", ctypes.c_int32),
    ]


class kvb_admit_stats(ctypes.Structure):
    _fields_ = [("admitted", ctypes.c_int32), ("feasible", ctypes.c_int32), ("mandatory", ctypes.c_int32),
                ("capacity_evicted", ctypes.c_int32), ("size", ctypes.c_int32), ("moved", ctypes.c_int32),
                ("near_ties", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def make_config(**kw) -> kvb_config:
    """kvb_config with the pages' defaults (tau 2, eps 1e-3, s 2, synchronised heads)."""
    c = kvb_config()
    defaults = dict(method=KVB_DENSITYKV, dtype=KVB_BF16, layers=1, heads=12, head_dim=128, capacity=9360,
                    max_candidates=4680, tau=2.0, eps=1e-3, s=2.0, dist_scale=0.0, sync_heads=1,
                    frame_h=0, frame_w=0, seg_h=4, seg_w=4, hist_frames=21, max_new_frames=3,
                    retention=0.7, max_queries=4680, cand_order=KVB_ORDER_DISTURBANCE,
                    baselines=KVB_BASELINES_FIXED, evict_order=KVB_EVICT_THRESHOLD_RATIO,
                    bottomk_scope=KVB_BOTTOMK_FRAME, sim_source=KVB_SIM_PER_LAYER, storage=KVB_STORE_NATIVE)
    defaults.update(kw)
    for k, v in defaults.items():
        setattr(c, k, v)
    return c


class kvb_trace_record(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("ms", ctypes.c_float), ("device", ctypes.c_int32)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_compression_post_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i32, _f, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "kvb_workspace_size": (_sz, [ctypes.POINTER(kvb_config)]),
    "kvb_bank_create": (ctypes.c_int, [ctypes.POINTER(kvb_config), _vp, _sz, _vp, ctypes.POINTER(_vp)]),
    "kvb_bank_destroy": (ctypes.c_int, [_vp]),
    "kvb_admit": (ctypes.c_int, [_vp, _i32, _vp, _vp, _vp, _i32, _vp]),
    "kvb_prune_hybrid": (ctypes.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp]),
    "kvb_attend": (ctypes.c_int, [_vp, _i32, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp]),
    "kvb_read_stats": (ctypes.c_int, [_vp, _i32, ctypes.POINTER(kvb_admit_stats), _vp]),
    "kvb_bank_export": (ctypes.c_int, [_vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_i32), _vp]),
    "kvb_bank_import": (ctypes.c_int, [_vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp]),
    "kvb_device_status": (ctypes.c_int, [_vp, _vp]),
    "kvb_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvb_launch_count": (ctypes.c_ulonglong, []),
    "kvb_trace_enable": (ctypes.c_int, [_i32]),
    "kvb_trace_read": (ctypes.c_int, [ctypes.POINTER(kvb_trace_record), _i32, ctypes.POINTER(_i32)]),
    "kvb_density_workspace_size": (_sz, [_i32, _i32, _i32, _i32, ctypes.c_int]),
    "kvb_density": (ctypes.c_int, [_vp, _i32, _vp, _i32, _i32, _i32, ctypes.c_int, _f, _f, _f, _i32, _vp, _vp,
                                   _sz, _vp]),
    "kvb_density_noalloc": (ctypes.c_int, [_vp, _i32, _vp, _i32, _i32, _i32, ctypes.c_int, _f, _f, _f, _i32, _vp,
                                           _vp, _vp]),
    "kvb_segment_cosine": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_int, _vp,
                                          _vp]),
    "kvb_selftest_timeout": (ctypes.c_int, [_vp, _vp, ctypes.c_int64, _vp]),
    "kvb_admit_begin": (ctypes.c_int, [_vp, _i32, _vp, _vp, _vp, _i32, _vp, _vp]),
    "kvb_admit_finish": (ctypes.c_int, [_vp, _i32, _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str) -> None:
    if st != 0:
        raise KvbError(st, where)


def kvb_launch_count() -> int:
    return int(lib.kvb_launch_count())


def kvb_trace_enable(enable: bool) -> None:
    _check(lib.kvb_trace_enable(1 if enable else 0), "kvb_trace_enable")


def kvb_trace_read(max_records: int = 65536) -> list:
    """[(kernel name, device ms), ...] of the launches traced since the last read,
    in launch order (waits for their events)."""
    buf = (kvb_trace_record * max_records)()
    n = _i32(0)
    _check(lib.kvb_trace_read(buf, max_records, ctypes.byref(n)), "kvb_trace_read")
    return [(buf[i].kernel.decode(), float(buf[i].ms)) for i in range(min(n.value, max_records))]


def kvb_status_string(status: int) -> str:
    return lib.kvb_status_string(status).decode()


def kvb_workspace_size(cfg: kvb_config) -> int:
    return lib.kvb_workspace_size(ctypes.byref(cfg))


def kvb_bank_create(cfg: kvb_config, workspace, workspace_bytes: int, stream=None) -> int:
    out = _vp()
    _check(lib.kvb_bank_create(ctypes.byref(cfg), _ptr(workspace), workspace_bytes, _stream(stream),
                               ctypes.byref(out)), "kvb_bank_create")
    return out.value


def kvb_bank_destroy(bank: int) -> None:
    _check(lib.kvb_bank_destroy(bank), "kvb_bank_destroy")


def kvb_admit(bank: int, layer: int, candK, candV, cand_ids, N: int, stream=None) -> None:
    _check(lib.kvb_admit(bank, layer, _ptr(candK), _ptr(candV), _ptr(cand_ids), N, _stream(stream)), "kvb_admit")


def kvb_admit_begin(bank: int, layer: int, candK, candV, cand_ids, N: int, prefix_out, stream=None) -> None:
    _check(lib.kvb_admit_begin(bank, layer, _ptr(candK), _ptr(candV), _ptr(cand_ids), N, _ptr(prefix_out),
                               _stream(stream)), "kvb_admit_begin")


def kvb_admit_finish(bank: int, layer: int, prefix_bound=None, stream=None) -> None:
    _check(lib.kvb_admit_finish(bank, layer, _ptr(prefix_bound), _stream(stream)), "kvb_admit_finish")


def kvb_prune_hybrid(bank: int, layer: int, head_is_static, newK, newV, nextK, new_ids, n_frames: int,
                     stream=None) -> None:
    """head_is_static: host bytes / bytearray / numpy uint8 array of length H."""
    import numpy as np
    if isinstance(head_is_static, (bytes, bytearray)):
        arr = np.frombuffer(bytes(head_is_static), dtype=np.uint8).copy()
    else:
        arr = np.ascontiguousarray(np.asarray(head_is_static, dtype=np.uint8))
    _check(lib.kvb_prune_hybrid(bank, layer, arr.ctypes.data, _ptr(newK), _ptr(newV), _ptr(nextK),
                                _ptr(new_ids), n_frames, _stream(stream)), "kvb_prune_hybrid")


def kvb_attend(bank: int, layer: int, Q, Nq: int, sinkK, sinkV, Ls: int, winK, winV, Lw: int, O, lse=None,
               stream=None) -> None:
    _check(lib.kvb_attend(bank, layer, _ptr(Q), Nq, _ptr(sinkK), _ptr(sinkV), Ls, _ptr(winK), _ptr(winV), Lw,
                          _ptr(O), _ptr(lse), _stream(stream)), "kvb_attend")


def kvb_read_stats(bank: int, layer: int, heads: int, stream=None):
    arr = (kvb_admit_stats * heads)()
    _check(lib.kvb_read_stats(bank, layer, arr, _stream(stream)), "kvb_read_stats")
    return [dict(admitted=a.admitted, feasible=a.feasible, mandatory=a.mandatory,
                 capacity_evicted=a.capacity_evicted, size=a.size, moved=a.moved, near_ties=a.near_ties)
            for a in arr]


def kvb_bank_export(bank: int, layer: int, head: int, ids, rho, rho0, K, V, stream=None) -> int:
    n = _i32()
    _check(lib.kvb_bank_export(bank, layer, head, _ptr(ids), _ptr(rho), _ptr(rho0), _ptr(K), _ptr(V),
                               ctypes.byref(n), _stream(stream)), "kvb_bank_export")
    return n.value


def kvb_bank_import(bank: int, layer: int, head: int, ids, rho, rho0, K, V, size: int, stream=None) -> None:
    _check(lib.kvb_bank_import(bank, layer, head, _ptr(ids), _ptr(rho), _ptr(rho0), _ptr(K), _ptr(V), size,
                               _stream(stream)), "kvb_bank_import")


def kvb_device_status(bank: int, stream=None) -> int:
    return lib.kvb_device_status(bank, _stream(stream))


def kvb_density_workspace_size(heads: int, n_rows: int, n_cols: int, head_dim: int, dtype: int) -> int:
    return lib.kvb_density_workspace_size(heads, n_rows, n_cols, head_dim, dtype)


def kvb_density(rows, n_rows: int, cols, n_cols: int, heads: int, head_dim: int, dtype: int, dist_scale: float,
                eps: float, s: float, exclude_diagonal: int, out, workspace, workspace_bytes: int,
                stream=None) -> None:
    _check(lib.kvb_density(_ptr(rows), n_rows, _ptr(cols), n_cols, heads, head_dim, dtype, dist_scale, eps, s,
                           exclude_diagonal, _ptr(out), _ptr(workspace), workspace_bytes, _stream(stream)),
           "kvb_density")


def kvb_selftest_timeout(status, out, timeout_ns: int, stream=None) -> None:
    """Run the library's bounded mbarrier wait to expiry (see kvb.h): status is a
    device int32 word, out a device int64[4]."""
    _check(lib.kvb_selftest_timeout(_ptr(status), _ptr(out), int(timeout_ns), _stream(stream)), "kvb_selftest_timeout")


def kvb_density_noalloc(rows, n_rows: int, cols, n_cols: int, heads: int, head_dim: int, dtype: int,
                        dist_scale: float, eps: float, s: float, exclude_diagonal: int, out, status_out=None,
                        stream=None) -> None:
    """kvb_density without a workspace (scratch in a fixed device array of the library)."""
    _check(lib.kvb_density_noalloc(_ptr(rows), n_rows, _ptr(cols), n_cols, heads, head_dim, dtype, dist_scale, eps,
                                   s, exclude_diagonal, _ptr(out), _ptr(status_out), _stream(stream)),
           "kvb_density_noalloc")


def kvb_segment_cosine(K, nextK, heads: int, n_frames: int, frame_h: int, frame_w: int, seg_h: int, seg_w: int,
                       head_dim: int, dtype: int, sim, stream=None) -> None:
    _check(lib.kvb_segment_cosine(_ptr(K), _ptr(nextK), heads, n_frames, frame_h, frame_w, seg_h, seg_w, head_dim,
                                  dtype, _ptr(sim), _stream(stream)), "kvb_segment_cosine")


class Bank:
    """A kvb bank whose workspace is a torch uint8 tensor on the current device.

    Marshalling only: every method calls the C entry point of the same name."""

    def __init__(self, cfg: kvb_config, stream=None):
        import torch
        self.cfg = cfg
        self.nbytes = kvb_workspace_size(cfg)
        if self.nbytes == 0:
            raise KvbError(1, "kvb_workspace_size")
        self._buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device="cuda")
        self.ws = (self._buf.data_ptr() + 255) & ~255
        self.handle = kvb_bank_create(cfg, self.ws, self.nbytes, stream)

    def close(self):
        if getattr(self, "handle", None):
            kvb_bank_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def admit(self, layer, candK, candV, cand_ids, stream=None):
        kvb_admit(self.handle, layer, candK, candV, cand_ids, cand_ids.shape[0], stream)

    def admit_begin(self, layer, candK, candV, cand_ids, prefix_out, stream=None):
        kvb_admit_begin(self.handle, layer, candK, candV, cand_ids, cand_ids.shape[0], prefix_out, stream)
        # the library reads the candidates again in kvb_admit_finish: keep them alive
        self._pending = (candK, candV, cand_ids)

    def admit_finish(self, layer, prefix_bound=None, stream=None):
        kvb_admit_finish(self.handle, layer, prefix_bound, stream)
        self._pending = None

    def prune_hybrid(self, layer, head_is_static, newK, newV, nextK, new_ids, n_frames, stream=None):
        kvb_prune_hybrid(self.handle, layer, head_is_static, newK, newV, nextK, new_ids, n_frames, stream)

    def attend(self, layer, Q, sinkK, sinkV, winK, winV, O, lse=None, stream=None):
        kvb_attend(self.handle, layer, Q, Q.shape[1], sinkK, sinkV, sinkK.shape[1], winK, winV, winK.shape[1],
                   O, lse, stream)

    def stats(self, layer, stream=None):
        return kvb_read_stats(self.handle, layer, self.cfg.heads, stream)

    def status(self, stream=None) -> int:
        return kvb_device_status(self.handle, stream)

    def export(self, layer, head, stream=None):
        """(ids, rho, rho0, K, V) torch tensors of one (layer, head) bank or history."""
        import torch
        cap = self.cfg.capacity if self.cfg.method == KVB_DENSITYKV else \
            self.cfg.hist_frames * self.cfg.frame_h * self.cfg.frame_w
        dt = torch.bfloat16 if self.cfg.dtype == KVB_BF16 else torch.float32
        ids = torch.empty(cap, dtype=torch.int32, device="cuda")
        rho = torch.zeros(cap, dtype=torch.float32, device="cuda")
        rho0 = torch.zeros(cap, dtype=torch.float32, device="cuda")
        K = torch.empty(cap, self.cfg.head_dim, dtype=dt, device="cuda")
        V = torch.empty(cap, self.cfg.head_dim, dtype=dt, device="cuda")
        n = kvb_bank_export(self.handle, layer, head, ids, rho, rho0, K, V, stream)
        return ids[:n], rho[:n], rho0[:n], K[:n], V[:n]

    def import_(self, layer, head, ids, rho, rho0, K, V, stream=None):
        kvb_bank_import(self.handle, layer, head, ids, rho, rho0, K, V, int(ids.shape[0]), stream)
