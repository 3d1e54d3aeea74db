"""Python binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module converts
torch tensors to pointers and C status codes to exceptions.  PyTorch is used only
for device memory and streams.  Importing works without a GPU (so that the C ABI's
exports can be checked), but the library must be built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_CHECK"}
FMT_TERNARY, FMT_Q2, FMT_Q3 = 0, 1, 2
PATH_AUTO, PATH_DECODE, PATH_PREFILL, PATH_DECODE_FUSED = 0, 1, 2, 3
OUT_F32 = 0x10          # OR into a path: moe_forward writes fp32 y

# every symbol include/moe.h declares
EXPORTS = ["moe_packed_size", "moe_pack_experts", "moe_requantize_q3_to_q2", "moe_workspace_size",
           "moe_workspace_init", "moe_route",
           "moe_forward", "moe_forward_timed", "moe_get_error", "moe_decode_static", "moe_decode_static_get_error",
           "moe_workspace_set_test_stall", "moe_event_record", "moe_status_string", "moe_abi_version",
           "moe_route_fixed", "moe_gather_rows", "moe_combine_pairs", "moe_cache_size", "moe_cache_init",
           "moe_cache_load", "moe_forward_plan"]
# detail codes beside MOE_ERR_TIMEOUT / MOE_ERR_DEVICE_CHECK (high bits: what; low byte: where)
DETAIL = {"WAIT_FULL": 0x100, "WAIT_EMPTY": 0x200, "DRAIN": 0x300, "HEADER": 0x400, "ROUTED_T": 0x500,
          "RANGE": 0x600, "TEST_STALL": 0x700, "LOOP_CAP": 0x800, "FORMAT": 0x900}
FMT_TERNARY_DENSE = 3       # storage form of ternary experts (five codes per byte), see moe.h
STATIC_WS_BYTES = 8 << 20


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} -> {STATUS.get(status, status)}")


class Shape(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32)]


class Routing(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("topk_ids", "topk_w", "counts", "offsets", "perm", "inv_perm")]


class MatrixSrc(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("hi", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m bit_routed_expert_fp32_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        sh = ctypes.POINTER(Shape)
        L.moe_packed_size.argtypes = [sh, vp, ctypes.POINTER(sz)]
        L.moe_pack_experts.argtypes = [sh, vp, i32, i32, ctypes.POINTER(MatrixSrc), vp, sz]
        L.moe_requantize_q3_to_q2.argtypes = [i32, i32, ctypes.POINTER(MatrixSrc), vp, vp]
        L.moe_workspace_size.argtypes = [sh, i32, ctypes.POINTER(sz)]
        L.moe_forward_plan.argtypes = [sh, i32, i32, vp]
        L.moe_workspace_init.argtypes = [vp, sz, vp]
        L.moe_route.argtypes = [sh, i32, vp, vp, vp, ctypes.POINTER(Routing), vp, sz, vp]
        L.moe_forward.argtypes = [sh, i32, vp, vp, ctypes.POINTER(Routing), vp, ctypes.c_int, vp, sz, vp]
        L.moe_forward_timed.argtypes = [sh, i32, vp, vp, ctypes.POINTER(Routing), vp, ctypes.c_int, vp, sz, vp,
                                        ctypes.POINTER(vp), i32]
        L.moe_get_error.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_decode_static.argtypes = [sh, i32, vp, vp, vp, vp, ctypes.POINTER(Routing), vp, vp]
        L.moe_decode_static_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_workspace_set_test_stall.argtypes = [vp, sz, ctypes.c_uint32, vp]
        L.moe_route_fixed.argtypes = [sh, i32, vp, vp, vp, ctypes.POINTER(Routing), vp, sz, vp]
        L.moe_gather_rows.argtypes = [i32, i32, vp, i32, vp, i32, vp, vp, sz, vp]
        L.moe_combine_pairs.argtypes = [i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.moe_cache_size.argtypes = [sh, vp, i32, ctypes.POINTER(sz)]
        L.moe_cache_init.argtypes = [sh, vp, i32, vp, sz, vp]
        L.moe_cache_load.argtypes = [sh, vp, i32, vp, sz, vp, vp, i32, vp]
        L.moe_event_record.argtypes = [vp, vp]
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_abi_version.restype = i32
        for n in EXPORTS:
            if n not in ("moe_status_string", "moe_abi_version"):
                getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


def _shape(cfg) -> Shape:
    return Shape(cfg.H, cfg.I, cfg.E, cfg.k, cfg.S)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ---- packing (host) -----------------------------------------------------------

def moe_packed_size(cfg, fmt: np.ndarray) -> int:
    fmt = np.ascontiguousarray(fmt, dtype=np.uint8)
    out = ctypes.c_size_t(0)
    _check("moe_packed_size", lib().moe_packed_size(ctypes.byref(_shape(cfg)), fmt.ctypes.data, ctypes.byref(out)))
    return out.value


def moe_pack_experts(cfg, fmt: np.ndarray, first: int, mats: list, dst: np.ndarray) -> None:
    """Pack experts first..first+len(mats)-1 into the host buffer dst (uint8).
    mats[i] = {'gate','up','down'} -> (codes, hi, scales) in the interchange form."""
    fmt = np.ascontiguousarray(fmt, dtype=np.uint8)
    src = (MatrixSrc * (3 * len(mats)))()
    keep = []
    for i, m in enumerate(mats):
        for q, name in enumerate(("gate", "up", "down")):
            c, h, s = m[name]
            c = np.ascontiguousarray(c, dtype=np.uint8)
            s = np.ascontiguousarray(s, dtype=np.uint16)
            h = None if h is None else np.ascontiguousarray(h, dtype=np.uint8)
            keep += [c, s, h]
            src[3 * i + q] = MatrixSrc(c.ctypes.data, None if h is None else h.ctypes.data, s.ctypes.data)
    _check("moe_pack_experts", lib().moe_pack_experts(ctypes.byref(_shape(cfg)), fmt.ctypes.data, first, len(mats),
                                                       src, dst.ctypes.data, dst.nbytes))


def pack_layer(cfg, fmt: np.ndarray, expert_fn) -> np.ndarray:
    """Host packed buffer of all E+S experts; expert_fn(e) returns its matrices."""
    buf = np.zeros(moe_packed_size(cfg, fmt), dtype=np.uint8)
    for e in range(cfg.E + cfg.S):
        moe_pack_experts(cfg, fmt, e, [expert_fn(e)], buf)
    return buf


def moe_requantize_q3_to_q2(codes: np.ndarray, hi: np.ndarray, scales: np.ndarray):
    """2-bit copy of one 3-bit matrix (interchange form): codes [rows][K/4], hi
    [rows][K/8], fp16 scales [rows][K/64] -> (codes, None, scales) of c >> 1, 2 s."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    h = np.ascontiguousarray(hi, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint16)
    rows, K = c.shape[0], 4 * c.shape[1]
    if h.shape != (rows, K // 8) or s.shape != (rows, K // 64):
        raise ValueError("moe_requantize_q3_to_q2: codes, hi and scales disagree on the matrix shape")
    oc = np.empty_like(c)
    osc = np.empty_like(s)
    src = MatrixSrc(c.ctypes.data, h.ctypes.data, s.ctypes.data)
    _check("moe_requantize_q3_to_q2",
           lib().moe_requantize_q3_to_q2(rows, K, ctypes.byref(src), oc.ctypes.data, osc.ctypes.data))
    return oc, None, osc


def fast_copy(fmt: np.ndarray, expert_fn):
    """Formats and expert source of the fast-mode copy of a layer: every 3-bit expert
    (routed or shared) becomes its 2-bit copy (moe_requantize_q3_to_q2), the others
    are unchanged.  Pack the result with pack_layer / moe_pack_experts into a second
    buffer and pass that buffer, instead of the layer's own, to the calls that should
    read the 2-bit copy."""
    fmt = np.ascontiguousarray(fmt, dtype=np.uint8)
    fast = np.where(fmt == FMT_Q3, FMT_Q2, fmt).astype(np.uint8)

    def fn(e):
        m = expert_fn(e)
        if fmt[e] != FMT_Q3:
            return m
        return {name: moe_requantize_q3_to_q2(*m[name]) for name in ("gate", "up", "down")}

    return fast, fn


# ---- device calls -----------------------------------------------------------------

def moe_workspace_size(cfg, max_tokens: int) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(_shape(cfg)), max_tokens, ctypes.byref(out)))
    return out.value


def moe_forward_plan(cfg, T: int, path=PATH_AUTO) -> dict:
    """The library's plan for moe_route + moe_forward (host-only): which kernels run
    ("decode", "prefill" or "fused"), how many launches, and the K parts of the separate
    decode passes."""
    out = np.zeros(4, np.int32)
    _check("moe_forward_plan", lib().moe_forward_plan(ctypes.byref(_shape(cfg)), T, path, out.ctypes.data))
    kind = {PATH_DECODE: "decode", PATH_PREFILL: "prefill", PATH_DECODE_FUSED: "fused"}[int(out[0])]
    return {"path": kind, "launches": int(out[1]), "kparts_gu": int(out[2]), "kparts_dn": int(out[3])}


def moe_workspace_init(ws, stream=None) -> None:
    _check("moe_workspace_init", lib().moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def routing_struct(rt: dict) -> Routing:
    return Routing(*(rt[n].data_ptr() for n in ("topk_ids", "topk_w", "counts", "offsets", "perm", "inv_perm")))


def alloc_routing(cfg, T: int, device="cuda") -> dict:
    import torch
    i32 = dict(dtype=torch.int32, device=device)
    return {"topk_ids": torch.empty((T, cfg.k), **i32), "topk_w": torch.empty((T, cfg.k), dtype=torch.float32,
                                                                                device=device),
            "counts": torch.empty(cfg.E, **i32), "offsets": torch.empty(cfg.E + 1, **i32),
            "perm": torch.empty(max(T * cfg.k, 1), **i32), "inv_perm": torch.empty(max(T * cfg.k, 1), **i32)}


def moe_route(cfg, T, x, router_w, router_b, rt: dict, ws, stream=None) -> None:
    r = routing_struct(rt)
    _check("moe_route", lib().moe_route(ctypes.byref(_shape(cfg)), T, _ptr(x), _ptr(router_w), _ptr(router_b),
                                         ctypes.byref(r), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_forward(cfg, T, packed, x, rt: dict, y, path=PATH_AUTO, ws=None, stream=None, events=None) -> None:
    r = routing_struct(rt)
    if events is None:
        st = lib().moe_forward(ctypes.byref(_shape(cfg)), T, _ptr(packed), _ptr(x), ctypes.byref(r), _ptr(y), path,
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
        _check("moe_forward", st)
        return
    ev = (ctypes.c_void_p * 4)(*(ctypes.c_void_p(e.cuda_event) for e in events))
    st = lib().moe_forward_timed(ctypes.byref(_shape(cfg)), T, _ptr(packed), _ptr(x), ctypes.byref(r), _ptr(y),
                                 path, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream), ev, 4)
    _check("moe_forward_timed", st)


def moe_event_record(event, stream=None) -> None:
    """Records a torch.cuda.Event on the stream; inside graph capture the record becomes a
    graph node that every replay executes."""
    _check("moe_event_record", lib().moe_event_record(ctypes.c_void_p(event.cuda_event), _stream(stream)))


def moe_decode_static(cfg, T, x, router_w, router_b, packed, rt: dict, y, stream=None) -> None:
    """Route + decode forward using the library's own scratch array (no workspace)."""
    r = routing_struct(rt)
    _check("moe_decode_static", lib().moe_decode_static(ctypes.byref(_shape(cfg)), T, _ptr(x), _ptr(router_w),
                                                         _ptr(router_b), _ptr(packed), ctypes.byref(r), _ptr(y),
                                                         _stream(stream)))


def moe_decode_static_get_error(stream=None):
    """(status, detail) recorded on the device by moe_decode_static calls since the last
    read; synchronises the stream and clears the record."""
    d = ctypes.c_uint32(0)
    st = lib().moe_decode_static_get_error(_stream(stream), ctypes.byref(d))
    return st, d.value


def moe_workspace_set_test_stall(ws, cycles: int, stream=None) -> None:
    """Failure-path tests only: the expert kernels of the next moe_forward calls on ws
    first wait up to `cycles` SM cycles on a barrier nothing completes (0 = off)."""
    _check("moe_workspace_set_test_stall",
           lib().moe_workspace_set_test_stall(_ptr(ws), ws.numel() * ws.element_size(), cycles, _stream(stream)))


def moe_route_fixed(cfg, T, x, ids, gates, rt: dict, ws, stream=None) -> None:
    """Routing of caller-given expert ids / gates (device int32 / float32 [T][k])."""
    r = routing_struct(rt)
    _check("moe_route_fixed", lib().moe_route_fixed(ctypes.byref(_shape(cfg)), T, _ptr(x), _ptr(ids), _ptr(gates),
                                                     ctypes.byref(r), _ptr(ws), ws.numel() * ws.element_size(),
                                                     _stream(stream)))


def moe_gather_rows(src, index, divisor, dst, ws, n=None, stream=None) -> None:
    """dst[i] = src[index[i] // divisor] for the first n rows (bf16 [rows][H] tensors)."""
    n = index.numel() if n is None else n
    _check("moe_gather_rows", lib().moe_gather_rows(n, src.shape[1], _ptr(src), src.shape[0], _ptr(index), divisor,
                                                     _ptr(dst), _ptr(ws), ws.numel() * ws.element_size(),
                                                     _stream(stream)))


def moe_combine_pairs(T, k, rows, inv_perm, gates, shared, y, ws, stream=None) -> None:
    """y[t] = sum_j gates[t][j] rows[inv_perm[t k + j]] + shared[t] (bf16 rows)."""
    _check("moe_combine_pairs", lib().moe_combine_pairs(T, k, y.shape[1], _ptr(rows), rows.shape[0], _ptr(inv_perm),
                                                         _ptr(gates), _ptr(shared), _ptr(y), _ptr(ws),
                                                         ws.numel() * ws.element_size(), _stream(stream)))


def moe_get_error(ws, stream=None):
    d = ctypes.c_uint32(0)
    st = lib().moe_get_error(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream), ctypes.byref(d))
    return st, d.value


def bf16_to_device(bits: np.ndarray, device="cuda"):
    """uint16 bf16 bit patterns (host) -> torch.bfloat16 device tensor (bit-exact)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_to_host(t) -> np.ndarray:
    """torch.bfloat16 tensor -> uint16 bit patterns (host)."""
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def moe_status_string(st: int) -> str:
    return lib().moe_status_string(st).decode()


class MoeLayer:
    """Device-resident layer: packed experts, router, workspace and routing buffers."""

    def __init__(self, cfg, packed_host: np.ndarray, router_w: np.ndarray, router_b, max_tokens: int,
                 device="cuda"):
        import torch
        self.cfg = cfg
        self.device = device
        self.packed = torch.from_numpy(packed_host).to(device)
        self.router_w = torch.from_numpy(np.ascontiguousarray(router_w, np.float32)).to(device)
        self.router_b = None if router_b is None else torch.from_numpy(
            np.ascontiguousarray(router_b, np.float32)).to(device)
        self.max_tokens = max_tokens
        self.ws = torch.empty(moe_workspace_size(cfg, max_tokens), dtype=torch.uint8, device=device)
        moe_workspace_init(self.ws)
        self.rt = alloc_routing(cfg, max_tokens, device)

    def route(self, x, T=None, stream=None):
        T = x.shape[0] if T is None else T
        moe_route(self.cfg, T, x, self.router_w, self.router_b, self.rt, self.ws, stream)

    def forward(self, x, y, T=None, path=PATH_AUTO, stream=None, events=None):
        T = x.shape[0] if T is None else T
        moe_forward(self.cfg, T, self.packed, x, self.rt, y, path, self.ws, stream, events)

    def __call__(self, x, path=PATH_AUTO, stream=None):
        import torch
        y = torch.empty((x.shape[0], self.cfg.H), dtype=torch.bfloat16, device=x.device)
        self.route(x, stream=stream)
        self.forward(x, y, path=path, stream=stream)
        return y
