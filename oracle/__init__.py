"""CPU oracle of the routed-MoE layer (fp64, single-threaded C per call).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check in
__graft_entry__.py and by bench.py's CPU-baseline / reference leg, never by the
product package.  The arithmetic lives in oracle.c; this module only marshals
numpy arrays and runs independent per-token calls in a thread pool (ctypes drops
the GIL during each call, and every C call is itself single-threaded).

Weights come in the generator's interchange form (see synth/gen.py), never from
the CUDA library's packer.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_fp = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_i32 = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u16 = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i8 = np.ctypeslib.ndpointer(dtype=np.int8, flags="C_CONTIGUOUS")
_u8 = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain -O2, no fast-math, no threads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_f16_to_f64.restype = ctypes.c_double
        L.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f64.restype = ctypes.c_double
        L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_logits.restype = None
        L.oracle_logits.argtypes = [ctypes.c_int] * 3 + [_u16, _fp, _dp]
        L.oracle_select.restype = None
        L.oracle_select.argtypes = [ctypes.c_int] * 3 + [_dp, _vp, _i32, _dp, _vp]
        L.oracle_permute.restype = None
        L.oracle_permute.argtypes = [ctypes.c_int] * 3 + [_i32] * 5
        L.oracle_expert_ffn.restype = ctypes.c_int
        L.oracle_expert_ffn.argtypes = ([ctypes.c_int] * 3 + [_vp] * 9 +
                                        [ctypes.c_int, _u16, _dp, _dp])
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [ctypes.c_int] * 3 + [_dp, _dp, _vp, _dp]
        L.oracle_unpack.restype = ctypes.c_int
        L.oracle_unpack.argtypes = [_u8, ctypes.c_size_t, ctypes.c_int, ctypes.c_int, _i8, _u16,
                                    ctypes.POINTER(ctypes.c_int)]
        _lib = L
    return _lib


def _threads(n: int | None) -> int:
    return max(1, n if n else (os.cpu_count() or 1))


# ---- router logits, top-k, gates ------------------------------------------

def logits(x: np.ndarray, Wr: np.ndarray, threads: int | None = None) -> np.ndarray:
    """fp64 [T][E] router logits (no bias)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    chunks = np.array_split(np.arange(T), min(T, 4 * _threads(threads))) if T else []

    def run(idx):
        if idx.size == 0:
            return
        t0, t1 = int(idx[0]), int(idx[-1]) + 1
        part = np.empty((t1 - t0, E), dtype=np.float64)
        lib().oracle_logits(t1 - t0, H, E, np.ascontiguousarray(x[t0:t1]), Wr, part)
        out[t0:t1] = part

    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(run, chunks))
    return out


def select(L: np.ndarray, bias, k: int, want_p: bool = False):
    """(ids int32 [T][k], gates fp64 [T][k][, p fp64 [T][E]]) from fp64 logits."""
    L = np.ascontiguousarray(L, dtype=np.float64)
    T, E = L.shape
    if E > 1024:
        raise ValueError("oracle_select handles E <= 1024")
    ids = np.empty((T, k), dtype=np.int32)
    gates = np.empty((T, k), dtype=np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    p = np.empty((T, E), dtype=np.float64) if want_p else None
    lib().oracle_select(T, E, k, L, None if b is None else b.ctypes.data, ids, gates,
                        None if p is None else p.ctypes.data)
    return (ids, gates, p) if want_p else (ids, gates)


def route(x, Wr, bias, k, threads=None):
    """Full routing: (logits fp64 [T][E] without bias, ids, gates)."""
    L = logits(x, Wr, threads)
    ids, gates = select(L, bias, k)
    return L, ids, gates


def topk_gaps(L: np.ndarray, bias, k: int) -> np.ndarray:
    """Smallest gap between adjacent values among each token's k+1 largest biased
    logits (fp64).  Tokens with a gap below 1e-4 are redrawn by the test harness so
    that fp32 and fp64 routing cannot disagree."""
    z = L + (0.0 if bias is None else np.asarray(bias, dtype=np.float64)[None, :])
    kk = min(k + 1, z.shape[1])
    top = -np.sort(-z, axis=1)[:, :kk]
    if kk < 2:
        return np.full(z.shape[0], np.inf)
    return np.min(top[:, :-1] - top[:, 1:], axis=1)


# ---- histogram, scan, permutation -----------------------------------------

def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    lib().oracle_permute(T, E, k, ids, counts, offsets, perm, inv)
    return counts, offsets, perm, inv


# ---- expert FFNs and the combine ------------------------------------------

def _ptr(a):
    return None if a is None else a.ctypes.data


def expert_ffn(H: int, I: int, fmt: int, mats: dict, x: np.ndarray) -> np.ndarray:
    """fp64 [n][H] = Wd (silu(Wg x) * (Wu x)) for bf16 rows x [n][H]."""
    x = np.ascontiguousarray(x, dtype=np.uint16).reshape(-1, H)
    n = x.shape[0]
    y = np.empty((n, H), dtype=np.float64)
    scratch = np.empty(2 * max(H, I) + I * max(n, 1), dtype=np.float64)
    keep = []
    args = []
    for name in ("gate", "up", "down"):
        c, h, s = mats[name]
        c = np.ascontiguousarray(c, dtype=np.uint8)
        h = None if h is None else np.ascontiguousarray(h, dtype=np.uint8)
        s = np.ascontiguousarray(s, dtype=np.uint16)
        keep += [c, h, s]
        args += [_ptr(c), _ptr(h), _ptr(s)]
    if fmt == 2 and any(mats[m][1] is None for m in mats):
        raise ValueError("3-bit expert without its third-bit plane")
    rc = lib().oracle_expert_ffn(H, I, fmt, *args, n, x, y, scratch)
    if rc:
        raise ValueError("bad code in expert weights (ternary code 3)")
    return y


def combine(gates: np.ndarray, y_routed: np.ndarray, y_shared) -> np.ndarray:
    gates = np.ascontiguousarray(gates, dtype=np.float64)
    y_routed = np.ascontiguousarray(y_routed, dtype=np.float64)
    k, H = y_routed.shape
    S = 0 if y_shared is None else y_shared.shape[0]
    ys = None if y_shared is None else np.ascontiguousarray(y_shared, dtype=np.float64)
    y = np.empty(H, dtype=np.float64)
    lib().oracle_combine(H, k, S, gates, y_routed, _ptr(ys), y)
    return y


def forward_tokens(layer, x: np.ndarray, ids: np.ndarray, gates: np.ndarray, tokens,
                   threads: int | None = None, expert_cache: dict | None = None) -> np.ndarray:
    """fp64 [len(tokens)][H] layer output for the listed tokens.

    layer: object with .cfg (H, I, E, S), .fmt and .expert(e) -> {'gate','up','down'}
    (e.g. synth.Layer).  Work is done expert by expert (each expert's weights are
    drawn once), running the listed tokens of that expert in one C call; expert
    calls run in a thread pool."""
    cfg = layer.cfg
    H, I, E, S, k = cfg.H, cfg.I, cfg.E, cfg.S, ids.shape[1]
    tokens = [int(t) for t in tokens]
    need: dict[int, list] = {}
    for t in tokens:
        for j in range(k):
            need.setdefault(int(ids[t, j]), []).append(t)
    for s in range(S):
        need[E + s] = list(tokens)
    y_exp: dict[tuple, np.ndarray] = {}

    def run(e):
        mats = expert_cache.get(e) if expert_cache is not None else None
        if mats is None:
            mats = layer.expert(e)
        ts = need[e]
        ys = expert_ffn(H, I, int(layer.fmt[e]), mats, x[ts])
        return e, ts, ys

    with ThreadPoolExecutor(_threads(threads)) as ex:
        for e, ts, ys in ex.map(run, sorted(need)):
            for t, yrow in zip(ts, ys):
                y_exp[(e, t)] = yrow
    out = np.empty((len(tokens), H), dtype=np.float64)
    for i, t in enumerate(tokens):
        yr = np.stack([y_exp[(int(ids[t, j]), t)] for j in range(k)])
        ysh = np.stack([y_exp[(E + s, t)] for s in range(S)]) if S else None
        out[i] = combine(gates[t], yr, ysh)
    return out


def unpack(buf: np.ndarray, table: int, which: int, rows: int, K: int):
    """(fmt, codes int8 [rows][K], scales uint16 [rows][K/64]) read from a packed buffer."""
    buf = np.ascontiguousarray(buf, dtype=np.uint8)
    codes = np.empty((rows, K), dtype=np.int8)
    scales = np.empty((rows, K // 64), dtype=np.uint16)
    fmt = ctypes.c_int(-1)
    rc = lib().oracle_unpack(buf, buf.size, table, which, codes, scales, ctypes.byref(fmt))
    if rc:
        raise ValueError(f"oracle_unpack failed: {rc}")
    return fmt.value, codes, scales
