"""NumPy front end of the plain-C oracle of the routed-expert MoE layer.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the CPU
baseline leg of the benchmark may import this module; the product path may not.
It shares no code with the CUDA library.  Arrays in, arrays out; bf16 values are
passed as their uint16 bit patterns.

Every function wraps one routine of ``moe_oracle.c``; see that file for the
definitions and the readings taken where the pages are silent.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_f32 = ctypes.c_float
_f64 = ctypes.c_double
_vp = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        L.orc_row_bytes.restype = _i64
        L.orc_row_bytes.argtypes = [ctypes.c_int, _i64]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_double_to_bf16.argtypes = [_f64]
        L.orc_pack.argtypes = [_vp, _i64, _i64, ctypes.c_int, _vp]
        L.orc_unpack.argtypes = [_vp, _i64, _i64, ctypes.c_int, _vp]
        L.orc_quantize_rows.argtypes = [_vp, _i64, _i64, ctypes.c_int, _vp, _vp]
        L.orc_dequant_rows.argtypes = [_vp, _vp, _i64, _i64, ctypes.c_int, _vp]
        L.orc_route.argtypes = [_vp, _i64, _i64, _vp, _vp, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, _f32, _f32, _vp, _vp, _vp, _vp, _vp]
        L.orc_route_from_scores.argtypes = [_vp, _i64, _vp, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, _f32, _f32, _vp, _vp,
                                            _vp, _vp, _vp]
        L.orc_bucket.argtypes = [_vp, _i64, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
        L.orc_expert_ffn.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                     ctypes.c_int, _vp]
        L.orc_layer.argtypes = ([_vp, _i64, _i64, _i64, _vp, _vp, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_int, _f32, _f32]
                                + [_vp] * 6 + [ctypes.c_int] + [_vp] * 6 + [ctypes.c_int]
                                + [_vp] * 5)
        L.orc_rmsnorm_bf16.argtypes = [_vp, _i64, _i64, _f64, _vp, _vp]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _ok(rc, what):
    if rc != 0:
        raise OracleError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    """Threads the expert FFN rows are split over (results do not depend on it)."""
    lib().orc_set_num_threads(int(n))


def row_bytes(bits: int, cols: int) -> int:
    return int(lib().orc_row_bytes(bits, cols))


# ---------------------------------------------------------------- bf16
def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    flat, of = a.reshape(-1), out.reshape(-1)
    L = lib()
    for i in range(flat.size):
        of[i] = L.orc_double_to_bf16(float(flat[i]))
    return out


def double_to_bf16_bits(a) -> np.ndarray:
    a = _c(a, np.float64)
    out = np.empty(a.shape, np.uint16)
    flat, of = a.reshape(-1), out.reshape(-1)
    L = lib()
    for i in range(flat.size):
        of[i] = L.orc_double_to_bf16(float(flat[i]))
    return out


def bf16_bits_to_f64(b) -> np.ndarray:
    b = _c(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- quantisation
def pack(q, bits: int) -> np.ndarray:
    q = _c(q, np.int32)
    rows, cols = q.shape
    out = np.zeros((rows, row_bytes(bits, cols)), np.uint8)
    _ok(lib().orc_pack(_p(q), rows, cols, bits, _p(out)), "pack")
    return out


def unpack(packed, cols: int, bits: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    rows = packed.shape[0]
    q = np.zeros((rows, cols), np.int32)
    _ok(lib().orc_unpack(_p(packed), rows, cols, bits, _p(q)), "unpack")
    return q


def quantize_rows(w, bits: int):
    """Per-row symmetric quantisation; returns (packed uint8 [R, C*bits/8], scale fp32 [R])."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    q = np.zeros((rows, row_bytes(bits, cols)), np.uint8)
    s = np.zeros(rows, np.float32)
    _ok(lib().orc_quantize_rows(_p(w), rows, cols, bits, _p(q), _p(s)), "quantize_rows")
    return q, s


def dequant_rows(packed, scale, cols: int, bits: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    scale = _c(scale, np.float32)
    rows = packed.shape[0]
    out = np.zeros((rows, cols), np.float64)
    _ok(lib().orc_dequant_rows(_p(packed), _p(scale), rows, cols, bits, _p(out)), "dequant")
    return out


# ---------------------------------------------------------------- router
def route(x_bits, gate, bias, k, n_group=1, topk_group=1, rsf=1.0, topp=0.0):
    """Returns dict(idx [T,k] int32, w [T,k] fp32, gap [T], ggap [T], scores [T,E] fp32)."""
    x_bits = _c(x_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    T, H = x_bits.shape
    E = gate.shape[0]
    assert gate.shape == (E, H) and bias.shape == (E,)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    gap = np.zeros(T, np.float64)
    ggap = np.zeros(T, np.float64)
    scores = np.zeros((T, E), np.float32)
    _ok(lib().orc_route(_p(x_bits), T, H, _p(gate), _p(bias), E, k, n_group, topk_group,
                        rsf, topp, _p(idx), _p(w), _p(gap), _p(ggap), _p(scores)), "route")
    return dict(idx=idx, w=w, gap=gap, ggap=ggap, scores=scores)


def route_from_scores(scores, bias, k, n_group=1, topk_group=1, rsf=1.0, topp=0.0):
    scores = _c(scores, np.float32)
    bias = _c(bias, np.float32)
    T, E = scores.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    gap = np.zeros(T, np.float64)
    ggap = np.zeros(T, np.float64)
    gsel = np.zeros((T, n_group), np.int32)
    _ok(lib().orc_route_from_scores(_p(scores), T, _p(bias), E, k, n_group, topk_group, rsf,
                                    topp, _p(idx), _p(w), _p(gap), _p(ggap), _p(gsel)),
        "route_from_scores")
    return dict(idx=idx, w=w, gap=gap, ggap=ggap, group_sel=gsel)


# ---------------------------------------------------------------- bucketing
def bucket(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    lst = np.zeros(T * k, np.int32)
    uniq = np.zeros(E, np.int32)
    nu = np.zeros(1, np.int32)
    _ok(lib().orc_bucket(_p(idx), T, k, E, _p(counts), _p(offsets), _p(lst), _p(uniq), _p(nu)),
        "bucket")
    n = int(offsets[E])
    return dict(counts=counts, offsets=offsets, list=lst[:n], unique=uniq[:int(nu[0])])


# ---------------------------------------------------------------- FFN / layer
class Expert:
    """Host copy of one quantised expert: gate/up [I,H], down [H,I], packed + scales."""

    def __init__(self, qg, sg, qu, su, qd, sd, bits=4):
        self.qg, self.sg = _c(qg, np.uint8), _c(sg, np.float32)
        self.qu, self.su = _c(qu, np.uint8), _c(su, np.float32)
        self.qd, self.sd = _c(qd, np.uint8), _c(sd, np.float32)
        self.bits = bits

    def ptrs(self):
        return [_p(self.qg), _p(self.sg), _p(self.qu), _p(self.su), _p(self.qd), _p(self.sd)]


def expert_ffn(x_bits, ex: Expert, H: int, I: int) -> np.ndarray:
    x_bits = _c(x_bits, np.uint16)
    T = x_bits.shape[0]
    y = np.zeros((T, H), np.float64)
    _ok(lib().orc_expert_ffn(_p(x_bits), T, H, I, *ex.ptrs(), ex.bits, _p(y)), "expert_ffn")
    return y


def layer(x_bits, gate, bias, experts, shared, H, I, k, n_group=1, topk_group=1, rsf=1.0,
          topp=0.0, idx_in=None, w_in=None):
    """MoE layer.  ``experts`` is a list of E entries (Expert or None when unused)."""
    x_bits = _c(x_bits, np.uint16)
    gate = _c(gate, np.float32)
    bias = _c(bias, np.float32)
    T = x_bits.shape[0]
    E = len(experts)
    bits = next(e.bits for e in experts if e is not None) if any(
        e is not None for e in experts) else 4
    arrs = [(ctypes.c_void_p * E)() for _ in range(6)]
    for e, ex in enumerate(experts):
        if ex is None:
            continue
        for a, p in zip(arrs, ex.ptrs()):
            a[e] = p
    sh = shared.ptrs() if shared is not None else [None] * 6
    sh_bits = shared.bits if shared is not None else 4
    y = np.zeros((T, H), np.float64)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    if idx_in is not None:
        idx_in = _c(idx_in, np.int32)
        w_in = _c(w_in, np.float32)
    rc = lib().orc_layer(_p(x_bits), T, H, I, _p(gate), _p(bias), E, k, n_group, topk_group,
                         rsf, topp, *[ctypes.cast(a, _vp) for a in arrs], bits, *sh, sh_bits,
                         _p(idx_in), _p(w_in), _p(y), _p(idx), _p(w))
    if rc == 2:
        raise OracleError("a routed expert chosen by some token was not supplied")
    _ok(rc, "layer")
    return dict(y=y, idx=idx, w=w)


def rmsnorm_bf16(v, eps=1e-6):
    v = _c(v, np.float64)
    T, H = v.shape
    out = np.zeros((T, H), np.uint16)
    of = np.zeros((T, H), np.float64)
    _ok(lib().orc_rmsnorm_bf16(_p(v), T, H, eps, _p(out), _p(of)), "rmsnorm")
    return out, of
