"""Python binding of libmoe_b200.so, the sm_100a routed-expert MoE layer library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels; torch supplies device memory and the current stream.  The functions
keep the C names of include/moe.h.  There is no CPU fallback: without the
built library or a CUDA device every call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
          4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_DEVICE_FLAG"}
FLAG_BAD_EXPERT_INDEX = 0x1
FLAG_BAD_EXPERT_SHAPE = 0x2
FLAG_FP16_OVERFLOW = 0x4
FLAG_WAIT_TIMEOUT = 0x8
PATH_AUTO, PATH_GEMV, PATH_TENSOR = 0, 1, 2
LAYER_EVENTS = 6

# C functions declared in include/moe.h (the export test checks this list).
EXPORTS = ["moe_status_str", "moe_abi_version", "moe_workspace_init", "moe_workspace_status",
           "moe_quantize_rows", "moe_route_workspace_bytes", "moe_route_topk", "moe_bucket",
           "moe_expert_ffn_workspace_bytes", "moe_expert_ffn", "moe_layer_workspace_bytes",
           "moe_layer_forward", "moe_layer_forward_ex", "moe_rmsnorm_bf16",
           "moe_stack_workspace_bytes", "moe_stack_forward",
           "moe_route_noalloc_max_scratch_bytes", "moe_route_topk_noalloc",
           "moe_layer_workspace_bytes_ex", "moe_workspace_set_wait_limit"]


class MoEError(RuntimeError):
    def __init__(self, fn, code, flags=None):
        msg = f"{fn}: {STATUS.get(code, code)}"
        if flags:
            msg += f" (device flags 0x{flags:x})"
        super().__init__(msg)
        self.code = code
        self.flags = flags


class moe_qmat(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("bits", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class moe_expert(ctypes.Structure):
    _fields_ = [("gate", moe_qmat), ("up", moe_qmat), ("down", moe_qmat)]


class moe_router_cfg(ctypes.Structure):
    _fields_ = [("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("expert_topp", ctypes.c_float)]


class moe_layer_params(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("experts", ctypes.c_void_p), ("shared", ctypes.c_void_p),
                ("weight_bits", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None
_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t


def load():
    """Load the library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built (python -m int4_routed_expert_route_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    L.moe_status_str.restype = ctypes.c_char_p
    L.moe_abi_version.restype = _i32
    for name in ("moe_route_workspace_bytes", "moe_expert_ffn_workspace_bytes",
                 "moe_layer_workspace_bytes", "moe_stack_workspace_bytes",
                 "moe_route_noalloc_max_scratch_bytes", "moe_layer_workspace_bytes_ex"):
        getattr(L, name).restype = _sz
    L.moe_route_workspace_bytes.argtypes = [_i64, _i64, ctypes.POINTER(moe_router_cfg)]
    L.moe_expert_ffn_workspace_bytes.argtypes = [_i64, _i64, _i64]
    L.moe_layer_workspace_bytes.argtypes = [_i64, _i64, _i64, ctypes.POINTER(moe_router_cfg)]
    L.moe_stack_workspace_bytes.argtypes = [_i64, _i64, _i64, ctypes.POINTER(moe_router_cfg)]
    L.moe_layer_workspace_bytes_ex.argtypes = [_i64, _i64, _i64, ctypes.POINTER(moe_router_cfg), _i32]
    for name in EXPORTS:
        if name.endswith("_bytes") or name in ("moe_status_str", "moe_abi_version"):
            continue
        getattr(L, name).restype = ctypes.c_int
    L.moe_workspace_init.argtypes = [_vp, _sz, _vp]
    L.moe_workspace_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
    L.moe_workspace_set_wait_limit.argtypes = [_vp, _sz, ctypes.c_uint32, _vp]
    L.moe_quantize_rows.argtypes = [_vp, _i64, _i64, _i32, _vp, _vp, _vp]
    L.moe_route_topk.argtypes = [_vp, _i64, _i64, _vp, _vp, ctypes.POINTER(moe_router_cfg), _vp,
                                 _vp, _vp, _vp, _sz, _vp]
    L.moe_route_noalloc_max_scratch_bytes.argtypes = []
    L.moe_route_topk_noalloc.argtypes = [_vp, _i64, _i64, _vp, _vp,
                                         ctypes.POINTER(moe_router_cfg), _vp, _vp, _vp, _vp]
    L.moe_bucket.argtypes = [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp]
    L.moe_expert_ffn.argtypes = [_vp, _i64, _i64, _i64, ctypes.POINTER(moe_expert), _vp, _vp,
                                 _i64, _vp, _vp, _sz, _vp]
    L.moe_layer_forward.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp,
                                    ctypes.POINTER(moe_router_cfg), _vp, _vp, _i32, _vp, _vp, _vp,
                                    _vp, _sz, _vp]
    L.moe_layer_forward_ex.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp,
                                       ctypes.POINTER(moe_router_cfg), _vp, _vp, _i32, _vp, _vp,
                                       _vp, _vp, _sz, _i32, _i32, _vp, _vp]
    L.moe_rmsnorm_bf16.argtypes = [_vp, _i64, _i64, ctypes.c_float, _vp, _vp]
    L.moe_stack_forward.argtypes = [_vp, _i64, _i64, _i64, _i32, ctypes.POINTER(moe_layer_params),
                                    ctypes.POINTER(moe_router_cfg), ctypes.c_float, _vp, _vp, _vp,
                                    _sz, _vp]
    _lib = L
    return L


def _check(fn, rc):
    if rc != MOE_OK:
        raise MoEError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t


def _bf16(t, name):
    return _dev(t, torch.bfloat16, name)


def router_cfg(n_experts, top_k, n_group=1, topk_group=1, rsf=1.0, topp=0.0):
    return moe_router_cfg(n_experts, top_k, n_group, topk_group, rsf, topp)


class Workspace:
    """A caller-owned workspace (torch memory) with its device flag word cleared."""

    def __init__(self, nbytes, device=None):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        _check("moe_workspace_init", load().moe_workspace_init(_ptr(self.buf), self.nbytes,
                                                              _stream()))

    def ptr(self):
        return _ptr(self.buf)

    def flags(self):
        f = ctypes.c_uint32(0)
        rc = load().moe_workspace_status(_ptr(self.buf), _stream(), ctypes.byref(f))
        if rc not in (MOE_OK, 5):
            raise MoEError("moe_workspace_status", rc)
        return int(f.value)

    def reset(self):
        _check("moe_workspace_init", load().moe_workspace_init(_ptr(self.buf), self.nbytes,
                                                              _stream()))

    def set_wait_limit(self, wait_us, stream=None):
        """Bound the on-chip waits of calls on this workspace (0: two seconds)."""
        _check("moe_workspace_set_wait_limit",
               load().moe_workspace_set_wait_limit(_ptr(self.buf), self.nbytes, int(wait_us),
                                                   _stream(stream)))


# ----------------------------------------------------------------------------- quantise
def moe_quantize_rows(w, bits, q_out=None, scale_out=None, stream=None):
    """Per-row quantisation of fp32 [rows, cols] -> (packed uint8, fp32 scales)."""
    w = _dev(w, torch.float32, "w")
    rows, cols = w.shape
    if q_out is None:
        q_out = torch.empty((rows, (cols * bits + 7) // 8), dtype=torch.uint8, device=w.device)
    if scale_out is None:
        scale_out = torch.empty(rows, dtype=torch.float32, device=w.device)
    _check("moe_quantize_rows", load().moe_quantize_rows(_ptr(w), rows, cols, bits, _ptr(q_out),
                                                         _ptr(scale_out), _stream(stream)))
    return q_out, scale_out


class QuantExpert:
    """One quantised SwiGLU expert on the device (gate/up [I,H], down [H,I])."""

    def __init__(self, qg, sg, qu, su, qd, sd, bits, H, I):
        self.t = (qg, sg, qu, su, qd, sd)
        self.bits, self.H, self.I = bits, H, I

    @classmethod
    def from_fp32(cls, wg, wu, wd, bits=4):
        I, H = wg.shape
        qg, sg = moe_quantize_rows(wg, bits)
        qu, su = moe_quantize_rows(wu, bits)
        qd, sd = moe_quantize_rows(wd, bits)
        return cls(qg, sg, qu, su, qd, sd, bits, H, I)

    def struct(self):
        qg, sg, qu, su, qd, sd = self.t
        b, H, I = self.bits, self.H, self.I
        return moe_expert(moe_qmat(qg.data_ptr(), sg.data_ptr(), b, 0, I, H),
                          moe_qmat(qu.data_ptr(), su.data_ptr(), b, 0, I, H),
                          moe_qmat(qd.data_ptr(), sd.data_ptr(), b, 0, H, I))

    def nbytes(self):
        return sum(t.numel() * t.element_size() for t in self.t)


class ExpertTable:
    """Device array of moe_expert structs (keeps the expert tensors alive)."""

    def __init__(self, experts, device="cuda"):
        self.experts = list(experts)
        arr = (moe_expert * len(self.experts))(*[e.struct() for e in self.experts])
        raw = bytes(memoryview(arr).cast("B"))
        self.dev = torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(device)

    def ptr(self):
        return _ptr(self.dev)


class SharedExpert(ExpertTable):
    def __init__(self, expert, device="cuda"):
        super().__init__([expert], device)


# ----------------------------------------------------------------------------- router
def moe_route_workspace_bytes(T, H, cfg):
    return int(load().moe_route_workspace_bytes(T, H, ctypes.byref(cfg)))


def moe_route_topk(x, gate, bias, cfg, ws=None, with_gap=False, stream=None):
    x = _bf16(x, "x")
    gate = _dev(gate, torch.float32, "gate")
    bias = _dev(bias, torch.float32, "bias")
    T, H = x.shape
    k = cfg.top_k
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    gap = torch.empty(T, dtype=torch.float32, device=x.device) if with_gap else None
    if ws is None:
        ws = Workspace(moe_route_workspace_bytes(T, H, cfg), x.device)
    _check("moe_route_topk", load().moe_route_topk(_ptr(x), T, H, _ptr(gate), _ptr(bias),
                                                   ctypes.byref(cfg), _ptr(idx), _ptr(w),
                                                   _ptr(gap), ws.ptr(), ws.nbytes,
                                                   _stream(stream)))
    return idx, w, gap


def moe_route_topk_noalloc(x, gate, bias, cfg, with_gap=False, stream=None):
    """moe_route_topk with the library's built-in scratch (no workspace)."""
    x = _bf16(x, "x")
    gate = _dev(gate, torch.float32, "gate")
    bias = _dev(bias, torch.float32, "bias")
    T, H = x.shape
    k = cfg.top_k
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    gap = torch.empty(T, dtype=torch.float32, device=x.device) if with_gap else None
    _check("moe_route_topk_noalloc", load().moe_route_topk_noalloc(
        _ptr(x), T, H, _ptr(gate), _ptr(bias), ctypes.byref(cfg), _ptr(idx), _ptr(w), _ptr(gap),
        _stream(stream)))
    return idx, w, gap


def moe_bucket(idx, E, stream=None):
    idx = _dev(idx, torch.int32, "idx")
    T, k = idx.shape
    d = idx.device
    counts = torch.empty(E, dtype=torch.int32, device=d)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=d)
    lst = torch.empty(max(T * k, 1), dtype=torch.int32, device=d)
    uniq = torch.empty(E, dtype=torch.int32, device=d)
    nu = torch.empty(1, dtype=torch.int32, device=d)
    _check("moe_bucket", load().moe_bucket(_ptr(idx), T, k, E, _ptr(counts), _ptr(offsets),
                                           _ptr(lst), _ptr(uniq), _ptr(nu), _stream(stream)))
    return dict(counts=counts, offsets=offsets, list=lst, unique=uniq, n_unique=nu)


# ----------------------------------------------------------------------------- FFN / layer
def moe_expert_ffn(x, expert: QuantExpert, y, rows=None, row_w=None, ws=None, stream=None):
    """y[rows] += row_w * FFN(x[rows]) (in place)."""
    x = _bf16(x, "x")
    y = _dev(y, torch.float32, "y")
    T, H = x.shape
    n_rows = T if rows is None else rows.numel()
    if ws is None:
        ws = Workspace(load().moe_expert_ffn_workspace_bytes(n_rows, H, expert.I), x.device)
    st = expert.struct()
    _check("moe_expert_ffn", load().moe_expert_ffn(_ptr(x), T, H, expert.I, ctypes.byref(st),
                                                   _ptr(rows), _ptr(row_w), n_rows, _ptr(y),
                                                   ws.ptr(), ws.nbytes, _stream(stream)))
    return y


def moe_layer_workspace_bytes(T, H, I, cfg, path=PATH_AUTO):
    return int(load().moe_layer_workspace_bytes_ex(T, H, I, ctypes.byref(cfg), path))


def moe_layer_forward(x, gate, bias, cfg, experts: ExpertTable, shared=None, weight_bits=4,
                      y=None, idx_out=None, w_out=None, ws=None, path=PATH_AUTO, accumulate=False,
                      events=None, stream=None, I=None):
    x = _bf16(x, "x")
    T, H = x.shape
    if I is None:
        I = experts.experts[0].I
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = Workspace(moe_layer_workspace_bytes(T, H, I, cfg, path), x.device)
    ev = None
    if events is not None:
        ev = (ctypes.c_void_p * LAYER_EVENTS)(*[e.cuda_event if e is not None else None for e in events])
    rc = load().moe_layer_forward_ex(_ptr(x), T, H, I, _ptr(gate), _ptr(bias), ctypes.byref(cfg),
                                     experts.ptr(), shared.ptr() if shared is not None else None,
                                     weight_bits, _ptr(y), _ptr(idx_out), _ptr(w_out), ws.ptr(),
                                     ws.nbytes, path, 1 if accumulate else 0, ev, _stream(stream))
    _check("moe_layer_forward", rc)
    return y


def moe_rmsnorm_bf16(v, eps=1e-6, out=None, stream=None):
    v = _dev(v, torch.float32, "v")
    T, H = v.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=v.device)
    _check("moe_rmsnorm_bf16", load().moe_rmsnorm_bf16(_ptr(v), T, H, eps, _ptr(out),
                                                       _stream(stream)))
    return out


def moe_stack_workspace_bytes(T, H, I, cfg):
    return int(load().moe_stack_workspace_bytes(T, H, I, ctypes.byref(cfg)))


def moe_stack_forward(resid, layers, cfg, I, eps=1e-6, layer_inputs=None, idx_out=None, ws=None,
                      stream=None):
    """layers: list of (gate, bias, ExpertTable, SharedExpert-or-None, weight_bits)."""
    resid = _dev(resid, torch.float32, "resid")
    T, H = resid.shape
    arr = (moe_layer_params * len(layers))(*[
        moe_layer_params(g.data_ptr(), b.data_ptr(), et.dev.data_ptr(),
                         sh.dev.data_ptr() if sh is not None else None, bits, 0)
        for (g, b, et, sh, bits) in layers])
    if ws is None:
        ws = Workspace(moe_stack_workspace_bytes(T, H, I, cfg), resid.device)
    _check("moe_stack_forward", load().moe_stack_forward(
        _ptr(resid), T, H, I, len(layers), arr, ctypes.byref(cfg), eps, _ptr(layer_inputs),
        _ptr(idx_out), ws.ptr(), ws.nbytes, _stream(stream)))
    return resid
