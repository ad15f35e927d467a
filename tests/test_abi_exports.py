"""CPU checks of the C-ABI library: it loads, exports every entry point that
include/moe.h declares, and rejects invalid arguments on the host (these paths
return before any CUDA call, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def so():
    from int4_routed_expert_route_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_and_binding_agree():
    import int4_routed_expert_route_b200 as m
    assert declared() == sorted(m.EXPORTS)


def test_library_exports_every_declared_symbol(so):
    for name in declared():
        assert hasattr(so, name), name


def test_status_strings_and_version(so):
    so.moe_status_str.restype = ctypes.c_char_p
    assert so.moe_status_str(0) == b"MOE_OK"
    assert so.moe_status_str(4) == b"MOE_ERR_WORKSPACE"
    assert so.moe_abi_version() >= 1


def test_host_side_validation(so):
    import int4_routed_expert_route_b200 as m
    so.moe_quantize_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p]
    fake = ctypes.c_void_p(0x1000)
    assert so.moe_quantize_rows(fake, 4, 8, 3, fake, fake, None) == 1  # bad bits
    assert so.moe_quantize_rows(fake, 4, 7, 4, fake, fake, None) == 1  # odd cols for int4
    assert so.moe_quantize_rows(fake, 4, 6, 2, fake, fake, None) == 1  # cols % 4 for int2
    assert so.moe_quantize_rows(None, 4, 8, 4, fake, fake, None) == 1  # null input
    so.moe_layer_workspace_bytes.restype = ctypes.c_size_t
    so.moe_layer_workspace_bytes.argtypes = [ctypes.c_int64] * 3 + [ctypes.POINTER(m.moe_router_cfg)]
    good = m.router_cfg(256, 8, 8, 4, 2.5)
    assert so.moe_layer_workspace_bytes(1, 6144, 2048, ctypes.byref(good)) > 0
    for bad in (m.router_cfg(256, 8, 8, 9, 2.5),   # topk_group > n_group
                m.router_cfg(256, 40, 8, 4, 2.5),  # k > 32
                m.router_cfg(2048, 8, 8, 4, 2.5),  # E > 1024
                m.router_cfg(8, 2, 8, 1, 2.5),     # one expert per group
                m.router_cfg(256, 129, 8, 4, 2.5)):
        assert so.moe_layer_workspace_bytes(1, 6144, 2048, ctypes.byref(bad)) == 0
    so.moe_layer_forward.argtypes = m.load().moe_layer_forward.argtypes
    so.moe_layer_forward.restype = ctypes.c_int
    # workspace too small is refused before any launch
    rc = so.moe_layer_forward(fake, 1, 6144, 2048, fake, fake, ctypes.byref(good), fake, None, 4,
                              fake, None, None, fake, 16, None)
    assert rc == 4
    # misaligned activations
    rc = so.moe_layer_forward(ctypes.c_void_p(0x1002), 1, 6144, 2048, fake, fake,
                              ctypes.byref(good), fake, None, 4, fake, None, None, fake,
                              1 << 30, None)
    assert rc == 1
    # bad bit width
    rc = so.moe_layer_forward(fake, 1, 6144, 2048, fake, fake, ctypes.byref(good), fake, None, 3,
                              fake, None, None, fake, 1 << 30, None)
    assert rc == 1
    # hidden size not a multiple of 64
    rc = so.moe_layer_forward(fake, 1, 6100, 2048, fake, fake, ctypes.byref(good), fake, None, 4,
                              fake, None, None, fake, 1 << 30, None)
    assert rc == 1


def test_workspace_sizes_grow_with_batch(so):
    import int4_routed_expert_route_b200 as m
    L = m.load()
    cfg = m.router_cfg(256, 8, 8, 4, 2.5)
    a = m.moe_layer_workspace_bytes(1, 6144, 2048, cfg)
    b = m.moe_layer_workspace_bytes(32, 6144, 2048, cfg)
    assert 0 < a < b
    assert L.moe_expert_ffn_workspace_bytes(4, 6144, 2048) >= 256 + 4 * 2048 * 4


def test_library_has_no_unresolved_internal_symbols(so):
    """Every internal (namespace moe) function the library calls is defined in it."""
    import subprocess
    from int4_routed_expert_route_b200 import build
    out = subprocess.run(["nm", "-u", build.LIB], capture_output=True, text=True).stdout
    assert "_ZN3moe" not in out


def test_host_side_path_and_size_contracts(so):
    """Refusals the boundary makes on the host, before any launch (no GPU needed)."""
    import int4_routed_expert_route_b200 as m
    L = m.load()
    fake = ctypes.c_void_p(0x1000)
    cfg = m.router_cfg(256, 8, 8, 4, 2.5)
    big = 1 << 40

    def fwd(T, H, I, bits, path, ws_bytes=big):
        return L.moe_layer_forward_ex(fake, T, H, I, fake, fake, ctypes.byref(cfg), fake, None,
                                      bits, fake, None, None, fake, ws_bytes, path, 0, None, None)

    # the tensor-core path takes int4 experts with H, I multiples of 128 only
    assert fwd(256, 6144, 2048, 8, m.PATH_TENSOR) == 2
    assert fwd(256, 6144 + 64, 2048, 4, m.PATH_TENSOR) == 2
    # the CUDA-core path stops at 4096 tokens
    assert fwd(4097, 6144, 2048, 4, m.PATH_GEMV) == 2
    # an empty batch is fine and launches nothing
    assert fwd(0, 6144, 2048, 4, m.PATH_AUTO) == 0
    # AUTO runs int8/int2 layers on the CUDA-core path: its workspace must fit in the one
    # sized for AUTO (which plans the tensor path from 9 tokens on)
    for T in (1, 2, 8, 9, 63, 64, 256, 4096):
        auto = m.moe_layer_workspace_bytes(T, 6144, 2048, cfg)
        gemv = m.moe_layer_workspace_bytes(T, 6144, 2048, cfg, m.PATH_GEMV)
        assert 0 < gemv <= auto, T
        assert fwd(T, 6144, 2048, 8, m.PATH_AUTO, ws_bytes=gemv - 1) == 4  # sized for GEMV
    # stack and RMSNorm argument errors
    assert L.moe_stack_forward(fake, 1, 6144, 2048, -1, None, ctypes.byref(cfg), 1e-6, None, None,
                               fake, big, None) == 1
    need = L.moe_stack_workspace_bytes(1, 6144, 2048, ctypes.byref(cfg))
    assert need > m.moe_layer_workspace_bytes(1, 6144, 2048, cfg)
    assert L.moe_stack_forward(fake, 1, 6144, 2048, 0, None, ctypes.byref(cfg), 1e-6, None, None,
                               fake, need - 1, None) == 4
    assert L.moe_rmsnorm_bf16(fake, 1, 6144, ctypes.c_float(-1.0), fake, None) == 1
    assert L.moe_rmsnorm_bf16(fake, 1, 6144, ctypes.c_float(float("nan")), fake, None) == 1


def test_bucket_limits_refused_on_host(so):
    """moe_bucket's limits (its counters live in shared memory: E <= 1024; pair
    indices fit 24 bits) are checked before any launch."""
    so.moe_bucket.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32] + \
        [ctypes.c_void_p] * 6
    so.moe_bucket.restype = ctypes.c_int
    f = ctypes.c_void_p(0x1000)

    def call(T, k, E, idx=f, lst=f):
        return so.moe_bucket(idx, T, k, E, f, f, lst, f, f, None)

    assert call(4, 8, 1025) == 1              # more experts than shared-memory counters
    assert call((1 << 24) // 8 + 1, 8, 256) == 1  # T * k above 2^24
    assert call(4, 0, 256) == 1               # no slots
    assert call(-1, 8, 256) == 1              # negative batch
    assert call(4, 8, 256, idx=None) == 1     # pairs without indices
    assert call(4, 8, 256, lst=None) == 1     # pairs without a list

