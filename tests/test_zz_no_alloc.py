"""moe_route_topk_noalloc, the router entry point for callers that cannot
allocate device memory (fixed memory plans, code that must not call an
allocator): it takes its scratch from an array inside the library.  Checked
through the C ABI against moe_route_topk (which uses a caller workspace) on two
calls in a row, so the second call runs on scratch the first one left behind,
against the oracle on the same inputs, and for the property it exists for: a
call allocates no device memory.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _compare(lib, cfg, T, seed, gate, bias):
    x = syn.activations(T, cfg.H, seed, "cuda")
    rc = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf, cfg.topp)
    i1, w1, g1 = lib.moe_route_topk(x, gate, bias, rc, with_gap=True)
    i2, w2, g2 = lib.moe_route_topk_noalloc(x, gate, bias, rc, with_gap=True)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2)
    assert torch.allclose(w1, w2, rtol=2e-6, atol=0)
    assert torch.allclose(g1, g2, rtol=1e-3, atol=1e-6)
    return x, i2, w2, g2


def test_noalloc_matches_workspace_router_twice(lib):
    cfg = syn.DECODE
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    _compare(lib, cfg, 8, 501, gate, bias)   # first call (sets the scratch address up)
    _compare(lib, cfg, 3, 502, gate, bias)   # second call reuses the scratch


def test_noalloc_large_batch_and_tiny(lib):
    cfg = syn.DECODE
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    _compare(lib, cfg, 300, 503, gate, bias)
    t = syn.TINY
    _compare(lib, t, 4, 504, syn.router_gate(t, 0, "cuda"), syn.router_bias(t, 0, "cuda"))


def test_noalloc_matches_oracle(lib, orc):
    cfg = syn.DECODE
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    x, idx, w, gap = _compare(lib, cfg, 16, 505, gate, bias)
    r = orc.route(syn.bf16_bits(x), gate.cpu().numpy(), bias.cpu().numpy(), cfg.k, cfg.n_group,
                  cfg.topk_group, cfg.rsf)
    ok = np.minimum(r["gap"], r["ggap"]) >= 1e-6  # near-ties may legitimately differ
    assert np.array_equal(idx.cpu().numpy()[ok], r["idx"][ok])
    assert np.allclose(w.cpu().numpy()[ok], r["w"][ok], rtol=2e-6, atol=0)


def test_noalloc_allocates_nothing(lib):
    """After the first call (which looks the scratch address up), further calls
    change neither the free device memory nor torch's allocator."""
    cfg = syn.DECODE
    gate = syn.router_gate(cfg, 0, "cuda")
    bias = syn.router_bias(cfg, 0, "cuda")
    rc = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf, cfg.topp)
    L = lib.load()
    T = 64
    x = syn.activations(T, cfg.H, 506, "cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        st = L.moe_route_topk_noalloc(ctypes.c_void_p(x.data_ptr()), T, cfg.H,
                                      ctypes.c_void_p(gate.data_ptr()), ctypes.c_void_p(bias.data_ptr()),
                                      ctypes.byref(rc), ctypes.c_void_p(idx.data_ptr()),
                                      ctypes.c_void_p(w.data_ptr()), None, ctypes.c_void_p(stream))
        assert st == 0

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0


def test_noalloc_rejects_oversized_request(lib):
    L = lib.load()
    cfg = syn.DECODE
    rc = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf)
    limit = L.moe_route_noalloc_max_scratch_bytes()
    assert limit == 4 << 20
    T = 8192  # 8192 x 256 x 4 B of fp32 logits > 4 MiB
    assert lib.moe_route_workspace_bytes(T, cfg.H, rc) - 256 > limit
    fake = ctypes.c_void_p(0x100000)
    st = L.moe_route_topk_noalloc(fake, T, cfg.H, fake, fake, ctypes.byref(rc), fake, fake, None,
                                  None)
    assert st == 4  # MOE_ERR_WORKSPACE, returned before any launch
