"""The failure path of the tensor-core passes, on the GPU without a fault.

Their warps hand work to one another through mbarriers, and every wait is
bounded by the workspace's wait bound (moe_workspace_set_wait_limit; two
seconds by default).  With the bound set to one microsecond the epilogue warps
give up waiting for their first accumulator (a tile's k-loop takes longer), so
the call must still return, with MOE_FLAG_WAIT_TIMEOUT latched; the drains of
TMA loads and MMAs keep their full bound, so nothing is left in flight.  After
moe_workspace_init (which restores the default bound) the same workspace gives
the oracle's answer again.

The fused decode kernel reads the same bound but is not driven into a timeout
here: its abort path (consumers releasing stages whose copies an aborted wait
never saw land, the producer queueing nothing more once it sees the abort, the
exit drain) is checked by reading only."""
import numpy as np
import pytest
import torch

from int4_routed_expert_route_b200 import synthetic as syn
from layer_util import GpuLayer, OracleLayer, rel_err
from test_gpu_layer import TOL

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT = 0x8

# a small layer whose tensor-core tiles have 32 / 16 k-steps (H = 2048, I = 1024)
CFG = syn.LayerConfig("wait-limit H2048 I1024 E8 top2", H=2048, I=1024, E=8, k=2, n_group=1,
                      topk_group=1, bias_amp=0.1, T=256)


def test_tensor_path_wait_timeout_then_recovers(lib, orc):
    L = GpuLayer(lib, CFG)
    OL = OracleLayer(orc, CFG)
    T = CFG.T
    x = syn.activations(T, CFG.H, 31, "cuda")
    ws = lib.Workspace(lib.moe_layer_workspace_bytes(T, CFG.H, CFG.I, L.rcfg, lib.PATH_TENSOR))
    ws.set_wait_limit(1)
    lib.moe_layer_forward(x, L.gate, L.bias, L.rcfg, L.table, L.shared, 4, ws=ws, path=lib.PATH_TENSOR)
    torch.cuda.synchronize()
    assert ws.flags() & WAIT_TIMEOUT
    # the context is usable and the workspace recovers after re-init
    ws.reset()
    idx = torch.empty((T, CFG.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, CFG.k), dtype=torch.float32, device="cuda")
    y = lib.moe_layer_forward(x, L.gate, L.bias, L.rcfg, L.table, L.shared, 4, ws=ws, idx_out=idx,
                              w_out=w, path=lib.PATH_TENSOR)
    torch.cuda.synchronize()
    assert ws.flags() == 0
    sample = np.r_[0:8, T - 8:T]
    xb = syn.bf16_bits(x)[sample]
    ref = OL.layer_y(xb, idx.cpu().numpy()[sample], w.cpu().numpy()[sample])["y"]
    err = rel_err(y.cpu().numpy()[sample], ref)
    assert err <= TOL, err


def test_default_bound_does_not_fire(lib):
    """A long bound set explicitly (one second) behaves like the default."""
    L = GpuLayer(lib, CFG)
    x = syn.activations(64, CFG.H, 32, "cuda")
    ws = lib.Workspace(lib.moe_layer_workspace_bytes(64, CFG.H, CFG.I, L.rcfg, lib.PATH_TENSOR))
    ws.set_wait_limit(1_000_000)
    a = lib.moe_layer_forward(x, L.gate, L.bias, L.rcfg, L.table, L.shared, 4, ws=ws, path=lib.PATH_TENSOR)
    torch.cuda.synchronize()
    assert ws.flags() == 0
    ws.reset()
    b = lib.moe_layer_forward(x, L.gate, L.bias, L.rcfg, L.table, L.shared, 4, ws=ws, path=lib.PATH_TENSOR)
    assert torch.equal(a, b)
