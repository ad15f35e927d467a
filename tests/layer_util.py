"""Test helpers: build a layer's inputs once on the device for the CUDA library
and, from the same generator output, the oracle's own quantised copies."""
import numpy as np
import torch

from int4_routed_expert_route_b200 import synthetic as syn

FLAG_TOL = 1e-6  # decision margin under which routing is compared as valid sets


class GpuLayer:
    """All experts of one layer quantised on the device by the library."""

    def __init__(self, lib, cfg, layer=0, bits=None, device="cuda"):
        self.cfg, self.layer = cfg, layer
        self.bits = bits or cfg.bits
        self.device = device
        ex = []
        for e in range(cfg.E + 1):
            w = [syn.expert_weight(cfg, layer, e, m, device) for m in ("gate", "up", "down")]
            ex.append(lib.QuantExpert.from_fp32(*w, bits=self.bits))
            del w
        self.experts = ex[:cfg.E]
        self.shared_q = ex[cfg.E]
        self.table = lib.ExpertTable(self.experts)
        self.shared = lib.SharedExpert(self.shared_q) if cfg.shared else None
        self.gate = syn.router_gate(cfg, layer, device)
        self.bias = syn.router_bias(cfg, layer, device)
        self.rcfg = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf, cfg.topp)
        torch.cuda.synchronize()


class OracleLayer:
    """The oracle's view of the same layer: fp32 weights from the generator,
    quantised by the oracle itself, on demand."""

    def __init__(self, orc, cfg, layer=0, bits=None, device="cuda"):
        self.orc, self.cfg, self.layer = orc, cfg, layer
        self.bits = bits or cfg.bits
        self.device = device
        self.cache = {}
        self.gate = syn.router_gate(cfg, layer, device).cpu().numpy()
        self.bias = syn.router_bias(cfg, layer, device).cpu().numpy()

    def expert(self, e):
        if e not in self.cache:
            w = [syn.expert_weight(self.cfg, self.layer, e, m, self.device).cpu().numpy()
                 for m in ("gate", "up", "down")]
            q = [self.orc.quantize_rows(wi, self.bits) for wi in w]
            self.cache[e] = self.orc.Expert(q[0][0], q[0][1], q[1][0], q[1][1], q[2][0], q[2][1],
                                            self.bits)
        return self.cache[e]

    def route(self, xb):
        c = self.cfg
        return self.orc.route(xb, self.gate, self.bias, c.k, c.n_group, c.topk_group, c.rsf,
                              c.topp)

    def layer_y(self, xb, idx=None, w=None):
        c = self.cfg
        if idx is None:
            r = self.route(xb)
            idx, w = r["idx"], r["w"]
        need = sorted(set(int(e) for e in idx.reshape(-1) if e >= 0))
        experts = [self.expert(e) if e in need else None for e in range(c.E)]
        shared = self.expert(c.E) if c.shared else None
        return self.orc.layer(xb, self.gate, self.bias, experts, shared, c.H, c.I, c.k,
                              c.n_group, c.topk_group, c.rsf, c.topp, idx_in=idx, w_in=w)


def flagged(r):
    return (r["gap"] < FLAG_TOL) | (r["ggap"] < FLAG_TOL)


def routing_is_valid(scores, bias, idx, cfg, tol=FLAG_TOL):
    """A selection is valid when it is a top-k under the group rule up to
    decisions closer than tol (used for flagged tokens only): its groups, filled
    up with the best other groups, are within tol of the kept-group threshold,
    and no unchosen candidate of those groups beats a chosen expert by > tol."""
    b = scores.astype(np.float32) + bias.astype(np.float32)
    E, gs = cfg.E, cfg.E // cfg.n_group
    chosen = [int(e) for e in idx if e >= 0]
    if len(set(chosen)) != len(chosen) or any(e >= E for e in chosen):
        return False
    if cfg.n_group > 1:
        gscore = np.array([np.float32(np.sort(b[g * gs:(g + 1) * gs])[-1])
                           + np.float32(np.sort(b[g * gs:(g + 1) * gs])[-2])
                           for g in range(cfg.n_group)])
        groups = sorted(set(e // gs for e in chosen))
        if len(groups) > cfg.topk_group:
            return False
        for g in np.argsort(-gscore, kind="stable"):
            if len(groups) == cfg.topk_group:
                break
            if g not in groups:
                groups.append(int(g))
        kth = np.sort(gscore)[-cfg.topk_group]
        if any(gscore[g] < kth - tol for g in groups):
            return False
        cand = [e for e in range(E) if e // gs in groups]
    else:
        cand = list(range(E))
    rest = [float(b[e]) for e in cand if e not in chosen]
    return not rest or min(float(b[e]) for e in chosen) >= max(rest) - tol


def rel_err(y, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(np.asarray(y, np.float64) - ref)) / max(np.max(np.abs(ref)), 1e-30))
