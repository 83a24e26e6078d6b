"""Helpers for the GPU parity tests: upload seeded inputs, call the C ABI, compare with
the fp64 oracle.  Imported only by tests marked `gpu`."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from expert_offload_serving_router_b200 import build as ftbuild
from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs

TOL = {inputs.WDTYPE_BF16: 1e-2, inputs.WDTYPE_MXFP4: 3e-2}   # max|y - y64| <= TOL * max|y64|
U32 = 2.0 ** -24


def ensure_built():
    ftbuild.build()
    F.lib()


def dev(a: np.ndarray | None) -> torch.Tensor | None:
    """numpy -> CUDA tensor with identical bytes (bf16 bits travel as int16)."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor, dtype) -> np.ndarray:
    a = t.cpu().numpy()
    return a.view(dtype) if a.dtype != dtype else a


def shape_of(cfg: inputs.LayerConfig) -> F.ft_moe_shape:
    return F.make_shape(cfg.hidden, cfg.ffn, cfg.num_experts, cfg.top_k, cfg.num_shared, cfg.wdtype)


def oshape(cfg: inputs.LayerConfig) -> dict:
    return dict(hidden=cfg.hidden, ffn=cfg.ffn, num_experts=cfg.num_experts, top_k=cfg.top_k,
                num_shared=cfg.num_shared, wdtype=cfg.wdtype)


class DevLayer:
    """One layer's weights resident on the GPU plus the structs the ABI wants."""

    def __init__(self, cfg: inputs.LayerConfig, layer: dict):
        self.cfg = cfg
        self.np = layer
        self.t = {k: dev(v) for k, v in layer.items() if v is not None}
        self.shape = shape_of(cfg)
        g = self.t.get
        self.weights = F.make_weights(g("w13"), g("w13_scale"), g("w2"), g("w2_scale"), None, g("shared_w13"),
                                      g("shared_w13_scale"), g("shared_w2"), g("shared_w2_scale"))


def workspace(shape: F.ft_moe_shape, T: int) -> torch.Tensor:
    n = F.ft_moe_workspace_bytes(shape, T)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    F.ft_moe_workspace_init(ws)
    return ws


def run_layer(L: DevLayer, x: np.ndarray, ws=None):
    """Whole-layer forward through the C ABI; returns (y bits, idx, logits) as numpy."""
    T = x.shape[0]
    H, E, k = L.cfg.hidden, L.cfg.num_experts, L.cfg.top_k
    ws = workspace(L.shape, T) if ws is None else ws
    xd = dev(x)
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    F.ft_moe_layer_forward(L.shape, T, xd, L.t["w_router"], L.t.get("bias"), L.weights, y, idx, lg, ws)
    F.ft_moe_check(ws)
    return host(y, np.uint16), host(idx, np.int32), host(lg, np.float32)


def logits_bound(absdot: np.ndarray, bias, H: int) -> np.ndarray:
    """|fl32(sum) - exact| <= gamma_{H+1} * (sum|x w| + |b|), gamma_n = n u / (1 - n u)."""
    n = H + 1
    gam = n * U32 / (1 - n * U32)
    b = 0.0 if bias is None else np.abs(bias.astype(np.float64))[None, :]
    return gam * (absdot + b)


def check_logits(x, L: DevLayer, lg_gpu: np.ndarray, rows=None):
    rows = np.arange(x.shape[0]) if rows is None else np.asarray(rows)
    l64, ad = oracle.router_logits(x[rows], L.np["w_router"], L.np.get("bias"), with_absdot=True)
    err = np.abs(lg_gpu[rows].astype(np.float64) - l64)
    bound = logits_bound(ad, L.np.get("bias"), L.cfg.hidden)
    assert np.all(err <= bound + 1e-30), f"logit error {err.max()} above fp32 dot bound {bound[err > bound].min()}"


def check_y(y_bits: np.ndarray, y64: np.ndarray, wdtype: int, what: str = ""):
    y = inputs.bf16_bits_to_f32(y_bits).astype(np.float64)
    scale = np.max(np.abs(y64))
    err = np.max(np.abs(y - y64))
    assert scale > 0
    assert err <= TOL[wdtype] * scale, f"{what}: max|y-y64| = {err:.3e} > {TOL[wdtype]} * {scale:.3e}"
    return err / scale


def oracle_rows(L: DevLayer, x, lg_gpu, rows):
    """Oracle routing from the GPU's fp32 logits, oracle y (fp64) for the listed rows."""
    idx, g = oracle.topk(lg_gpu, L.cfg.top_k)
    y64 = oracle.moe_layer(oshape(L.cfg), x, idx, g, L.np, tokens=rows)
    return idx, g, y64


def sample_rows(T: int, n: int, seed: int = 0) -> np.ndarray:
    if T <= n:
        return np.arange(T, dtype=np.int32)
    r = np.random.default_rng(seed).choice(T, size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, T - 1], r])).astype(np.int32)


def group_rows(idx: np.ndarray, num_experts: int, num_shared: int = 0, tile: int = 256) -> np.ndarray:
    """Tokens whose rows cover every non-empty expert group of the permutation the routing
    idx gives (the oracle's stable counting sort): the first row of every `tile`-row token
    tile of each group (the grouped GEMM's tiles) and the group's last row (its ragged tail).
    The shared group (S = 1) holds every token in order, so it is covered by any rows."""
    T, k = idx.shape
    offsets, sf, _ = oracle.permute(idx, num_experts, num_shared)
    picks = []
    for g in range(num_experts):
        lo, hi = int(offsets[g]), int(offsets[g + 1])
        if hi == lo:
            continue
        picks.extend(range(lo, hi, tile))
        picks.append(hi - 1)
    flat = sf[np.asarray(picks, dtype=np.int64)]
    return np.unique(np.where(flat < T * k, flat // k, flat - T * k)).astype(np.int32)
