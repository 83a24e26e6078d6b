"""GPU parity of the router (step 1) and the permutation (step 2) in isolation."""
import numpy as np
import pytest

import oracle
from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs

pytestmark = pytest.mark.gpu


def _route(cfg, x, w_r, bias):
    import torch
    from gpu_util import dev, ensure_built, host, shape_of, workspace
    ensure_built()
    s = shape_of(cfg)
    T = x.shape[0]
    ws = workspace(s, T)
    idx = torch.empty((T, cfg.top_k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, cfg.top_k), dtype=torch.float32, device="cuda")
    lg = torch.empty((T, cfg.num_experts), dtype=torch.float32, device="cuda")
    F.ft_moe_route(s, T, dev(x), dev(w_r), dev(bias), idx, gw, lg, ws)
    F.ft_moe_check(ws)
    return host(idx, np.int32), host(gw, np.float32), host(lg, np.float32)


# T <= 32: decode router; 32 < T: tensor-core router, split K across CTAs while the grid is
# under one wave (T = 9700: 76 token tiles, no split), ragged last tile everywhere
@pytest.mark.parametrize("E,k,T", [(8, 2, 1), (8, 2, 64), (8, 8, 40), (128, 8, 16), (128, 8, 100), (256, 6, 8),
                                   (256, 6, 333), (96, 3, 50), (8, 2, 9700), (40, 4, 2000)])
def test_route_matches_oracle_with_ties(E, k, T):
    from gpu_util import logits_bound
    cfg = inputs.custom_config(hidden=512, ffn=64, num_experts=E, top_k=k, config_id=60)
    w_r, _ = inputs.make_router(cfg, seed=1)
    w_r[5] = w_r[2]                      # experts 2 and 5 always tie: the lower index must win
    w_r[E - 1] = w_r[0]
    bias = inputs.zipf_bias(1, 60, E)
    bias[5] = bias[2]
    bias[E - 1] = bias[0]
    x = inputs.make_tokens(cfg, T, seed=1)
    idx, gw, lg = _route(cfg, x, w_r, bias)
    assert np.array_equal(lg[:, 2], lg[:, 5])
    oidx, og = oracle.topk(lg, k)
    assert np.array_equal(idx, oidx)
    assert np.max(np.abs(gw - og)) <= 2e-6
    assert np.all(np.abs(gw.sum(1) - 1) <= 1e-6)
    l64, ad = oracle.router_logits(x, w_r, bias, with_absdot=True)
    assert np.all(np.abs(lg - l64) <= logits_bound(ad, bias, cfg.hidden))


def test_route_without_logits_output():
    import torch
    from gpu_util import dev, ensure_built, host, shape_of, workspace
    ensure_built()
    cfg = inputs.CONFIGS["tiny"]
    w_r, _ = inputs.make_router(cfg)
    x = inputs.make_tokens(cfg, 64)
    idx_ref, _, lg = _route(cfg, x, w_r, None)
    s = shape_of(cfg)
    ws = workspace(s, 64)
    idx = torch.empty((64, 2), dtype=torch.int32, device="cuda")
    gw = torch.empty((64, 2), dtype=torch.float32, device="cuda")
    F.ft_moe_route(s, 64, dev(x), dev(w_r), None, idx, gw, None, ws)
    assert np.array_equal(host(idx, np.int32), idx_ref)


def _permute(E, k, S, idx, H=256):
    import torch
    from gpu_util import dev, ensure_built, host, workspace
    ensure_built()
    T = idx.shape[0]
    s = F.make_shape(H, 64, E, k, S)
    R = T * k + (T if S else 0)
    G = E + (1 if S else 0)
    ws = workspace(s, T)
    x = inputs.make_tokens(inputs.custom_config(hidden=H), T, seed=2)
    off = torch.empty(G + 1, dtype=torch.int32, device="cuda")
    sf = torch.empty(max(R, 1), dtype=torch.int32, device="cuda")
    inv = torch.empty(max(R, 1), dtype=torch.int32, device="cuda")
    xs = torch.empty((max(R, 1), H), dtype=torch.int16, device="cuda")
    F.ft_moe_permute(s, T, dev(idx), dev(x), off, sf, inv, xs, ws)
    F.ft_moe_check(ws)
    return x, host(off, np.int32), host(sf, np.int32)[:R], host(inv, np.int32)[:R], host(xs, np.uint16)[:R]


@pytest.mark.parametrize("E,k,T,S", [(8, 2, 1, 0), (8, 2, 64, 0), (128, 8, 16, 0), (128, 8, 4096, 0),
                                     (256, 6, 8192, 0), (128, 8, 2048, 1), (128, 8, 1, 1), (8, 2, 513, 1),
                                     (256, 6, 170, 0)])
def test_permute_bit_exact(E, k, T, S):
    g = np.random.default_rng(E * 7 + T)
    zipf = np.exp(inputs.zipf_bias(3, 61, E).astype(np.float64))
    p = zipf / zipf.sum()
    idx = np.stack([g.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    x, off, sf, inv, xs = _permute(E, k, S, idx)
    ooff, osf, oinv = oracle.permute(idx, E, S)
    assert np.array_equal(off, ooff)
    assert np.array_equal(sf, osf)
    assert np.array_equal(inv, oinv)
    tok = np.where(osf < T * k, osf // k, osf - T * k)
    assert np.array_equal(xs, x[tok])


def test_permute_single_expert_and_duplicates():
    idx = np.full((1500, 2), 3, dtype=np.int32)     # every pair to expert 3 (duplicates inside a token)
    x, off, sf, inv, xs = _permute(8, 2, 0, idx)
    ooff, osf, oinv = oracle.permute(idx, 8, 0)
    assert np.array_equal(off, ooff) and np.array_equal(sf, osf) and np.array_equal(inv, oinv)


@pytest.mark.parametrize("T", [10, 2000])
def test_out_of_range_id_is_reported_not_written(T):
    """An id outside [0, E) is the kernel's own bounds check: the pair is dropped and
    ft_moe_check reports FT_ERR_DEVICE_CHECK."""
    import torch
    from gpu_util import dev, ensure_built, workspace
    ensure_built()
    E, k = 8, 2
    idx = np.random.default_rng(0).integers(0, E, size=(T, k)).astype(np.int32)
    idx[T // 2, 1] = E + 5
    s = F.make_shape(256, 64, E, k)
    ws = workspace(s, T)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sf = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    F.ft_moe_permute(s, T, dev(idx), None, off, sf, inv, None, ws)
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_check(ws)
    assert ei.value.status == F.FT_ERR_DEVICE_CHECK
    assert int(off[E]) == T * k - 1
    F.ft_moe_check(ws)     # the status word was cleared by the failing check
