"""GPU parity of the whole layer (route -> permute -> experts -> combine) against the
fp64 oracle, through the C ABI.  Routing is bit-exact given the GPU's fp32 logits;
outputs are within max|y - y64| <= 1e-2 max|y64| (BF16) / 3e-2 max|y64| (MXFP4)."""
import numpy as np
import pytest

import oracle
from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs

pytestmark = pytest.mark.gpu

_LAYERS = {}


def layer(name, **kw):
    from gpu_util import DevLayer, ensure_built
    ensure_built()
    key = (name, tuple(sorted(kw.items())))
    if key not in _LAYERS:
        cfg = inputs.CONFIGS[name] if name in inputs.CONFIGS else inputs.custom_config(**kw)
        _LAYERS[key] = DevLayer(cfg, inputs.make_layer(cfg, seed=0))
    return _LAYERS[key]


def full_check(L, x, n_rows=12, seed=0):
    """Whole layer on the GPU; routing compared for every token, outputs for a seeded sample of
    n_rows tokens plus, at every size, tokens covering each non-empty expert group (the first
    row of each 256-row token tile and the group's last row)."""
    from gpu_util import check_logits, check_y, group_rows, oracle_rows, run_layer, sample_rows
    y, idx, lg = run_layer(L, x)
    rows = np.union1d(sample_rows(x.shape[0], n_rows, seed),
                      group_rows(idx, L.cfg.num_experts, L.cfg.num_shared)).astype(np.int32)
    check_logits(x, L, lg, rows)
    oidx, og, y64 = oracle_rows(L, x, lg, rows)
    assert np.array_equal(idx, oidx), "routing differs from the oracle's top-k on the GPU logits"
    rel = check_y(y[rows], y64, L.cfg.wdtype, f"{L.cfg.name} T={x.shape[0]}")
    return y, idx, lg, rel


# decode batches (T <= 32): BF16 T >= 4, or T >= 2 with a shared expert, run on the tensor cores
# (qwen3_a3b 4/8/16/32, gemma4_26b_a4b 2/16, tiny 8), smaller ones on the GEMVs (qwen3_a3b 1/3,
# gemma4_26b_a4b 1, tiny 1/3); MXFP4 (dsv4_flash) T >= 4 on the block-scaled tensor cores, T = 1 on
# the GEMVs (the GEMV variants for larger batches: test_mxfp4_gemv_decode below); larger T on the
# grouped GEMMs
CASES = [("tiny", 64), ("tiny", 1), ("tiny", 37), ("tiny", 8), ("tiny", 3),
         ("qwen3_a3b", 1), ("qwen3_a3b", 3), ("qwen3_a3b", 4), ("qwen3_a3b", 8), ("qwen3_a3b", 16), ("qwen3_a3b", 32), ("qwen3_a3b", 4096),
         ("dsv4_flash", 1), ("dsv4_flash", 8), ("dsv4_flash", 20), ("dsv4_flash", 8192),
         ("gemma4_26b_a4b", 1), ("gemma4_26b_a4b", 2), ("gemma4_26b_a4b", 16), ("gemma4_26b_a4b", 2048)]


@pytest.mark.parametrize("name,T", CASES)
def test_layer_matches_oracle(name, T):
    L = layer(name)
    x = inputs.make_tokens(L.cfg, T, seed=0)
    full_check(L, x)


@pytest.mark.parametrize("name,T", [("tiny", 5), ("qwen3_a3b", 16), ("dsv4_flash", 8), ("gemma4_26b_a4b", 3),
                                    ("tiny", 32)])
def test_decode_and_gemm_paths_agree_at_crossover(name, T):
    from gpu_util import check_y, oracle_rows, run_layer
    L = layer(name)
    x = inputs.make_tokens(L.cfg, T, seed=3)
    y_dec, idx_dec, lg_dec = run_layer(L, x)
    prev = F.ft_set_decode_max_tokens(0)      # force the tcgen05 grouped GEMM for tiny T
    try:
        y_gem, idx_gem, lg_gem = run_layer(L, x)
    finally:
        F.ft_set_decode_max_tokens(prev)
    assert np.array_equal(idx_dec, idx_gem)
    rows = np.arange(T, dtype=np.int32)
    _, _, y64 = oracle_rows(L, x, lg_dec, rows)
    check_y(y_dec, y64, L.cfg.wdtype, "decode path")
    check_y(y_gem, y64, L.cfg.wdtype, "grouped GEMM path")


def test_just_above_threshold_uses_gemm_and_matches():
    L = layer("qwen3_a3b")
    x = inputs.make_tokens(L.cfg, F.ft_get_decode_max_tokens() + 1, seed=4)
    full_check(L, x, n_rows=33)


@pytest.mark.parametrize("wd", [inputs.WDTYPE_BF16, inputs.WDTYPE_MXFP4])
@pytest.mark.parametrize("S", [0, 1])
@pytest.mark.parametrize("T", [3, 300])
def test_small_custom_layers(wd, S, T):
    L = layer("custom", hidden=256, ffn=128, num_experts=8, top_k=2, num_shared=S, wdtype=wd,
              config_id=80 + 2 * wd + S)
    x = inputs.make_tokens(L.cfg, T, seed=5)
    full_check(L, x, n_rows=T)


@pytest.mark.parametrize("S", [0, 1])
@pytest.mark.parametrize("T", [3, 300, 1100])
def test_mxfp4_cta_pair_gemm_shapes(S, T):
    """MXFP4 layers whose gate/up (K = 1024) and down (K = 512) GEMMs both run on the CTA-pair
    kernel with TMA-streamed codes: routed and shared groups, ragged token tiles, groups of
    more than 256 rows (T = 1100), and a decode-sized batch forced onto the grouped GEMM."""
    L = layer("custom", hidden=1024, ffn=512, num_experts=8, top_k=2, num_shared=S, wdtype=inputs.WDTYPE_MXFP4,
              config_id=60 + S)
    x = inputs.make_tokens(L.cfg, T, seed=9)
    prev = F.ft_set_decode_max_tokens(0) if T <= 32 else None
    try:
        full_check(L, x, n_rows=min(T, 48))
    finally:
        if prev is not None:
            F.ft_set_decode_max_tokens(prev)


@pytest.mark.parametrize("S", [0, 1])
def test_cta_pair_gemm_shapes(S):
    """Long-K BF16 gate/up with F a multiple of 256 runs on CTA pairs: routed and shared groups,
    ragged token tiles."""
    L = layer("custom", hidden=1536, ffn=256, num_experts=8, top_k=2, num_shared=S, config_id=70 + S)
    x = inputs.make_tokens(L.cfg, 300, seed=8)
    full_check(L, x, n_rows=40)


def test_all_experts_selected_k_equals_E():
    L = layer("custom", hidden=128, ffn=64, num_experts=4, top_k=4, config_id=90)
    x = inputs.make_tokens(L.cfg, 50, seed=6)
    full_check(L, x, n_rows=50)


@pytest.mark.parametrize("T,hidden,ffn,wd", [(700, 256, 128, 0), (9, 256, 128, 0), (700, 1536, 512, 0),
                                            (700, 1024, 512, 1)])
def test_skewed_routing_multi_tile_and_empty_groups(T, hidden, ffn, wd):
    """A bias sends every token to experts 3 and 5: two groups of T rows (several 256-row
    tiles on the GEMM path), six empty groups; hidden 1536 takes the CTA-pair BF16 gate/up
    GEMM, the MXFP4 case (hidden 1024, ffn 512) the CTA-pair MXFP4 GEMMs."""
    from gpu_util import DevLayer, ensure_built
    ensure_built()
    cfg = inputs.custom_config(hidden=hidden, ffn=ffn, num_experts=8, top_k=2, wdtype=wd, config_id=91 + wd)
    d = inputs.make_layer(cfg, seed=7)
    d["bias"] = np.zeros(8, np.float32)
    d["bias"][[3, 5]] = 50.0
    L = DevLayer(cfg, d)
    x = inputs.make_tokens(cfg, T, seed=7)
    y, idx, lg, _ = full_check(L, x, n_rows=24)
    assert set(np.unique(idx)) == {3, 5}


def test_deterministic_and_stepwise_equals_fused():
    import torch
    from gpu_util import dev, host, run_layer, workspace
    L = layer("qwen3_a3b")
    T = 4096
    x = inputs.make_tokens(L.cfg, T, seed=8)
    y1, i1, l1 = run_layer(L, x)
    y2, i2, l2 = run_layer(L, x)
    assert np.array_equal(y1, y2) and np.array_equal(i1, i2) and np.array_equal(l1, l2)
    # step by step through the public entry points
    cfg, s = L.cfg, L.shape
    k, H, E, F_ = cfg.top_k, cfg.hidden, cfg.num_experts, cfg.ffn
    R = T * k
    ws = workspace(s, T)
    xd = dev(x)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sf = torch.empty(R, dtype=torch.int32, device="cuda")
    inv = torch.empty(R, dtype=torch.int32, device="cuda")
    xs = torch.empty((R, H), dtype=torch.int16, device="cuda")
    h = torch.empty((R, F_), dtype=torch.int16, device="cuda")
    o = torch.empty((R, H), dtype=torch.int16, device="cuda")
    o2 = torch.empty((R, H), dtype=torch.int16, device="cuda")
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    F.ft_moe_route(s, T, xd, L.t["w_router"], L.t.get("bias"), idx, gw, None, ws)
    F.ft_moe_permute(s, T, idx, xd, off, sf, inv, xs, ws)
    F.ft_moe_experts(s, T, L.weights, xd, xs, off, sf, o, ws)
    F.ft_moe_experts_gateup(s, T, L.weights, xs, off, h, ws)
    F.ft_moe_experts_down(s, T, L.weights, h, off, o2, ws)
    F.ft_moe_combine(s, T, o, inv, gw, y)
    F.ft_moe_check(ws)
    assert np.array_equal(host(idx, np.int32), i1)
    assert np.array_equal(host(o, np.uint16), host(o2, np.uint16))
    assert np.array_equal(host(y, np.uint16), y1)
    # permutation outputs are the oracle's counting sort of the GPU ids, bit for bit
    ooff, osf, oinv = oracle.permute(host(idx, np.int32), E)
    assert np.array_equal(host(off, np.int32), ooff)
    assert np.array_equal(host(sf, np.int32), osf)
    assert np.array_equal(host(inv, np.int32), oinv)
    assert np.array_equal(host(xs, np.uint16), x[osf // k])
    # gates: oracle softmax over the GPU's kept logits (fp32 on the GPU vs fp64)
    _, og = oracle.topk(l1, k)
    assert np.max(np.abs(host(gw, np.float32) - og)) <= 2e-6


def test_empty_batch_is_a_noop():
    L = layer("tiny")
    F.ft_moe_layer_forward(L.shape, 0, None, None, None, L.weights, None, None, None, None, 0)


@pytest.mark.parametrize("name,T", [("qwen3_a3b", 1), ("dsv4_flash", 1), ("gemma4_26b_a4b", 1), ("qwen3_a3b", 4),
                                    ("qwen3_a3b", 8), ("gemma4_26b_a4b", 16), ("tiny", 64)])
def test_chained_layers_without_host_sync(name, T):
    """Layer calls back to back on one stream, each consuming the previous output: the
    dependent-launch overlap between calls must never let a kernel read an input before the
    kernel producing it has finished.  Equal bit for bit to the same chain run one call at a
    time with a synchronisation in between."""
    import torch
    from gpu_util import dev, host, run_layer, workspace
    L = layer(name)
    H, E, k = L.cfg.hidden, L.cfg.num_experts, L.cfg.top_k
    steps = 6
    x0 = inputs.make_tokens(L.cfg, T, seed=11)
    # reference: one call at a time
    ref = []
    x = x0
    for _ in range(steps):
        y, _, _ = run_layer(L, x)
        ref.append(y)
        x = y
    # chained: no synchronisation between the calls
    ws = workspace(L.shape, T)
    bufs = [dev(x0)] + [torch.empty((T, H), dtype=torch.int16, device="cuda") for _ in range(steps)]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    for s in range(steps):
        F.ft_moe_layer_forward(L.shape, T, bufs[s], L.t["w_router"], L.t.get("bias"), L.weights, bufs[s + 1], idx,
                               None, ws)
    F.ft_moe_check(ws)
    for s in range(steps):
        assert np.array_equal(host(bufs[s + 1], np.uint16), ref[s]), f"step {s} differs"


@pytest.fixture
def block_scaled_decode():
    prev = F.ft_set_block_scaled_decode(1)
    try:
        yield
    finally:
        assert F.ft_set_block_scaled_decode(prev) == 1


@pytest.mark.parametrize("name,T,kw", [("dsv4_flash", 1, {}), ("dsv4_flash", 8, {}), ("dsv4_flash", 16, {}),
                                       ("dsv4_flash", 20, {}), ("dsv4_flash", 32, {}),
                                       # few gate/up items: some CTAs start on down items and wait
                                       # for other CTAs' gate/up epilogues
                                       ("custom", 4, dict(hidden=512, ffn=512, num_experts=4, top_k=1,
                                                          num_shared=0, wdtype=inputs.WDTYPE_MXFP4, config_id=92)),
                                       ("custom", 13, dict(hidden=1024, ffn=512, num_experts=16, top_k=4,
                                                           num_shared=0, wdtype=inputs.WDTYPE_MXFP4, config_id=83)),
                                       # FFN 4096: one activation-scale buffer in TMEM for down, a
                                       # single weight-atom buffer, and runs of items that cross groups
                                       ("custom", 12, dict(hidden=1024, ffn=4096, num_experts=24, top_k=4,
                                                           num_shared=0, wdtype=inputs.WDTYPE_MXFP4, config_id=91))])
def test_block_scaled_mxfp4_decode_matches_oracle(block_scaled_decode, name, T, kw):
    """MXFP4 decode on tcgen05.mma.kind::mxf8f6f4.block_scale (E2M1 weights with their E8M0
    scales read as stored, activations as two E4M3 planes): every token checked against the
    fp64 oracle within the MXFP4 tolerance, routing bit-exact."""
    L = layer(name, **kw)
    x = inputs.make_tokens(L.cfg, T, seed=5)
    _, _, _, rel = full_check(L, x, n_rows=T)
    assert rel < 1e-2, f"two-plane activations should stay well inside the MXFP4 bound, got {rel:.2e}"


def test_block_scaled_decode_chained_is_deterministic(block_scaled_decode):
    """Back-to-back block-scaled decode calls (ticketed combine, dependent launches) equal the
    same chain run one call at a time."""
    import torch
    from gpu_util import dev, host, run_layer, workspace
    L = layer("dsv4_flash")
    T, H, k = 8, L.cfg.hidden, L.cfg.top_k
    x0 = inputs.make_tokens(L.cfg, T, seed=12)
    ref, x = [], x0
    for _ in range(4):
        y, _, _ = run_layer(L, x)
        ref.append(y)
        x = y
    ws = workspace(L.shape, T)
    bufs = [dev(x0)] + [torch.empty((T, H), dtype=torch.int16, device="cuda") for _ in range(4)]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    for s in range(4):
        F.ft_moe_layer_forward(L.shape, T, bufs[s], L.t["w_router"], L.t.get("bias"), L.weights, bufs[s + 1], idx,
                               None, ws)
    F.ft_moe_check(ws)
    for s in range(4):
        assert np.array_equal(host(bufs[s + 1], np.uint16), ref[s]), f"step {s} differs"


@pytest.mark.parametrize("T", [4, 8, 20, 32])
def test_mxfp4_gemv_decode_matches_oracle(T):
    """The MXFP4 GEMV decode kept for batches the block-scaled path does not take (block-scaled
    decode switched off): T = 20 and 32 exceed 64 KB of x rows and take the variant that stages
    each group's rows per batch."""
    prev = F.ft_set_block_scaled_decode(0)
    try:
        L = layer("dsv4_flash")
        x = inputs.make_tokens(L.cfg, T, seed=6)
        full_check(L, x, n_rows=T)
    finally:
        assert F.ft_set_block_scaled_decode(prev) == 0
