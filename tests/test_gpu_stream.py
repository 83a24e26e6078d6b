"""GPU tests of ft_expert_stream on a small stacked MXFP4 model: streamed results equal
the resident layer bit for bit, the slot cache follows the oracle's LRU simulation,
and a host-side injected copy failure is reported and rolled back."""
import numpy as np
import pytest

import oracle
from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs

pytestmark = pytest.mark.gpu

NL, SLOTS = 3, 4


class Stack:
    def __init__(self, wdtype=inputs.WDTYPE_MXFP4, zipf=True, cache_policy=F.FT_CACHE_PER_LAYER, cfg=None,
                 nl=NL, slots=SLOTS, config_id=None):
        import torch
        from gpu_util import DevLayer, ensure_built, shape_of
        ensure_built()
        self.cfg = cfg or inputs.custom_config(hidden=256, ffn=128, num_experts=16, top_k=2, wdtype=wdtype,
                                               zipf_bias=zipf, config_id=95)
        self.nl, self.slots = nl, slots
        self.layers = [DevLayer(self.cfg, inputs.make_layer(self.cfg, seed=0, layer=l, zipf=zipf, config_id=config_id))
                       for l in range(nl)]
        self.shape = shape_of(self.cfg)
        self.pinned = []
        hl = (F.ft_moe_weights * nl)()
        for l, L in enumerate(self.layers):
            ph = {}
            for key in ("w13", "w13_scale", "w2", "w2_scale"):
                a = L.np.get(key)
                if a is None:
                    continue
                a = np.ascontiguousarray(a)
                t = torch.empty(a.nbytes, dtype=torch.uint8, pin_memory=True)
                t.numpy()[:] = a.view(np.uint8).ravel()
                ph[key] = t
                self.pinned.append(t)
            hl[l] = F.make_weights(ph.get("w13"), ph.get("w13_scale"), ph.get("w2"), ph.get("w2_scale"))
        self.host_layers = hl
        cfg = F.ft_stream_cfg(nl, slots, self.shape, hl, None, 0, 20000, cache_policy)
        n = F.ft_expert_stream_arena_bytes(cfg)
        self.arena = torch.empty(n, dtype=torch.uint8, device="cuda")
        cfg.hbm_arena = self.arena.data_ptr()
        cfg.hbm_arena_bytes = n
        self.handle = F.ft_expert_stream_create(cfg)
        self.copy_stream = torch.cuda.Stream()

    def run(self, kind, x):
        import torch
        from gpu_util import dev, host, workspace
        T, H = x.shape
        ws = workspace(self.shape, T)
        y = torch.empty((self.nl, T, H), dtype=torch.int16, device="cuda")
        xl = torch.empty((self.nl, T, H), dtype=torch.int16, device="cuda")
        fn = {"prefill": F.ft_expert_stream_prefill, "prefill_routed": F.ft_expert_stream_prefill_routed,
              "decode": F.ft_expert_stream_decode_step}[kind]
        fn(self.handle, T, dev(x), [L.t["w_router"] for L in self.layers], [L.t.get("bias") for L in self.layers],
           y, xl, ws, copy_stream=self.copy_stream)
        F.ft_moe_check(ws)
        return host(y, np.uint16), host(xl, np.uint16)

    def close(self):
        F.ft_expert_stream_destroy(self.handle)
        self.handle = None


@pytest.fixture(scope="module")
def stack():
    s = Stack()
    yield s
    s.close()


def _resident(L, x):
    from gpu_util import run_layer
    return run_layer(L, x)


def test_prefill_streamed_equals_resident_and_oracle(stack):
    from gpu_util import check_y, oracle_rows
    T = 64
    x = inputs.make_tokens(stack.cfg, T, seed=11)
    y, xl = stack.run("prefill", x)
    assert np.array_equal(xl[0], x)
    for l, L in enumerate(stack.layers):
        yr, idx, lg = _resident(L, xl[l])
        assert np.array_equal(y[l], yr), f"layer {l}: streamed != resident"
        rows = np.arange(T, dtype=np.int32)
        _, _, y64 = oracle_rows(L, xl[l], lg, rows)
        check_y(y[l], y64, stack.cfg.wdtype, f"prefill layer {l}")
        if l + 1 < NL:   # chaining: x_{l+1} = unit_rms(y_l), within one bf16 ulp of the fp64 value
            want = oracle.unit_rms(inputs.bf16_bits_to_f32(y[l]).astype(np.float64))
            got = inputs.bf16_bits_to_f32(xl[l + 1]).astype(np.float64)
            assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-30)
    st = F.ft_expert_stream_stats(stack.handle, -1)
    assert st[4] == NL       # one full-layer copy per layer


def test_routed_only_prefill_equals_full_layer_prefill(stack):
    T = 40
    x = inputs.make_tokens(stack.cfg, T, seed=21)
    y_full, xl_full = stack.run("prefill", x)
    F.ft_expert_stream_reset_cache(stack.handle)          # zero the counters
    y_r, xl_r = stack.run("prefill_routed", x)
    assert np.array_equal(y_r, y_full) and np.array_equal(xl_r, xl_full)
    # exactly the experts each layer's router picked crossed the link
    cfg = stack.cfg
    per_expert = 3 * cfg.hidden * cfg.ffn // 2 + 3 * cfg.hidden * cfg.ffn // 32   # MXFP4 codes + scales
    for l, L in enumerate(stack.layers):
        _, idx, _ = _resident(L, xl_r[l])
        st = F.ft_expert_stream_stats(stack.handle, l)
        assert st[2] == len(set(idx.ravel().tolist())) * per_expert
        assert st[4] == 1


def test_decode_follows_oracle_lru_and_equals_resident(stack):
    F.ft_expert_stream_reset_cache(stack.handle)
    steps = 24
    routed = [[] for _ in range(NL)]
    for s in range(steps):
        x = inputs.make_tokens(stack.cfg, 1, seed=12, stream=s)
        y, xl = stack.run("decode", x)
        for l, L in enumerate(stack.layers):
            yr, idx, lg = _resident(L, xl[l])
            assert np.array_equal(y[l], yr), f"step {s} layer {l}: slot-cache result != resident"
            routed[l].append(sorted(set(idx.ravel().tolist())))
    tot_h = tot_m = 0
    for l in range(NL):
        oslot, ohit, ose, h, m = oracle.lru_sim(stack.cfg.num_experts, SLOTS, routed[l])
        st = F.ft_expert_stream_stats(stack.handle, l)
        assert (st[0], st[1], st[3]) == (h, m, steps)
        assert F.ft_expert_stream_slots(stack.handle, l, SLOTS) == ose[-1].tolist()
        tot_h += h
        tot_m += m
    assert tot_m >= NL * 2          # cold start: the first step misses
    assert tot_h > 0                # Zipf-skewed routing revisits hot experts


def test_global_cache_follows_oracle_global_lru_and_equals_resident():
    g = Stack(cache_policy=F.FT_CACHE_GLOBAL)
    try:
        steps = 24
        routed = [[] for _ in range(NL)]
        for s in range(steps):
            x = inputs.make_tokens(g.cfg, 1, seed=12, stream=s)
            y, xl = g.run("decode", x)
            for l, L in enumerate(g.layers):
                yr, idx, lg = _resident(L, xl[l])
                assert np.array_equal(y[l], yr), f"step {s} layer {l}: pooled-cache result != resident"
                routed[l].append(sorted(set(idx.ravel().tolist())))
        oh, om, oslots = oracle.lru_sim_global(NL, g.cfg.num_experts, NL * SLOTS, routed)
        for l in range(NL):
            st = F.ft_expert_stream_stats(g.handle, l)
            assert (st[0], st[1], st[3]) == (oh[l], om[l], steps)
        assert F.ft_expert_stream_slots(g.handle, -1, NL * SLOTS) == oslots
        with pytest.raises(F.FtError) as ei:      # the pool has no per-layer view
            F.ft_expert_stream_slots(g.handle, 0, SLOTS)
        assert ei.value.status == F.FT_ERR_INVALID_ARG
        F.ft_expert_stream_reset_cache(g.handle)
        assert F.ft_expert_stream_slots(g.handle, -1, NL * SLOTS) == [-1] * (NL * SLOTS)
    finally:
        g.close()


@pytest.mark.parametrize("policy", [F.FT_CACHE_PER_LAYER, F.FT_CACHE_GLOBAL])
def test_slot_budget_change_between_steps(policy):
    """Shrink the budget to the minimum (k slots per layer) and grow it back between decode
    steps: results stay equal to the resident layers, hits/misses and slot contents follow the
    oracle's resizable LRU."""
    g = Stack(cache_policy=policy)
    try:
        steps, k = 30, g.cfg.top_k
        resize = {10: k, 20: SLOTS}
        routed = [[] for _ in range(NL)]
        for s in range(steps):
            if s in resize:
                F.ft_expert_stream_set_slots(g.handle, resize[s], copy_stream=g.copy_stream)
            x = inputs.make_tokens(g.cfg, 1, seed=15, stream=s)
            y, xl = g.run("decode", x)
            for l, L in enumerate(g.layers):
                yr, idx, lg = _resident(L, xl[l])
                assert np.array_equal(y[l], yr), f"step {s} layer {l}: result after budget change != resident"
                routed[l].append(sorted(set(idx.ravel().tolist())))
        E = g.cfg.num_experts
        if policy == F.FT_CACHE_GLOBAL:
            oh, om, oc = oracle.lru_sim_global_resizable(NL, E, SLOTS, routed, resize)
            assert F.ft_expert_stream_slots(g.handle, -1, NL * SLOTS) == oc
        else:
            oh, om = [], []
            for l in range(NL):
                _, _, oc, h, m = oracle.lru_sim_resizable(E, SLOTS, routed[l], resize)
                oh.append(h)
                om.append(m)
                assert F.ft_expert_stream_slots(g.handle, l, SLOTS) == oc
        for l in range(NL):
            st = F.ft_expert_stream_stats(g.handle, l)
            assert (st[0], st[1]) == (oh[l], om[l])
        with pytest.raises(F.FtError) as ei:      # beyond what the arena holds
            F.ft_expert_stream_set_slots(g.handle, SLOTS + 1, copy_stream=g.copy_stream)
        assert ei.value.status == F.FT_ERR_INVALID_ARG
    finally:
        g.close()


def test_injected_copy_failure_is_reported_and_rolled_back(stack):
    F.ft_expert_stream_reset_cache(stack.handle)
    x0 = inputs.make_tokens(stack.cfg, 1, seed=13, stream=0)
    stack.run("decode", x0)                                # warm: every layer holds 1-2 experts
    before = [F.ft_expert_stream_slots(stack.handle, l, SLOTS) for l in range(NL)]
    stats_before = F.ft_expert_stream_stats(stack.handle, -1)
    F.ft_expert_stream_inject_copy_failure(stack.handle, 1)   # fail the very next expert copy
    failed_layer = None
    for s in range(1, 40):
        x = inputs.make_tokens(stack.cfg, 1, seed=13, stream=s)
        try:
            stack.run("decode", x)
        except F.FtError as e:
            assert e.status == F.FT_ERR_CUDA and "injected" in str(e)
            failed_layer = int(str(e).split("layer ")[1].split(":")[0])
            break
        before = [F.ft_expert_stream_slots(stack.handle, l, SLOTS) for l in range(NL)]
        stats_before = F.ft_expert_stream_stats(stack.handle, -1)
    assert failed_layer is not None, "no miss happened in 40 steps"
    after = F.ft_expert_stream_slots(stack.handle, failed_layer, SLOTS)
    # the failing copy was the first of its step: nothing was overwritten, state is as before
    assert after == before[failed_layer]
    F.ft_expert_stream_inject_copy_failure(stack.handle, 0)
    y, xl = stack.run("decode", inputs.make_tokens(stack.cfg, 1, seed=14))   # usable again
    for l, L in enumerate(stack.layers):
        yr, _, _ = _resident(L, xl[l])
        assert np.array_equal(y[l], yr)


def test_unpinned_host_memory_is_rejected():
    import torch
    from gpu_util import ensure_built
    ensure_built()
    cfg = inputs.custom_config(hidden=256, ffn=128, num_experts=16, top_k=2, wdtype=inputs.WDTYPE_MXFP4,
                               config_id=96)
    d = inputs.make_layer(cfg)
    keep = [np.ascontiguousarray(d[k]) for k in ("w13", "w13_scale", "w2", "w2_scale")]
    hl = (F.ft_moe_weights * 1)()
    hl[0] = F.make_weights(*[a.ctypes.data for a in keep])
    s = F.make_shape(256, 128, 16, 2, 0, 1)
    c = F.ft_stream_cfg(1, 4, s, hl, None, 0, 1000)
    n = F.ft_expert_stream_arena_bytes(c)
    arena = torch.empty(n, dtype=torch.uint8, device="cuda")
    c.hbm_arena, c.hbm_arena_bytes = arena.data_ptr(), n
    with pytest.raises(F.FtError) as ei:
        F.ft_expert_stream_create(c)
    assert ei.value.status == F.FT_ERR_NOT_PINNED


def test_deepseek_v4_flash_shaped_stack_prefill_and_decode():
    """Two DeepSeek-V4-Flash-shaped MXFP4 layers (hidden 4096, FFN 2048, 256 experts, top-6,
    13.37 MB per expert, Zipf-skewed routers) served from pinned host memory with 32 HBM slots
    per layer: the full-layer-streamed 8192-token prefill and 16 single-token decode steps
    through the slot cache (256-entry pointer tables) equal the resident layers bit for bit, the
    cache follows the oracle's LRU, and sampled outputs match the fp64 oracle."""
    from gpu_util import check_y, oracle_rows, sample_rows
    st = inputs.STACK
    cfg = inputs.CONFIGS[st["layer"]]
    nl, slots = 2, st["slots_per_layer"]
    g = Stack(cfg=cfg, nl=nl, slots=slots, zipf=True, config_id=st["config_id"])
    try:
        T = st["prefill_tokens"]
        x = inputs.make_tokens(cfg, T, seed=31)
        y, xl = g.run("prefill", x)
        assert np.array_equal(xl[0], x)
        for l, L in enumerate(g.layers):
            yr, idx, lg = _resident(L, xl[l])
            assert np.array_equal(y[l], yr), f"prefill layer {l}: streamed != resident"
            rows = sample_rows(T, 8, seed=l)
            _, _, y64 = oracle_rows(L, xl[l], lg, rows)
            check_y(y[l][rows], y64, cfg.wdtype, f"stack prefill layer {l}")
        assert F.ft_expert_stream_stats(g.handle, -1)[4] == nl

        F.ft_expert_stream_reset_cache(g.handle)
        steps = 16
        routed = [[] for _ in range(nl)]
        for s in range(steps):
            xd = inputs.make_tokens(cfg, 1, seed=32, stream=s)
            y, xl = g.run("decode", xd)
            for l, L in enumerate(g.layers):
                yr, idx, lg = _resident(L, xl[l])
                assert np.array_equal(y[l], yr), f"decode step {s} layer {l}: slot-cache result != resident"
                routed[l].append(sorted(set(idx.ravel().tolist())))
        per_expert = 3 * cfg.hidden * cfg.ffn // 2 + 3 * cfg.hidden * cfg.ffn // 32
        for l in range(nl):
            oslot, ohit, ose, h, m = oracle.lru_sim(cfg.num_experts, slots, routed[l])
            stl = F.ft_expert_stream_stats(g.handle, l)
            assert (stl[0], stl[1], stl[3]) == (h, m, steps)
            assert stl[2] == m * per_expert            # every miss copied one whole expert
            assert F.ft_expert_stream_slots(g.handle, l, slots) == ose[-1].tolist()
    finally:
        g.close()
