"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/ftmoe.h declares, sizes workspaces, rejects bad arguments before any
CUDA call, and its host LRU policy matches the oracle's simulator."""
import ctypes
import random

import numpy as np
import pytest

import oracle
from expert_offload_serving_router_b200 import build as ftbuild
from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs


@pytest.fixture(scope="module", autouse=True)
def _built():
    ftbuild.build()


def test_exports_every_header_symbol():
    names = F.header_functions()
    assert len(names) >= 20
    L = ctypes.CDLL(F.LIB_PATH)
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert set(F._SIGS) == set(names)


def test_version_and_threshold():
    assert "sm_100a" in F.ft_version()
    prev = F.ft_set_decode_max_tokens(7)
    assert F.ft_get_decode_max_tokens() == 7
    assert F.ft_set_decode_max_tokens(1000) == 7 and F.ft_get_decode_max_tokens() == 32
    assert F.ft_set_decode_max_tokens(-1) == -1
    F.ft_set_decode_max_tokens(prev)


def _shape(name):
    c = inputs.CONFIGS[name]
    return F.make_shape(c.hidden, c.ffn, c.num_experts, c.top_k, c.num_shared, c.wdtype)


def test_workspace_bytes_grow_with_tokens():
    s = _shape("qwen3_a3b")
    a, b = F.ft_moe_workspace_bytes(s, 16), F.ft_moe_workspace_bytes(s, 4096)
    assert 0 < a < b
    # x_sorted + h + o_sorted dominate: R*(2H + F)*2 bytes
    R = 4096 * 8
    assert b >= R * (2 * 2048 + 768) * 2
    assert F.ft_moe_workspace_bytes(F.make_shape(100, 512, 8, 2), 4) == 0     # H % 128 != 0
    assert F.ft_moe_workspace_bytes(s, -1) == 0


FAKE = 1 << 20   # 16-byte aligned non-null address; never dereferenced (validation fails first)


@pytest.mark.parametrize("shape,code", [
    (F.make_shape(100, 512, 8, 2), F.FT_ERR_UNSUPPORTED),
    (F.make_shape(256, 500, 8, 2), F.FT_ERR_UNSUPPORTED),
    (F.make_shape(256, 512, 300, 2), F.FT_ERR_UNSUPPORTED),
    (F.make_shape(256, 512, 8, 9), F.FT_ERR_UNSUPPORTED),
    (F.make_shape(256, 512, 4, 5), F.FT_ERR_UNSUPPORTED),
    (F.make_shape(256, 512, 8, 0), F.FT_ERR_INVALID_ARG),
    (F.make_shape(256, 512, 8, 2, num_shared=2), F.FT_ERR_INVALID_ARG),
    (F.make_shape(256, 512, 8, 2, wdtype=7), F.FT_ERR_INVALID_ARG),
])
def test_bad_shapes_rejected_on_host(shape, code):
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_route(shape, 4, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 30, stream=0)
    assert ei.value.status == code


def test_bad_pointers_and_workspace_rejected_on_host():
    s = _shape("tiny")
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_route(s, 4, None, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 30, stream=0)
    assert ei.value.status == F.FT_ERR_INVALID_ARG
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_route(s, 4, FAKE + 2, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 30, stream=0)
    assert ei.value.status == F.FT_ERR_INVALID_ARG and "aligned" in str(ei.value)
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_route(s, 4, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, 64, stream=0)
    assert ei.value.status == F.FT_ERR_WORKSPACE
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_route(s, 4, FAKE, FAKE, None, FAKE, FAKE, None, FAKE + 16, 1 << 30, stream=0)
    assert ei.value.status == F.FT_ERR_INVALID_ARG
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_route(s, -1, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 30, stream=0)
    assert ei.value.status == F.FT_ERR_INVALID_ARG
    # T == 0 is a no-op that needs no pointers at all
    F.ft_moe_route(s, 0, None, None, None, None, None, None, None, 0, stream=0)
    F.ft_moe_layer_forward(s, 0, None, None, None, F.make_weights(), None, None, None, None, 0, stream=0)
    w = F.make_weights()   # NULL weights
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_layer_forward(s, 4, FAKE, FAKE, None, w, FAKE, None, None, FAKE, 1 << 30, stream=0)
    assert ei.value.status == F.FT_ERR_INVALID_ARG
    # expert_ptrs tables are decode-only
    wt = F.make_weights(expert_ptrs=FAKE)
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_layer_forward(s, 64, FAKE, FAKE, None, wt, FAKE, None, None, FAKE, 1 << 30, stream=0)
    assert ei.value.status == F.FT_ERR_UNSUPPORTED
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_unit_rms(4, 100, FAKE, FAKE, stream=0)
    assert ei.value.status == F.FT_ERR_INVALID_ARG


def test_stream_config_rejected_on_host():
    s = _shape("dsv4_flash")
    layers = (F.ft_moe_weights * 2)()
    cfg = F.ft_stream_cfg(2, 8, s, layers, FAKE * 256, 1 << 20, 1000)
    assert F.ft_expert_stream_arena_bytes(cfg) > 2 * 256 * 13_000_000
    with pytest.raises(F.FtError) as ei:          # arena too small
        F.ft_expert_stream_create(cfg)
    assert ei.value.status == F.FT_ERR_WORKSPACE
    cfg.slots_per_layer = 3                       # fewer slots than k = 6
    with pytest.raises(F.FtError) as ei:
        F.ft_expert_stream_create(cfg)
    assert ei.value.status == F.FT_ERR_INVALID_ARG
    cfg.slots_per_layer = 8
    cfg.hbm_arena_bytes = F.ft_expert_stream_arena_bytes(cfg)
    with pytest.raises(F.FtError) as ei:          # NULL host pointers
        F.ft_expert_stream_create(cfg)
    assert ei.value.status == F.FT_ERR_INVALID_ARG
    cfg.cache_policy = 2                          # not a ft_cache_policy
    with pytest.raises(F.FtError) as ei:
        F.ft_expert_stream_create(cfg)
    assert ei.value.status == F.FT_ERR_INVALID_ARG and "cache_policy" in str(ei.value)
    cfg.cache_policy = F.FT_CACHE_GLOBAL          # same arena size: the pool has L * S slots
    assert F.ft_expert_stream_arena_bytes(cfg) == cfg.hbm_arena_bytes


@pytest.mark.parametrize("seed", range(4))
def test_host_lru_policy_matches_oracle(seed):
    r = random.Random(100 + seed)
    E, n_slots = r.choice([(8, 3), (64, 8), (256, 32)])
    steps = []
    for _ in range(80):
        kk = r.randint(0, min(6, n_slots))
        steps.append(sorted(set(min(E - 1, int(r.paretovariate(0.8)) - 1 + r.randint(0, 3)) for _ in range(kk))))
    oslot, ohit, ose, h, m = oracle.lru_sim(E, n_slots, steps)
    content = np.full(n_slots, -1, np.int32)
    stamp = np.full(n_slots, -1, np.int64)
    where = np.full(E, -1, np.int32)
    for s, ids in enumerate(steps):
        ids_a = np.array(ids, np.int32)
        out_slot = np.empty(len(ids), np.int32)
        out_hit = np.empty(len(ids), np.uint8)
        F.ft_lru_step(E, n_slots, content, stamp, where, s, ids_a, out_slot, out_hit)
        assert out_slot.tolist() == oslot[s]
        assert out_hit.astype(bool).tolist() == ohit[s]
        assert content.tolist() == ose[s].tolist()


def test_host_lru_rejects_unsorted_or_oversized():
    content = np.full(2, -1, np.int32)
    stamp = np.full(2, -1, np.int64)
    where = np.full(8, -1, np.int32)
    o = np.empty(3, np.int32)
    hh = np.empty(3, np.uint8)
    with pytest.raises(F.FtError):
        F.ft_lru_step(8, 2, content, stamp, where, 0, np.array([1, 2, 3], np.int32), o, hh)
    with pytest.raises(F.FtError):
        F.ft_lru_step(8, 2, content, stamp, where, 0, np.array([2, 1], np.int32), o[:2], hh[:2])


def test_host_lru_policy_as_global_pool_matches_oracle():
    """The global cache drives ft_lru_step over keys layer * E + expert, L * S slots and one
    policy step per (decode step, layer); that must reproduce the oracle's global LRU."""
    r = random.Random(5)
    L, E, S = 3, 32, 4
    steps = 50
    routed = [[sorted(set(min(E - 1, int(r.paretovariate(0.9)) - 1 + r.randint(0, 4)) for _ in range(r.randint(1, 4))))
               for _ in range(steps)] for _ in range(L)]
    oh, om, oslots = oracle.lru_sim_global(L, E, L * S, routed)
    content = np.full(L * S, -1, np.int32)
    stamp = np.full(L * S, -1, np.int64)
    where = np.full(L * E, -1, np.int32)
    hits, misses = [0] * L, [0] * L
    for s in range(steps):
        for l in range(L):
            keys = np.array([l * E + e for e in routed[l][s]], np.int32)
            out_slot = np.empty(len(keys), np.int32)
            out_hit = np.empty(len(keys), np.uint8)
            F.ft_lru_step(L * E, L * S, content, stamp, where, s * L + l, keys, out_slot, out_hit)
            hits[l] += int(out_hit.sum())
            misses[l] += len(keys) - int(out_hit.sum())
    assert (hits, misses) == (oh, om)
    assert content.tolist() == oslots


@pytest.mark.parametrize("seed", range(6))
def test_host_lru_resize_matches_oracle(seed):
    r = random.Random(300 + seed)
    E = 64
    n_old = r.randint(1, 12)
    n_new = r.randint(1, 16)
    ids = r.sample(range(E), n_old)
    stamps = r.sample(range(1000), n_old)
    occ = [r.random() < 0.75 for _ in range(n_old)]
    content = [e if o else -1 for e, o in zip(ids, occ)]
    stamp = [t if o else -1 for t, o in zip(stamps, occ)]
    where = {e: i for i, e in enumerate(content) if e >= 0}
    oc, os_, ow = list(content), list(stamp), dict(where)
    omoves = oracle.lru_resize(oc, os_, ow, n_new)
    cap = max(n_old, n_new)
    c = np.full(cap, -1, np.int32); c[:n_old] = content
    st = np.full(cap, -1, np.int64); st[:n_old] = stamp
    w = np.full(E, -1, np.int32)
    for e, i in where.items():
        w[e] = i
    moves = F.ft_lru_resize(E, n_old, n_new, c, st, w)
    assert moves == omoves
    assert c[:n_new].tolist() == oc and st[:n_new].tolist() == os_
    assert {e: int(w[e]) for e in range(E) if w[e] >= 0} == ow


def test_stream_calls_reject_a_null_handle_on_host():
    """Every expert-stream entry point validates its handle before touching CUDA."""
    for call in (lambda: F.ft_expert_stream_set_slots(None, 8, compute_stream=0, copy_stream=0),
                 lambda: F.ft_expert_stream_reset_cache(None),
                 lambda: F.ft_expert_stream_stats(None, -1),
                 lambda: F.ft_expert_stream_slots(None, 0, 4),
                 lambda: F.ft_expert_stream_prefill_routed(None, 64, FAKE, [FAKE], None, FAKE, FAKE, FAKE, 1 << 30,
                                                           compute_stream=0, copy_stream=0)):
        with pytest.raises(F.FtError) as ei:
            call()
        assert ei.value.status == F.FT_ERR_INVALID_ARG


def test_pipeline_wait_limit_setter_round_trips():
    prev = F.ft_set_pipeline_wait_limit_ns(12345)
    assert prev == 4_000_000_000
    assert F.ft_set_pipeline_wait_limit_ns(0) == 12345          # 0 restores the default
    assert F.ft_set_pipeline_wait_limit_ns(prev) == 4_000_000_000


def test_read_probe_rejects_bad_arguments_on_host():
    for args in [(None, 1024, FAKE, 1), (FAKE + 4, 1024, FAKE, 1), (FAKE, 1000, FAKE, 1), (FAKE, 0, FAKE, 1),
                 (FAKE, 1024, None, 1), (FAKE, 1024, FAKE, 0), (FAKE, 1024, FAKE, 9)]:
        with pytest.raises(F.FtError) as ei:
            F.ft_hbm_read_probe(*args, stream=0)
        assert ei.value.status == F.FT_ERR_INVALID_ARG


def test_block_scaled_decode_switch_returns_previous_setting():
    from expert_offload_serving_router_b200 import ftmoe as F
    assert F.ft_set_block_scaled_decode(1) == 2          # default: from 4 tokens on
    assert F.ft_set_block_scaled_decode(7) == -1         # rejected, nothing changes
    assert F.ft_set_block_scaled_decode(0) == 1
    assert F.ft_set_block_scaled_decode(2) == 0


def test_tma_probe_rejects_bad_arguments_on_host():
    from expert_offload_serving_router_b200 import ftmoe as F
    for args in [(3, 4096, 1 << 30, 0, 4096), (0, 0, 1 << 30, 0, 4096), (0, 4096, 1 << 30, 0, 0), (0, 4104, 1 << 30, 0, 4096),
                 (0, 4096, 128, 0, 4096), (2, 4096, 1 << 30, 2 << 30, 4096)]:
        mode, buf, n, region, status = args
        with pytest.raises(F.FtError) as ei:
            F.ft_tma_read_probe(mode, buf, n, region, status, stream=0)
        assert ei.value.status == F.FT_ERR_INVALID_ARG


def test_decode_kernel_count_follows_the_dispatch():
    """ft_moe_decode_kernels: router + the expert kernels of the path a decode-sized layer call
    takes (host-only).  BF16: GEMVs (gate/up, down with the combine) or the tensor-core decode
    (one kernel + combine) -- three either way; MXFP4: GEMVs below 4 tokens, then the x planes +
    the fused block-scaled kernel + combine up to 16 tokens, then two projection launches and
    the h planes; nothing above the decode threshold."""
    if "FTMOE_LIB" in __import__("os").environ:
        pytest.skip("counts are for the normal build")
    qwen, gemma, dsv4 = _shape("qwen3_a3b"), _shape("gemma4_26b_a4b"), _shape("dsv4_flash")
    for T in (1, 3, 4, 16, 32):
        assert F.ft_moe_decode_kernels(qwen, T) == 3
        assert F.ft_moe_decode_kernels(gemma, T) == 3
    assert [F.ft_moe_decode_kernels(dsv4, T) for T in (1, 3, 4, 8, 16, 17, 32)] == [3, 3, 4, 4, 4, 6, 6]
    wide = F.make_shape(1024, 4096, 24, 4, 0, F.FT_W_MXFP4)        # FFN > 2048: two launches
    assert F.ft_moe_decode_kernels(wide, 8) == 6
    assert F.ft_moe_decode_kernels(dsv4, 0) == 0 and F.ft_moe_decode_kernels(dsv4, 33) == 0
    assert F.ft_moe_decode_kernels(dsv4, -1) == -1
    assert F.ft_moe_decode_kernels(F.make_shape(1000, 768, 128, 8), 4) == -1   # invalid shape
    prev = F.ft_set_block_scaled_decode(0)
    try:
        assert F.ft_moe_decode_kernels(dsv4, 8) == 3                # GEMVs only
        F.ft_set_block_scaled_decode(1)
        assert F.ft_moe_decode_kernels(dsv4, 1) == 4                # block-scaled at every size
    finally:
        F.ft_set_block_scaled_decode(prev)
    prev_max = F.ft_set_decode_max_tokens(8)
    try:
        assert F.ft_moe_decode_kernels(qwen, 8) == 3 and F.ft_moe_decode_kernels(qwen, 9) == 0
    finally:
        F.ft_set_decode_max_tokens(prev_max)
