"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test would fail on a plausible slip in the oracle: a dropped term, a wrong
sign or index, a transposed operand, a wrong expert offset, an unstable sort,
a wrong tie rule.
"""
import math
import os
import random

import numpy as np
import pytest

import oracle
from expert_offload_serving_router_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _softmax64(v):
    # library routine (scipy) as the independent reference for a full softmax
    from scipy.special import softmax
    return softmax(np.asarray(v, dtype=np.float64))


# ------------------------------------------------------------------ formats
def test_e2m1_matches_ocp_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_ocp_mx_v1.txt")) if l.strip() and not l.startswith("#")]
    assert len(rows) == 16
    for code_s, val_s in rows:
        code = int(code_s, 2)
        want = float(val_s)
        got = oracle.e2m1_to_f64(code)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (code, got, want)


def test_e8m0_all_bytes():
    v = [oracle.e8m0_to_f64(b) for b in range(256)]
    assert v[127] == 1.0
    assert v[0] == float.fromhex("0x1p-127")
    assert v[254] == float.fromhex("0x1p+127")
    for b in range(254):
        assert v[b + 1] == 2.0 * v[b]
    assert math.isnan(v[255])


def test_bf16_decode_matches_float32_view():
    g = np.random.default_rng(1)
    bits = g.integers(0, 1 << 16, size=5000, dtype=np.uint32).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # no inf/nan patterns
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = np.array([oracle.bf16_to_f64(b) for b in bits])
    assert np.array_equal(got, ref)


def test_mxfp4_matrix_packing_and_scale():
    # one row of 64 columns: byte 0 = 0x21 -> col0 code 1 (0.5), col1 code 2 (1.0);
    # byte 16 (cols 32,33) = 0xF7 -> col32 code 7 (6.0), col33 code 15 (-6.0)
    codes = np.zeros((1, 32), dtype=np.uint8)
    codes[0, 0] = 0x21
    codes[0, 16] = 0xF7
    scales = np.array([[127 + 2, 127 - 3]], dtype=np.uint8)  # block 0: x4, block 1: x1/8
    m = oracle.decode_matrix(1, codes, scales, 1, 64)
    assert m[0, 0] == 0.5 * 4 and m[0, 1] == 1.0 * 4
    assert m[0, 32] == 6.0 / 8 and m[0, 33] == -6.0 / 8
    assert np.count_nonzero(m) == 4


# ------------------------------------------------------------------ routing
def test_router_logits_vs_numpy_matmul():
    cfg = inputs.custom_config(hidden=256, num_experts=16)
    x = inputs.make_tokens(cfg, 7, seed=3)
    w, _ = inputs.make_router(cfg, seed=3)
    b = np.linspace(-1, 1, 16).astype(np.float32)
    l64, ad = oracle.router_logits(x, w, b, with_absdot=True)
    x64 = inputs.bf16_bits_to_f32(x).astype(np.float64)
    ref = x64 @ w.astype(np.float64).T + b.astype(np.float64)
    assert np.allclose(l64, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(ad, np.abs(x64) @ np.abs(w.astype(np.float64)).T, rtol=1e-12)


def _brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


@pytest.mark.parametrize("k", [1, 2, 8])
def test_topk_brute_force_with_ties(k):
    g = np.random.default_rng(k)
    T, E = 200, 8
    l = g.standard_normal((T, E)).astype(np.float32)
    # inject ties: quantise half the rows to a few levels, and +-0 pairs
    l[::2] = np.round(l[::2] * 2) / 2
    l[1::7, 3] = 0.0
    l[1::7, 5] = -0.0
    l[1::7, [0, 1, 2, 4, 6, 7]] = -1.0
    idx, gate = oracle.topk(l, k)
    for t in range(T):
        assert idx[t].tolist() == _brute_topk(l[t], k)
    # rows where -0 and +0 tie at the top pick index 3 (lower) first
    for t in range(1, T, 7):
        assert idx[t, 0] == 3 and (k == 1 or idx[t, 1] == 5)
    s = gate.sum(axis=1)
    assert np.all(np.abs(s - 1.0) <= 1e-12)
    assert np.all(np.diff(gate, axis=1) <= 1e-15)


def test_topk_full_k_is_full_softmax():
    g = np.random.default_rng(5)
    l = g.standard_normal((20, 8)).astype(np.float32) * 3
    idx, gate = oracle.topk(l, 8)
    for t in range(20):
        sm = _softmax64(l[t].astype(np.float64))
        assert np.allclose(gate[t], sm[idx[t]], rtol=1e-13, atol=1e-15)


def test_gate_equals_renormalised_full_softmax():
    # softmax over all E, keep top-k, renormalise == softmax over the k kept
    g = np.random.default_rng(6)
    l = g.standard_normal((50, 32)).astype(np.float32) * 2
    idx, gate = oracle.topk(l, 4)
    for t in range(50):
        p = _softmax64(l[t].astype(np.float64))
        sel = p[idx[t]]
        assert np.allclose(gate[t], sel / sel.sum(), rtol=1e-12)


# ------------------------------------------------------------------ permutation
@pytest.mark.parametrize("S", [0, 1])
def test_permute_invariants(S):
    g = np.random.default_rng(7 + S)
    T, k, E = 97, 3, 11
    idx = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[5] = [10, 0, 4]
    off, sf, inv = oracle.permute(idx, E, S)
    P = T * k
    n = P + (T if S else 0)
    G = E + S
    assert off[0] == 0 and off[G] == n and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.diff(off)[:E], np.bincount(idx.ravel(), minlength=E))
    assert np.array_equal(np.sort(sf), np.arange(n))
    assert np.array_equal(inv[sf], np.arange(n))
    # stable counting sort == numpy's stable argsort of the expert keys
    keys = np.concatenate([idx.ravel(), np.full(T if S else 0, E)])
    assert np.array_equal(sf, np.argsort(keys, kind="stable"))
    for e in range(G):
        seg = sf[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_permute_empty_and_single_expert():
    off, sf, inv = oracle.permute(np.zeros((0, 2), dtype=np.int32), 4)
    assert off.tolist() == [0, 0, 0, 0, 0] and len(sf) == 0
    idx = np.full((5, 1), 2, dtype=np.int32)
    off, sf, inv = oracle.permute(idx, 4)
    assert off.tolist() == [0, 0, 0, 5, 5] and sf.tolist() == list(range(5))


# ------------------------------------------------------------------ expert FFN / layer
def _dense_swiglu_np(x64, w13_64, w2_64, F):
    a = w13_64[:F] @ x64
    b = w13_64[F:] @ x64
    h = a / (1.0 + np.exp(-a)) * b
    return w2_64 @ h


def _shape(cfg):
    return dict(hidden=cfg.hidden, ffn=cfg.ffn, num_experts=cfg.num_experts, top_k=cfg.top_k,
                num_shared=cfg.num_shared, wdtype=cfg.wdtype)


@pytest.mark.parametrize("wdtype", [inputs.WDTYPE_BF16, inputs.WDTYPE_MXFP4])
def test_dense_special_case_E1_k1(wdtype):
    cfg = inputs.custom_config(hidden=128, ffn=64, num_experts=1, top_k=1, wdtype=wdtype, config_id=71)
    L = inputs.make_layer(cfg, seed=11)
    x = inputs.make_tokens(cfg, 5, seed=11)
    r = oracle.full_layer(_shape(cfg), x, L["w_router"], None, L)
    assert np.all(r["idx"] == 0) and np.all(r["g"] == 1.0)
    H, F = cfg.hidden, cfg.ffn
    w13 = oracle.decode_matrix(wdtype, L["w13"][0], None if L["w13_scale"] is None else L["w13_scale"][0], 2 * F, H)
    w2 = oracle.decode_matrix(wdtype, L["w2"][0], None if L["w2_scale"] is None else L["w2_scale"][0], H, F)
    if wdtype == inputs.WDTYPE_BF16:
        assert np.array_equal(w13, inputs.bf16_bits_to_f32(L["w13"][0]).astype(np.float64))
    x64 = inputs.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(5):
        ref = _dense_swiglu_np(x64[t], w13, w2, F)
        assert np.max(np.abs(r["y"][t] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_layer_is_gate_weighted_sum_of_dense_experts_with_shared():
    cfg = inputs.custom_config(hidden=64, ffn=32, num_experts=4, top_k=2, num_shared=1, config_id=72)
    L = inputs.make_layer(cfg, seed=12)
    x = inputs.make_tokens(cfg, 9, seed=12)
    r = oracle.full_layer(_shape(cfg), x, L["w_router"], None, L)
    x64 = inputs.bf16_bits_to_f32(x).astype(np.float64)
    H, F = cfg.hidden, cfg.ffn
    dec = lambda a: inputs.bf16_bits_to_f32(a).astype(np.float64)
    for t in range(9):
        ref = np.zeros(H)
        for j in range(2):
            e = r["idx"][t, j]
            ref += r["g"][t, j] * _dense_swiglu_np(x64[t], dec(L["w13"][e]), dec(L["w2"][e]), F)
        ref += _dense_swiglu_np(x64[t], dec(L["shared_w13"][0]), dec(L["shared_w2"][0]), F)
        assert np.max(np.abs(r["y"][t] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_zero_up_gives_zero_and_down_scaling_is_exact():
    cfg = inputs.custom_config(hidden=64, ffn=32, num_experts=4, top_k=2, config_id=73)
    L = inputs.make_layer(cfg, seed=13)
    x = inputs.make_tokens(cfg, 6, seed=13)
    base = oracle.full_layer(_shape(cfg), x, L["w_router"], None, L)
    Z = dict(L)
    w13 = L["w13"].copy()
    w13[:, cfg.ffn:, :] = 0
    Z["w13"] = w13
    z = oracle.full_layer(_shape(cfg), x, L["w_router"], None, Z)
    assert np.all(z["y"] == 0.0)
    D = dict(L)
    w2 = inputs.bf16_bits_to_f32(L["w2"]) * 2  # exact power-of-two scaling
    D["w2"] = inputs.f32_to_bf16_bits(w2)
    d = oracle.full_layer(_shape(cfg), x, L["w_router"], None, D)
    assert np.array_equal(d["y"], 2 * base["y"])


def test_token_permutation_invariance():
    cfg = inputs.custom_config(hidden=64, ffn=32, num_experts=8, top_k=2, config_id=74)
    L = inputs.make_layer(cfg, seed=14)
    x = inputs.make_tokens(cfg, 12, seed=14)
    perm = np.random.default_rng(0).permutation(12)
    a = oracle.full_layer(_shape(cfg), x, L["w_router"], None, L)
    b = oracle.full_layer(_shape(cfg), x[perm], L["w_router"], None, L)
    assert np.array_equal(a["idx"][perm], b["idx"])
    assert np.array_equal(a["g"][perm], b["g"])
    assert np.array_equal(a["y"][perm], b["y"])
    # token subsets give the same rows as the full run
    sub = oracle.moe_layer(_shape(cfg), x, a["idx"], a["g"], L, tokens=[11, 0, 5])
    assert np.array_equal(sub, a["y"][[11, 0, 5]])


def test_expert_offsets_in_stacked_mxfp4():
    # each expert's output must come from its own slice of the stacked tensors
    cfg = inputs.custom_config(hidden=64, ffn=32, num_experts=3, top_k=1, wdtype=inputs.WDTYPE_MXFP4, config_id=75)
    L = inputs.make_layer(cfg, seed=15)
    x = inputs.make_tokens(cfg, 3, seed=15)
    idx = np.array([[2], [0], [1]], dtype=np.int32)
    g = np.ones((3, 1))
    y = oracle.moe_layer(_shape(cfg), x, idx, g, L)
    x64 = inputs.bf16_bits_to_f32(x).astype(np.float64)
    for t, e in enumerate([2, 0, 1]):
        w13 = oracle.decode_matrix(1, L["w13"][e], L["w13_scale"][e], 64, 64)
        w2 = oracle.decode_matrix(1, L["w2"][e], L["w2_scale"][e], 64, 32)
        ref = _dense_swiglu_np(x64[t], w13, w2, 32)
        assert np.max(np.abs(y[t] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_unit_rms_properties():
    g = np.random.default_rng(3)
    y = g.standard_normal((4, 256)) * 50
    out = oracle.unit_rms(y)
    ms = np.mean(y * y, axis=1)
    assert np.allclose(np.mean(out * out, axis=1), ms / (ms + 1e-6), rtol=1e-12)
    assert np.allclose(oracle.unit_rms(8 * y), out, rtol=1e-9)
    assert np.all(np.sign(out) == np.sign(y))


# ------------------------------------------------------------------ LRU
def _brute_lru(E, n_slots, steps):
    """Recency-list formulation: list ordered oldest -> newest; touched ids of a
    step move to the end in ascending id order; a miss takes the lowest empty
    slot, else the slot of the oldest untouched id."""
    recency, slot_of, slots = [], {}, [-1] * n_slots
    out_slot, out_hit = [], []
    for s in steps:
        u = sorted(set(s))
        hit = [e in slot_of for e in u]
        touched = set(e for e, h in zip(u, hit) if h)
        so = []
        for e, h in zip(u, hit):
            if h:
                so.append(slot_of[e])
                continue
            if -1 in slots:
                sl = slots.index(-1)
            else:
                victim = next(v for v in recency if v not in touched)
                recency.remove(victim)
                sl = slot_of.pop(victim)
            slots[sl] = e
            slot_of[e] = sl
            touched.add(e)
            so.append(sl)
        recency = [v for v in recency if v not in u] + u
        out_slot.append(so)
        out_hit.append(hit)
    return out_slot, out_hit, slots


@pytest.mark.parametrize("seed", range(6))
def test_lru_sim_vs_brute_force(seed):
    r = random.Random(seed)
    E, n_slots = r.choice([(8, 3), (16, 5), (32, 8), (256, 32)])
    steps = []
    for _ in range(60):
        kk = r.randint(0, min(6, n_slots))
        # skewed picks so there are hits
        steps.append([min(E - 1, int(r.paretovariate(1.0)) - 1 + r.randint(0, 2)) for _ in range(kk)])
    slot, hit, se, h, m = oracle.lru_sim(E, n_slots, steps)
    bslot, bhit, bslots = _brute_lru(E, n_slots, steps)
    assert slot == bslot and hit == bhit
    assert se[-1].tolist() == bslots
    assert h == sum(sum(x) for x in bhit) and m == sum(len(x) - sum(x) for x in bhit)


def test_lru_cold_start_and_capacity_errors():
    slot, hit, se, h, m = oracle.lru_sim(8, 2, [[3, 1], [1], [5], [3]])
    assert hit == [[False, False], [True], [False], [False]]
    assert slot[0] == [1, 0] or slot[0] == [0, 1]
    with pytest.raises(ValueError):
        oracle.lru_sim(8, 2, [[1, 2, 3]])


def test_global_lru_vs_brute_force_on_the_interleaved_trace():
    r = random.Random(7)
    L, E, n_slots = 3, 16, 9
    routed = [[sorted(set(min(E - 1, int(r.paretovariate(1.0)) - 1 + r.randint(0, 3)) for _ in range(r.randint(1, 3))))
               for _ in range(40)] for _ in range(L)]
    hits, misses, slots = oracle.lru_sim_global(L, E, n_slots, routed)
    flat = [[l * E + e for e in routed[l][s]] for s in range(40) for l in range(L)]
    bslot, bhit, bslots = _brute_lru(L * E, n_slots, flat)
    for l in range(L):
        assert hits[l] == sum(sum(bhit[i]) for i in range(l, len(flat), L))
        assert misses[l] == sum(len(bhit[i]) - sum(bhit[i]) for i in range(l, len(flat), L))
    assert slots == bslots


def test_global_lru_one_layer_is_the_per_layer_cache():
    steps = [[3, 1], [1], [5], [3], [2, 5], [1, 3]]
    _, hit, se, h, m = oracle.lru_sim(8, 2, steps)
    gh, gm, gs = oracle.lru_sim_global(1, 8, 2, [steps])
    assert (gh[0], gm[0]) == (h, m) and gs == se[-1].tolist()


def test_global_lru_worked_example():
    # layer 0 cycles through experts 0, 1, 2; layer 1 always uses expert 0.  Two slots per
    # layer: layer 0's own LRU misses on every step (three ids round-robin through two
    # slots).  Pooled (4 slots): after the first three steps everything is resident.
    n = 12
    routed = [[[s % 3] for s in range(n)], [[0] for _ in range(n)]]
    ph0, pm0 = oracle.lru_sim(4, 2, routed[0])[3:5]
    ph1, pm1 = oracle.lru_sim(4, 2, routed[1])[3:5]
    assert (ph0, pm0, ph1, pm1) == (0, n, n - 1, 1)
    gh, gm, gs = oracle.lru_sim_global(2, 4, 4, routed)
    assert gm == [3, 1] and gh == [n - 3, n - 1]
    assert sorted(gs) == [0, 1, 2, 4]          # keys: layer 0 experts 0-2, layer 1 expert 0


def test_global_lru_compulsory_misses_only_when_everything_fits():
    r = random.Random(3)
    L, E = 4, 8
    routed = [[sorted(set(r.randrange(E) for _ in range(3))) for _ in range(25)] for _ in range(L)]
    distinct = [len(set(e for st in routed[l] for e in st)) for l in range(L)]
    hits, misses, _ = oracle.lru_sim_global(L, E, L * E, routed)
    assert misses == distinct
    assert [h + m for h, m in zip(hits, misses)] == [sum(len(st) for st in routed[l]) for l in range(L)]


@pytest.mark.parametrize("seed", range(4))
def test_python_lru_run_equals_c_simulator(seed):
    r = random.Random(40 + seed)
    E, n_slots = r.choice([(8, 3), (32, 8), (256, 32)])
    steps = [[min(E - 1, int(r.paretovariate(1.0)) - 1 + r.randint(0, 2)) for _ in range(r.randint(0, min(6, n_slots)))]
             for _ in range(50)]
    cslot, chit, cse, ch, cm = oracle.lru_sim(E, n_slots, steps)
    pslot, phit, pcontent, ph, pm = oracle.lru_sim_resizable(E, n_slots, steps)
    assert (pslot, phit, ph, pm) == (cslot, chit, ch, cm)
    assert pcontent == cse[-1].tolist()
    routed = [steps[i::3] for i in range(3)]
    n = min(len(x) for x in routed)
    routed = [x[:n] for x in routed]
    assert oracle.lru_sim_global_resizable(3, E, n_slots, routed)[:2] == tuple(oracle.lru_sim_global(3, E, 3 * n_slots, routed)[:2])


def test_lru_resize_worked_example():
    # four slots holding experts 7, 3, 5, 9 last used at stamps 40, 10, 30, 20; shrink to two:
    # keep the two newest (7 @ 40 in slot 0, 5 @ 30 in slot 2), drop 3 and 9, move 5 to slot 1
    content, stamp = [7, 3, 5, 9], [40, 10, 30, 20]
    where = {7: 0, 3: 1, 5: 2, 9: 3}
    assert oracle.lru_resize(content, stamp, where, 2) == [(2, 1)]
    assert content == [7, 5] and stamp == [40, 30] and where == {7: 0, 5: 1}
    # grow back to four: two empty slots, the next misses fill the lowest empty slot first
    assert oracle.lru_resize(content, stamp, where, 4) == []
    assert content == [7, 5, -1, -1]
    # a trace: step 0 puts 1, 2 in slots 0, 1; step 1 puts 5, 6 in slots 2, 3; shrinking to two
    # keeps 5 and 6 (newest) and moves them to slots 0 and 1; step 2: 6 hits, 7 replaces the
    # untouched 5; growing to three adds slot 2, which step 3's miss (5) takes
    slot, hit, final, h, m = oracle.lru_sim_resizable(16, 4, [[1, 2], [5, 6], [6, 7], [5]], {2: 2, 3: 3})
    assert slot == [[0, 1], [2, 3], [1, 0], [2]]
    assert hit == [[False, False], [False, False], [True, False], [False]]
    assert final == [7, 6, 5] and (h, m) == (1, 6)


def test_lru_resize_rejects_a_step_larger_than_the_new_budget():
    with pytest.raises(ValueError):
        oracle.lru_sim_resizable(16, 4, [[1, 2], [1, 3, 4], [4]], {1: 2})


# ---------------------------------------------------------------- NVFP4 weights (decode only)
def _e2m1_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_ocp_mx_v1.txt")) if l.strip() and not l.startswith("#")]
    return np.array([float(v) for _, v in sorted((int(c, 2), v) for c, v in rows)])


def test_e4m3_decode_matches_torch_float8_for_every_byte():
    """The oracle's E4M3 byte decode against torch's float8_e4m3fn conversion (an independent
    implementation of the OCP FP8 E4M3 format), all 256 bytes, NaN included."""
    import torch
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref)) and np.isnan(got).sum() == 2      # 0x7F, 0xFF
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x7E] == 448.0 and got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0


def test_e4m3_decode_values_are_the_rounding_grid():
    """Every finite E4M3 value is a fixed point of the oracle's E4M3 rounding (written apart from
    the decode, for the MXFP8 study), and the values between consecutive positive codes round
    to one of the two."""
    vals = sorted({oracle.e4m3_to_f64(b) for b in range(128) if b != 0x7F})
    for v in vals:
        assert oracle.e4m3_round(v) == v and oracle.e4m3_round(-v) == -v
    for a, b in zip(vals, vals[1:]):
        assert oracle.e4m3_round((a + b) / 2) in (a, b)
        assert oracle.e4m3_round(a + (b - a) / 4) == a and oracle.e4m3_round(b - (b - a) / 4) == b


def test_nvfp4_decode_matches_tables():
    """NVFP4 decode = E2M1 value (the OCP table) x E4M3 block scale (torch's conversion) x tensor
    scale, per element with the block of 16 along the row and the low nibble first; plus one
    hand-worked row."""
    import torch
    rng = np.random.default_rng(3)
    rows, cols = 5, 64
    codes = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(rows, cols // 16), dtype=np.uint8)      # positive, not NaN
    ts = np.float32(0.0625)
    e2m1 = _e2m1_golden()
    sc = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(rows, cols)
    want = e2m1[nib] * np.repeat(sc, 16, axis=1) * float(ts)
    assert np.array_equal(oracle.decode_nvfp4(codes, scales, ts, rows, cols), want)
    # row by hand: codes 0x7 (6.0) and 0xF (-6.0) alternating, block scales 1.0 (0x38) and 2^-6 (0x08)
    c1 = np.full((1, 16), 0xF7, dtype=np.uint8)
    s1 = np.array([[0x38, 0x08]], dtype=np.uint8)
    got = oracle.decode_nvfp4(c1, s1, np.float32(0.5), 1, 32)[0]
    assert np.array_equal(got[:16], np.tile([3.0, -3.0], 8))
    assert np.array_equal(got[16:], np.tile([6.0 * 2 ** -7, -6.0 * 2 ** -7], 8))
