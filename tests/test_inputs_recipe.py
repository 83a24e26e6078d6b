"""The seeded synthetic inputs follow the stated recipe: bf16 by round-to-nearest-even, N(0,1)
tokens, N(0, 0.02^2) weights and router, Zipf(1) router bias over a seeded rank permutation,
MXFP4 codes uniform over all 16 values per nibble, E8M0 scale bytes uniform on 119..123,
layouts as documented, and determinism per (seed, config, tensor, layer, expert) stream."""
import numpy as np
import torch

from expert_offload_serving_router_b200 import inputs


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    # exact halfway cases between neighbouring finite bf16 values (low 16 bits = 0x8000); the
    # generators never produce NaN or infinity, so those are left out
    hi = rng.integers(0, 0x7F7F, 4000, dtype=np.uint32) | (rng.integers(0, 2, 4000, dtype=np.uint32) << 15)
    half = (hi << 16 | 0x8000).astype(np.uint32).view(np.float32)
    a = np.concatenate([a, half, np.array([0.0, -0.0, 1.0, -1.0], np.float32)])
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(inputs.f32_to_bf16_bits(a), want)
    assert np.array_equal(inputs.bf16_bits_to_f32(want), torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_zipf_bias_is_minus_log_of_a_rank_permutation():
    b = inputs.zipf_bias(seed=0, config_id=2, num_experts=128)
    r = np.exp(-b.astype(np.float64))
    assert np.allclose(np.sort(r), np.arange(1, 129), rtol=1e-6)
    assert not np.array_equal(np.argsort(-b), np.arange(128))       # the hottest experts are scattered
    assert np.array_equal(b, inputs.zipf_bias(seed=0, config_id=2, num_experts=128))
    assert not np.array_equal(b, inputs.zipf_bias(seed=0, config_id=2, num_experts=128, layer=1))


def test_token_and_weight_distributions():
    cfg = inputs.custom_config(hidden=1024, ffn=512, num_experts=4, top_k=2, num_shared=1, config_id=60)
    x = inputs.bf16_bits_to_f32(inputs.make_tokens(cfg, 256, seed=1))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    L = inputs.make_layer(cfg, seed=1)
    assert L["w13"].shape == (4, 1024, 1024) and L["w2"].shape == (4, 1024, 512)
    assert L["shared_w13"].shape == (1, 1024, 1024) and L["shared_w2"].shape == (1, 1024, 512)
    for key in ("w13", "w2", "shared_w13"):
        w = inputs.bf16_bits_to_f32(L[key])
        assert abs(w.std() - 0.02) < 0.0005, key
    assert L["w_router"].dtype == np.float32 and abs(L["w_router"].std() - 0.02) < 0.001
    assert L["bias"] is None
    # deterministic per stream, independent across streams
    assert np.array_equal(inputs.make_tokens(cfg, 8, seed=1), inputs.make_tokens(cfg, 8, seed=1))
    assert not np.array_equal(inputs.make_tokens(cfg, 8, seed=1, stream=1), inputs.make_tokens(cfg, 8, seed=1))


def test_mxfp4_codes_and_scales():
    cfg = inputs.custom_config(hidden=1024, ffn=512, num_experts=2, top_k=1, wdtype=inputs.WDTYPE_MXFP4, config_id=61)
    L = inputs.make_layer(cfg, seed=2)
    assert L["w13"].shape == (2, 1024, 512) and L["w13_scale"].shape == (2, 1024, 32)
    assert L["w2"].shape == (2, 1024, 256) and L["w2_scale"].shape == (2, 1024, 16)
    codes = L["w13"].ravel()
    nib = np.concatenate([codes & 15, codes >> 4])
    counts = np.bincount(nib, minlength=16)
    expect = nib.size / 16
    assert np.all(np.abs(counts - expect) < 6 * np.sqrt(expect))      # all 16 codes, -0 included
    sc = np.concatenate([L["w13_scale"].ravel(), L["w2_scale"].ravel()])
    assert set(np.unique(sc).tolist()) == {119, 120, 121, 122, 123}
