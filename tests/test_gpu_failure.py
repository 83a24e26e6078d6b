"""Failure handling without a GPU fault.  The grouped-GEMM kernels bound every pipeline wait;
ft_set_pipeline_wait_limit_ns(1) makes that bound shorter than any stage, so the waits run out
and each kernel takes its give-up path: raise the CTA's abort flag, record a timeout in the
workspace status word, let its own copies and MMAs finish, free its tensor memory and return.
Nothing traps and nothing is injected on the device.  ft_moe_check must report
FT_ERR_DEVICE_CHECK, the context must stay usable, and the next call under the default bound
must be bit-identical to the same call made before the failure."""
import numpy as np
import pytest

from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs

pytestmark = pytest.mark.gpu

# which kernels give up: qwen3_a3b gate/up = BF16 CTA-pair kernel, its down = single-CTA BF16
# kernel (128-row tiles); gemma4_26b_a4b gate/up = single-CTA BF16 kernel (256-row tiles);
# dsv4_flash = the MXFP4 CTA-pair kernel (both GEMMs); the custom MXFP4 layer (K = 1280 for
# gate/up, ten 128-row groups for down) = the single-CTA MXFP4 kernel whose converter warps
# load codes from global memory
CASES = [("qwen3_a3b", 4096, None), ("gemma4_26b_a4b", 2048, None), ("dsv4_flash", 2048, None),
         ("custom", 2000, dict(hidden=1280, ffn=512, num_experts=8, top_k=2, num_shared=1,
                               wdtype=inputs.WDTYPE_MXFP4, config_id=81))]


@pytest.mark.parametrize("name,T,kw", CASES)
def test_pipeline_wait_timeout_is_reported_and_the_next_call_is_exact(name, T, kw):
    import torch
    from gpu_util import DevLayer, dev, ensure_built, host, run_layer, workspace
    ensure_built()
    cfg = inputs.CONFIGS[name] if kw is None else inputs.custom_config(**kw)
    L = DevLayer(cfg, inputs.make_layer(cfg, seed=0))
    x = inputs.make_tokens(cfg, T, seed=21)
    ws = workspace(L.shape, T)
    y_ref, idx_ref, _ = run_layer(L, x, ws)

    y = torch.empty((T, cfg.hidden), dtype=torch.int16, device="cuda")
    prev = F.ft_set_pipeline_wait_limit_ns(1)
    try:
        F.ft_moe_layer_forward(L.shape, T, dev(x), L.t["w_router"], L.t.get("bias"), L.weights, y, None, None, ws)
        with pytest.raises(F.FtError) as ei:
            F.ft_moe_check(ws)
    finally:
        assert F.ft_set_pipeline_wait_limit_ns(prev) == 1
    assert ei.value.status == F.FT_ERR_DEVICE_CHECK
    assert "timed out" in str(ei.value)
    F.ft_moe_check(ws)   # the failing check cleared the status word; no CUDA error is pending

    y2, idx2, _ = run_layer(L, x, ws)
    assert np.array_equal(idx2, idx_ref)
    assert np.array_equal(y2, y_ref), "the call after the timed-out one differs"
    torch.cuda.synchronize()
    assert host(y, np.uint16).shape == (T, cfg.hidden)
