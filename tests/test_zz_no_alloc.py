"""ft_moe_permute_noalloc: the permutation for callers that cannot allocate device memory
(engines that reserve HBM for their own pools, plugins handed only their buffers).  It
must give exactly what ft_moe_permute gives with a workspace, on consecutive calls that
reuse the library's one static scratch array.  This file is collected last so that a
run stopping at the first failure has already run every other test."""
import numpy as np
import pytest

from expert_offload_serving_router_b200 import ftmoe as F
from expert_offload_serving_router_b200 import inputs

pytestmark = pytest.mark.gpu

CASES = [(128, 8, 4096, 0), (8, 2, 5, 1), (256, 6, 8192, 0), (128, 8, 2048, 1), (8, 2, 700, 0)]


def _run(fn_ws, E, k, T, S, seed):
    import torch
    from gpu_util import dev, ensure_built, host, workspace
    ensure_built()
    H = 256
    g = np.random.default_rng(seed)
    zipf = np.exp(inputs.zipf_bias(seed, 62, E).astype(np.float64))
    idx = np.stack([g.choice(E, size=k, replace=False, p=zipf / zipf.sum()) for _ in range(T)]).astype(np.int32)
    x = inputs.make_tokens(inputs.custom_config(hidden=H), T, seed=seed)
    s = F.make_shape(H, 64, E, k, S)
    R, G = T * k + (T if S else 0), E + (1 if S else 0)
    idd, xd = dev(idx), dev(x)
    outs = []
    for use_ws in (True, False):
        off = torch.full((G + 1,), -1, dtype=torch.int32, device="cuda")
        sf = torch.full((R,), -1, dtype=torch.int32, device="cuda")
        inv = torch.full((R,), -1, dtype=torch.int32, device="cuda")
        xs = torch.zeros((R, H), dtype=torch.int16, device="cuda")
        if use_ws:
            ws = workspace(s, T)
            F.ft_moe_permute(s, T, idd, xd, off, sf, inv, xs, ws)
        else:
            F.ft_moe_permute_noalloc(s, T, idd, xd, off, sf, inv, xs)
        torch.cuda.synchronize()
        outs.append([host(off, np.int32), host(sf, np.int32), host(inv, np.int32), host(xs, np.uint16)])
    return outs


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_permute_equals_workspace_permute_on_consecutive_calls(call):
    for n, (E, k, T, S) in enumerate(CASES):
        ref, got = _run(None, E, k, T, S, seed=10 * call + n)
        for a, b in zip(ref, got):
            assert np.array_equal(a, b)


def test_noalloc_permute_rejects_more_rows_than_its_scratch():
    from gpu_util import ensure_built
    ensure_built()
    s = F.make_shape(256, 64, 256, 8)
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_permute_noalloc(s, 8193, 1 << 20, None, 1 << 20, 1 << 20, 1 << 20, None)
    assert ei.value.status == F.FT_ERR_UNSUPPORTED and "65536" in str(ei.value)
