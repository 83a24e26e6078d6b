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

# (E, k, T, S, H), in call order: a large call with the shared group and 257 groups leaves
# the longest [chunk][group] layout in the scratch; the next large call has fewer groups, the
# one after it takes the single-warp path (R <= 1024) on top of that stale scratch; H = 4096
# rows take the one-warp-per-row gather.
CASES = [(256, 6, 8192, 1, 256), (128, 8, 4096, 0, 256), (8, 2, 5, 1, 256), (256, 6, 600, 0, 4096),
         (128, 8, 2048, 1, 256), (8, 2, 700, 0, 256)]


def _routing(E, k, T, seed):
    g = np.random.default_rng(seed)
    zipf = np.exp(inputs.zipf_bias(seed, 62, E).astype(np.float64))
    return np.stack([g.choice(E, size=k, replace=False, p=zipf / zipf.sum()) for _ in range(T)]).astype(np.int32)


def _run(E, k, T, S, H, idx, seed):
    """Workspace permute and static-scratch permute of the same routing; returns both."""
    import torch
    from gpu_util import dev, ensure_built, host, workspace
    ensure_built()
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
        ws = None
        if use_ws:
            ws = workspace(s, T)
            F.ft_moe_permute(s, T, idd, xd, off, sf, inv, xs, ws)
        else:
            F.ft_moe_permute_noalloc(s, T, idd, xd, off, sf, inv, xs)
        torch.cuda.synchronize()
        outs.append(([host(off, np.int32), host(sf, np.int32), host(inv, np.int32), host(xs, np.uint16)], ws))
    return outs


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_permute_equals_workspace_permute_on_consecutive_calls(call):
    for n, (E, k, T, S, H) in enumerate(CASES):
        seed = 10 * call + n
        (ref, _), (got, _) = _run(E, k, T, S, H, _routing(E, k, T, seed), seed)
        for a, b in zip(ref, got):
            assert np.array_equal(a, b), f"case {(E, k, T, S, H)} differs"


def test_noalloc_out_of_range_id_drops_its_pair_and_the_next_call_is_exact():
    """The documented sign of an id outside [0, E): its pair is dropped, so offsets[E+S] = R - 1
    (the workspace permute drops the same pair and flags its status word); a valid call
    right after it on the same scratch is again exact."""
    from gpu_util import ensure_built
    ensure_built()
    E, k, T, S, H = 16, 2, 900, 1, 256
    idx = _routing(E, k, T, 5)
    idx[T // 3, 1] = E + 3
    (ref, ws), (got, _) = _run(E, k, T, S, H, idx, 5)
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_check(ws)
    assert ei.value.status == F.FT_ERR_DEVICE_CHECK
    R = T * k + T
    assert int(got[0][E + S]) == R - 1
    for a, b in zip(ref, got):
        assert np.array_equal(a, b)
    idx[T // 3, 1] = 0 if idx[T // 3, 0] != 0 else 1
    (ref, _), (got, _) = _run(E, k, T, S, H, idx, 6)
    assert int(got[0][E + S]) == R
    for a, b in zip(ref, got):
        assert np.array_equal(a, b)


def test_noalloc_permute_rejects_more_rows_than_its_scratch():
    from gpu_util import ensure_built
    ensure_built()
    s = F.make_shape(256, 64, 256, 8)
    with pytest.raises(F.FtError) as ei:
        F.ft_moe_permute_noalloc(s, 8193, 1 << 20, None, 1 << 20, 1 << 20, 1 << 20, None)
    assert ei.value.status == F.FT_ERR_UNSUPPORTED and "65536" in str(ei.value)
