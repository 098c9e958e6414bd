"""moe_permute_noalloc: the permutation without a caller workspace.

For callers that cannot allocate device memory (a plug-in inside a runtime
that owns all device memory, or a path where cudaMalloc's implicit device
synchronisation is not allowed), the entry point keeps its scratch in a
fixed array inside the library.  Its results must equal moe_permute's
(which takes a caller workspace) on the same inputs - bit for bit, as all
permutation results are - and stay right on consecutive calls that reuse the
same scratch.  This file is collected last so that a run stopping at the
first failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

from split_weight_b200 import _lib as L


def _inputs(T, k, E, H, seed, dev):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(dev).bfloat16()
    return torch.from_numpy(idx).to(dev), x


def _outputs(T, k, E, H, dev):
    rows = T * k + T
    return dict(offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
                perm_src=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
                inv_pos=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                x_perm=torch.zeros(rows, H, dtype=torch.bfloat16, device=dev))


def _run(fn_noalloc, T, k, E, H, idx, x, out, stream):
    common = (T, k, E, H, idx.data_ptr(), x.data_ptr(), L.MOE_BF16, L.MOE_BF16, 1,
              out["offsets"].data_ptr(), out["perm_src"].data_ptr(), out["inv_pos"].data_ptr(),
              out["x_perm"].data_ptr(), None)
    if fn_noalloc:
        return L.moe_permute_noalloc(*common, stream)
    ws = torch.empty(max(L.moe_permute_workspace_size(T, k, E), 16), dtype=torch.uint8,
                     device=x.device)
    rc = L.moe_permute(*common, ws.data_ptr(), ws.numel(), stream)
    torch.cuda.synchronize()
    return rc


@pytest.mark.gpu
def test_noalloc_matches_workspace_permute_on_consecutive_calls(cuda_device):
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row with different shapes: the second reuses the scratch
    # the first left behind
    for T, k, E, H, seed in [(3000, 8, 256, 256, 1), (777, 4, 96, 128, 2)]:
        idx, x = _inputs(T, k, E, H, seed, cuda_device)
        ref = _outputs(T, k, E, H, cuda_device)
        L.check(_run(False, T, k, E, H, idx, x, ref, stream))
        got = _outputs(T, k, E, H, cuda_device)
        L.check(_run(True, T, k, E, H, idx, x, got, stream))
        torch.cuda.synchronize()
        L.check(L.moe_check_device())
        for name in ("offsets", "perm_src", "inv_pos", "x_perm"):
            assert torch.equal(got[name], ref[name]), f"{name} differs (T={T}, E={E})"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 8 * ceil(T*k/2048) * E bytes > 1 MiB: refused before any GPU work
    T, k, E = 600000, 8, 256
    assert L.moe_permute_workspace_size(T, k, E) > (1 << 20)
    rc = L.moe_permute_noalloc(T, k, E, 256, 16, 16, L.MOE_BF16, L.MOE_BF16, 0, 16, 16, 16, None,
                               None, None)
    assert rc == L.MOE_ERR_WORKSPACE
    assert "built-in" in L.moe_last_error()


def test_noalloc_checks_arguments_before_any_cuda_call():
    # a bad hidden size (not a multiple of 128) is an argument error, found on
    # the host before the scratch array's address is looked up
    rc = L.moe_permute_noalloc(4, 2, 8, 100, 16, 16, L.MOE_BF16, L.MOE_BF16, 0, 16, 16, 16, None,
                               None, None)
    assert rc == L.MOE_ERR_INVALID_ARG
    rc = L.moe_permute_noalloc(4, 2, 8, 256, 16, 16, L.MOE_E4M3, L.MOE_BF16, 0, 16, 16, 16, None,
                               None, None)
    assert rc == L.MOE_ERR_UNSUPPORTED
