"""moe_permute_noalloc: the dispatch for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or hand the library a workspace (a serving
process whose memory pool already owns the device, a plugin inside a framework
that owns every allocation, code with a hard latency budget).  This entry point
runs the same dispatch with its scratch in a fixed array inside the library.
The test calls it through the C ABI three times in a row, on inputs of different
shapes, and checks every output against moe_permute with a caller workspace: all outputs
are integers or copied bits, so the tolerance is exact equality.  It lives in
its own file, collected last, and passes alone or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from expert_ffn_layer_moe_b200 import moe

pytestmark = pytest.mark.gpu

MOE_ERR_UNSUPPORTED = 2


def _inputs(N, H, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(N)]).to(torch.int32)
    idx[: N // 4, 0] = E - 1                      # a hot expert, so groups are ragged
    x = torch.randn((N, H), generator=g).to(torch.bfloat16)
    return x.cuda(), idx.cuda()


def _noalloc_via_c_abi(x, idx, E):
    N, H = x.shape
    k = idx.shape[1]
    out = dict(counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
               row_to_token=torch.full((N * k,), -7, dtype=torch.int32, device="cuda"),
               token_to_row=torch.full((N, k), -7, dtype=torch.int32, device="cuda"),
               x_perm=torch.zeros((N * k, H), dtype=torch.bfloat16, device="cuda"))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = moe.lib().moe_permute_noalloc(p(x), p(idx), N, H, E, k, p(out["counts"]), p(out["offsets"]),
                                       p(out["row_to_token"]), p(out["token_to_row"]), p(out["x_perm"]),
                                       stream)
    assert rc == 0, moe.STATUS.get(rc, rc)
    return out


# Every case has more than 2048 assignments (above the one-block limit of 1024), so each
# call takes the multi-block dispatch whose per-block histograms live in the fixed array
# (smaller batches run a one-block dispatch that never touches it).  The cases change E
# and the block count from call to call, so each call starts on an array that still holds
# the previous call's histograms laid out differently: 94 blocks of 256 assignments x 128
# experts, then 12 x 16, then 41 x 200.
CALLS = ((3000, 256, 128, 8), (1500, 128, 16, 2), (2600, 64, 200, 4))


def test_noalloc_permute_matches_workspace_permute_on_consecutive_calls():
    for seed, (N, H, E, k) in enumerate(CALLS):
        assert N * k > 2048
        x, idx = _inputs(N, H, E, k, seed)
        got = _noalloc_via_c_abi(x, idx, E)
        want = moe.moe_permute(x, idx, E)
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        for name in ("counts", "offsets", "row_to_token", "token_to_row"):
            assert torch.equal(got[name], want[name]), name
        assert torch.equal(got["x_perm"].view(torch.int16), want["x_perm"].view(torch.int16))


def test_noalloc_rejects_requests_beyond_its_scratch():
    # ceil(200000*8/1024) * 256 histogram entries exceed the fixed array: refused before any launch
    null = ctypes.c_void_p(0)
    rc = moe.lib().moe_permute_noalloc(null, null, 200000, 256, 256, 8, null, null, null, null, null, null)
    assert rc == MOE_ERR_UNSUPPORTED
