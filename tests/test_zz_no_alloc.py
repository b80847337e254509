"""dv_topk_static: selection for callers that cannot allocate device memory
(for example a plugin running inside a host framework that owns all device
memory and gives it no allocator). It keeps its scratch in the library's
file-scope device array instead of a caller workspace.

Checked through the C ABI against dv_topk (the workspace version) on
consecutive calls with different sizes, up to the largest size the array
holds (16 rows of 65,536 scores): the index sets and counts must be
identical, and equal to the oracle's selection of the same scores. Collected
last so that a failure here comes after every other test has run; it also
passes alone in a fresh process.
"""

import numpy as np
import pytest
import torch

from oracle import dejavu_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from attention_predictor_gemv_b200 import binding as bd


def _with_workspace(scores, k, mode, tau):
    B, n = scores.shape
    idx = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = bd.workspace(bd.DV_OP_TOPK, bd.dims(B=B, N=n, k_max=min(n, max(k, 0))))
    bd.dv_topk(scores, k, idx, cnt, ws, tau=tau, mode=mode)
    torch.cuda.synchronize()
    return idx[: int(cnt.item())].cpu().numpy(), int(cnt.item())


def _static(scores, k, mode, tau):
    B, n = scores.shape
    idx = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    bd.dv_topk_static(scores, k, idx, cnt, tau=tau, mode=mode)
    torch.cuda.synchronize()
    return idx[: int(cnt.item())].cpu().numpy(), int(cnt.item())


def test_topk_static_matches_workspace_version_on_consecutive_calls():
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    cases = [
        (torch.randn(3, 5000, generator=g, device="cuda"), 123, bd.DV_TOPK, 0.0),
        (torch.randn(1, 65536, generator=g, device="cuda"), 6554, bd.DV_TOPK, 0.0),
        (torch.randn(16, 2048, generator=g, device="cuda"), 0, bd.DV_THRESHOLD, 1.5),
        # the largest accepted size: every bitmap word of the array in use
        (torch.randn(16, 65536, generator=g, device="cuda"), 3000, bd.DV_TOPK, 0.0),
        (torch.randn(16, 65536, generator=g, device="cuda"), 0, bd.DV_THRESHOLD, 2.5),
        (torch.randn(2, 777, generator=g, device="cuda"), 40, bd.DV_TOPK, 0.0),
    ]
    for scores, k, mode, tau in cases:  # consecutive calls share the one scratch array
        want_idx, want_cnt = _with_workspace(scores, k, mode, tau)
        got_idx, got_cnt = _static(scores, k, mode, tau)
        assert got_cnt == want_cnt
        assert np.array_equal(got_idx, want_idx)
        ref = O.select(scores.cpu().numpy(), k=k, tau=tau, mode="topk" if mode == bd.DV_TOPK else "threshold")
        assert np.array_equal(got_idx, ref)


def test_topk_static_rejects_sizes_beyond_its_array():
    scores = torch.zeros(1, 65537, device="cuda")
    idx = torch.zeros(65537, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(bd.DvError) as e:
        bd.dv_topk_static(scores, 10, idx, cnt)
    assert e.value.status == bd.DV_ERR_UNSUPPORTED
    rows = torch.zeros(17, 100, device="cuda")
    with pytest.raises(bd.DvError) as e:
        bd.dv_topk_static(rows, 10, idx, cnt)
    assert e.value.status == bd.DV_ERR_UNSUPPORTED
