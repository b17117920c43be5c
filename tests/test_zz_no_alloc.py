"""The permutation entry point that allocates nothing (GPU).

Some callers cannot allocate device memory at the point where they route tokens (a
serving loop with a fixed memory reservation, a host whose allocator is not exposed to
plug-ins, code being recorded into a CUDA graph). moe_permute_noalloc keeps its scratch
in a fixed device array inside the library. These checks compare it with moe_permute
(workspace-based) on calls in a row of different sizes: four 2048-slot chunks, then two
(the per-chunk histograms of the first call's later chunks are still in the array), then
one, so contents left in the shared array by an earlier call would show. This file runs
last in the suite.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_ffn_gemv_b200 import inputs
from sparse_moe_ffn_gemv_b200 import moe as M

pytestmark = pytest.mark.gpu


def _routing(T, k, E, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)


def _outputs(T, k, E):
    dev = dict(dtype=torch.int32, device="cuda")
    return (torch.full((E + 1,), -7, **dev), torch.full((T * k,), -7, **dev), torch.full((T * k,), -7, **dev))


def test_noalloc_permutation_matches_the_workspace_permutation_on_calls_in_a_row():
    spec = inputs.KLEAR_BF16
    cfg = M.config_from_spec(spec)
    k, E = spec.top_k, spec.num_experts
    ws = torch.zeros(M.moe_workspace_size(cfg, 1000), dtype=torch.uint8, device="cuda")
    # 1000 tokens (four 2048-slot chunks), 300 tokens (two chunks), 37 tokens (one chunk,
    # experts 64..255 empty)
    for T, seed in ((1000, 11), (300, 15), (37, 12)):
        idx = _routing(T, k, E, seed)
        if T == 37:
            idx = idx % 64                      # experts 64..255 empty on the second call
        idx_d = idx.cuda()
        ref = _outputs(T, k, E)
        M.moe_permute(cfg, idx_d, T, *ref, ws)
        got = _outputs(T, k, E)
        M.moe_permute_noalloc(cfg, idx_d, T, *got)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        o_off, o_ss, o_sp = oracle.permute(idx.numpy(), E)
        np.testing.assert_array_equal(got[0].cpu().numpy(), o_off)
        np.testing.assert_array_equal(got[1].cpu().numpy(), o_ss)
        np.testing.assert_array_equal(got[2].cpu().numpy(), o_sp)


def test_noalloc_permutation_reports_an_out_of_range_expert_id():
    spec = inputs.KLEAR_BF16
    cfg = M.config_from_spec(spec)
    T, k, E = 5, spec.top_k, spec.num_experts
    idx = _routing(T, k, E, 13)
    idx[3, 2] = 999
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _outputs(T, k, E)
    M.moe_permute_noalloc(cfg, idx.cuda(), T, *out, device_status=status)
    torch.cuda.synchronize()
    assert M.STATUS[int(status.item())] == "MOE_ERR_DEVICE_CHECK"
    assert int(out[0][-1]) == T * k - 1        # the bad slot was dropped
    # a clean call right after does not inherit the fixed array's previous contents
    out2 = _outputs(T, k, E)
    idx2 = _routing(T, k, E, 14)
    M.moe_permute_noalloc(cfg, idx2.cuda(), T, *out2)
    torch.cuda.synchronize()
    o_off, o_ss, _ = oracle.permute(idx2.numpy(), E)
    np.testing.assert_array_equal(out2[0].cpu().numpy(), o_off)
    np.testing.assert_array_equal(out2[1].cpu().numpy(), o_ss)
