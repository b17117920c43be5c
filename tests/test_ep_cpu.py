"""Expert-parallel sharding on the CPU: the host logic of sparse_moe_ffn_gemv_b200.ep with
two gloo ranks (no GPU).

Each rank's partial routed sum is the oracle's block output with every expert outside the
rank's range switched off (its down plane zeroed): the per-expert outputs of the other
rank never enter it. The reduce-scatter of the two partial sums must give each rank the
complete routed sum of its own token shard, equal to the oracle's single-device result.
"""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from sparse_moe_ffn_gemv_b200 import ep  # noqa: E402


def test_expert_ranges_cover_every_expert_once():
    for E, world in ((256, 2), (256, 8), (384, 8), (128, 3), (6, 4), (7, 7)):
        ranges = [ep.expert_range(E, world, r) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == E
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        sizes = [e - b for b, e in ranges]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        ep.expert_range(3, 4, 0)


def test_token_shards_cover_every_token_once_with_aligned_starts():
    for T, world in ((1, 2), (5, 2), (64, 8), (4096, 8), (8192, 3), (37, 4)):
        rows = ep.shard_rows(T, world)
        assert rows % 8 == 0 and rows * world >= T
        spans = [ep.token_range(T, world, r) for r in range(world)]
        covered = np.zeros(T, dtype=int)
        for t0, t1 in spans:
            assert t0 % 8 == 0 or t0 == T
            covered[t0:t1] += 1
        assert np.all(covered == 1)


def test_local_weights_cut_only_the_routed_planes():
    import torch
    w = {"router_w": torch.zeros(6, 4), "gate_w": torch.arange(6 * 2 * 4).reshape(6, 2, 4),
         "down_s": torch.arange(6 * 3).reshape(6, 3), "shared_gate_w": torch.ones(5, 4)}
    lw = ep.local_weights(w, 2, 5)
    assert lw["router_w"] is w["router_w"] and lw["shared_gate_w"] is w["shared_gate_w"]
    assert torch.equal(lw["gate_w"], w["gate_w"][2:5]) and torch.equal(lw["down_s"], w["down_s"][2:5])


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import oracle
    import tiny_specs as ts
    from sparse_moe_ffn_gemv_b200 import ep as EP
    from sparse_moe_ffn_gemv_b200 import inputs
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        spec = ts.SIG_BLEND.replace(shared_mode="none", shared_intermediate=0, name="t_ep", config_id=130)
        T = 21
        w = ts.np_weights(spec)
        x = ts.np_x(spec, T)
        b, e = EP.expert_range(spec.num_experts, world, rank)
        masked = dict(w)
        down = w["down_w"].copy()
        down[:b] = 0      # bf16 zero bits: experts outside [b, e) add nothing
        down[e:] = 0
        masked["down_w"] = down
        part = oracle.forward(spec, masked, x)["y"]          # this rank's partial routed sum
        rows = EP.shard_rows(T, world)
        padded = torch.zeros((rows * world, spec.hidden), dtype=torch.float64)
        padded[:T] = torch.from_numpy(part)
        shard = EP.reduce_scatter_routed(padded, world)
        t0, t1 = EP.token_range(T, world, rank)
        full = oracle.forward(spec, w, x)["y"]
        err = float(np.abs(shard[: t1 - t0].numpy() - full[t0:t1]).max()) if t1 > t0 else 0.0
        pad = float(shard[t1 - t0:].abs().max()) if rows > t1 - t0 else 0.0
        q.put((rank, (b, e), (t0, t1), err, pad))
    finally:
        dist.destroy_process_group()


def test_reduce_scattered_partial_sums_equal_the_single_device_result_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, rg0, tk0, err0, pad0), (r1, rg1, tk1, err1, pad1) = out
    assert rg0 == (0, 3) and rg1 == (3, 6)          # six experts over two ranks
    assert tk0 == (0, 16) and tk1 == (16, 21)        # 21 tokens, shards of 16 rows
    assert err0 < 1e-12 and err1 < 1e-12             # fp64 sums of the same terms
    assert pad0 == 0.0 and pad1 == 0.0
