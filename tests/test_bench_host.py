"""Host-side logic of bench.py that needs no GPU: the N > 1 path's
max-over-ranks timing and whole-job aggregation (world size 2 over gloo on
CPU), the workload table and the algorithmic byte count."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import moe_synth as ms


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(1.5 + rank, world, device="cpu")  # rank 1 is slower
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_aggregate_is_whole_job():
    one = bench.aggregate_gbs(1_000_000, 1, 1.0)
    assert one == pytest.approx(1.0)            # 1 MB per ms = 1 GB/s
    assert bench.aggregate_gbs(1_000_000, 8, 1.0) == pytest.approx(8.0)
    assert bench.max_over_ranks(3.0, 1) == 3.0


def test_algorithmic_bytes_q30b():
    S = ms.SHAPES["q30b"]
    total, ffn = bench.algorithmic_bytes(S, 16, 15)
    per_expert = 3 * 2048 * 768 * 2
    assert per_expert == 9_437_184
    assert ffn == 15 * per_expert + 2 * 16 * 2048 * 4
    assert total == ffn + 128 * 2048 * 4 + 128 * 4


def test_workloads_describe_real_shapes():
    for name, w in bench.WORKLOADS.items():
        desc = bench.workload_desc(w)
        S = ms.SHAPES[w["shape"]]
        assert f"d={S.d}" in desc and f"B={w['B']}" in desc, name


def test_reference_arm_other_ranks_do_nothing(capsys):
    class A:
        steps, warmup, gpus = 3, 3, 2
    bench.run_reference(A, bench.WORKLOADS["q30b_b16_oea4"], rank=1)
    assert capsys.readouterr().out == ""


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device path")
def test_every_timed_configuration_passes_host_validation():
    # each bench workload and sweep row is a valid call: the library's host
    # validation accepts it and only the (absent) device stops it
    import aware_expert_routing_moe_b200 as moe
    from aware_expert_routing_moe_b200 import Dims, Rule
    from aware_expert_routing_moe_b200 import build
    build.build()
    lib = moe.load_library()
    A = 0x10000
    rows = [(w["shape"], w["B"], w["mode"], w["k0"], w["budget"], w.get("group", 1)) for w in bench.WORKLOADS.values()]
    for shape, cfgs in bench.SWEEP.items():
        rows += [(shape, r[0], r[1], r[2], r[3], r[5] if len(r) > 5 else 1) for r in cfgs]
    for shape, B, mode, k0, budget, group in rows:
        S = ms.SHAPES[shape]
        dims = Dims(B, S.d, S.E, S.k, S.F)
        nbytes = lib.moe_workspace_bytes(dims)
        assert nbytes > 0, (shape, B)
        st = lib.moe_layer_decode(A, A, A, A, A, A, dims, Rule(mode, k0, budget, group), A, None, None, None, A,
                                  nbytes, None)
        assert st == 5, (shape, B, mode, k0, budget, group, st)    # MOE_ERR_CUDA: validation passed


def test_channel_bytes_match_the_oracle_sector_count(oracle_lib):
    # bench.py counts the channel path's weight bytes itself (the timed code
    # may not call the oracle); it must agree with the oracle's sector count
    import bench
    rng = np.random.default_rng(5)
    B, k, E, d, F = 3, 4, 10, 256, 128
    sel = rng.integers(-1, E, size=(B, k)).astype(np.int32)
    keep = (rng.random((B, k, F)) < 0.2).astype(np.uint8)
    keep[sel < 0] = 0
    bits = np.packbits(keep, axis=-1, bitorder="little").view(np.uint32)
    got = bench.channel_bytes(bits, sel, d, F, B, k) - (B * k * F * 4 + 2 * B * d * 4)
    assert got == oracle_lib.channel_sector_bytes(keep, sel, E, d, down_channel_major=True)


def test_recorded_layer_traffic_matches_the_algorithmic_bytes():
    # Each ncu traffic entry of the fused layer kernel (DRAM bytes read +
    # written per launch, from the capture of that workload) must cover the
    # call's algorithmic bytes and exceed them by at most 3 %: every
    # activated expert's weights read once, the rest small writes (y, H,
    # logits, the selection's outputs).  The activated count comes from the
    # oracle's routing of the workload's own seeded inputs.
    import oracle
    checked = 0
    for name, traffic in bench.NCU_TRAFFIC.items():
        w = bench.WORKLOADS[name]
        if "channels" in w:
            continue  # sector-counted bytes, checked against the oracle above
        S = ms.SHAPES[w["shape"]]
        L = ms.make_weights(S, 0, experts=False)
        x = ms.make_tokens(S, w["B"], 0, kind=w.get("kind", "normal"))
        logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
        sel, wt = oracle.reselect(logits, probs, S.k, w["mode"], w["k0"], w["budget"], w.get("group", 1))
        n_active = oracle.lists(sel, wt, S.E)["n_active"]
        total, _ = bench.algorithmic_bytes(S, w["B"], n_active)
        assert total <= traffic <= 1.03 * total, (name, n_active, total, traffic)
        checked += 1
    assert checked >= 1
