"""Host-side logic of bench.py, on the CPU: work accounting, the weak-scaling
aggregate over ranks (2 gloo ranks), clock-record rejection, and the staleness
check of committed profile figures."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench


def brute_visible_pairs(Tq, S, start):
    i = np.arange(Tq)[:, None] + start
    j = np.arange(S)[None, :]
    return int((j <= i).sum())


@pytest.mark.parametrize("Tq,S,start", [(16, 16, 0), (7, 30, 23), (1, 9, 8), (5, 12, 3)])
def test_visible_pairs_match_a_mask_count(Tq, S, start):
    w = dict(kind="cached", Tnew=Tq, S=S, start=start)
    assert bench.visible_pairs(w) == brute_visible_pairs(Tq, S, start)


@pytest.mark.parametrize("Tq,S,start,win", [(16, 16, 0, 4), (7, 30, 23, 10), (40, 40, 0, 64)])
def test_windowed_visible_pairs_match_a_mask_count(Tq, S, start, win):
    w = dict(kind="cached", Tnew=Tq, S=S, start=start, window=win)
    i = np.arange(Tq)[:, None] + start
    j = np.arange(S)[None, :]
    assert bench.visible_pairs(w) == int(((j <= i) & (j > i - win)).sum())


def test_workload_work_figures():
    W = bench.WORKLOADS
    # 4*d FLOPs per visible pair per query head
    assert bench.algorithmic_flops(W["bitnet3b_mha_prefill_bf16"]) == 4 * 80 * 32 * 2048 * 2049 // 2
    assert bench.algorithmic_flops(W["gqa16x8_prefill_bf16"]) == 4 * 128 * 8 * 16 * 4096 * 4097 // 2
    pairs = sum(3584 + i + 1 for i in range(512))
    assert pairs == 1966336
    assert bench.algorithmic_flops(W["mqa_chunked_prefill_f16"]) == 4 * 128 * 32 * 8 * pairs
    # decode: K + V once per K/V head, plus Q and O
    assert bench.algorithmic_bytes(W["gqa_decode_bf16"]) == 2148532224
    assert bench.bound(W["gqa_decode_bf16"]) == "hbm"
    assert bench.bound(W["mqa_chunked_prefill_f16"]) == "tensor"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    ctx = bench.DistCtx(backend="gloo")
    ctx.barrier()
    slowest = ctx.max(1.0 + rank)       # rank 1 is the slow one: 2.0 ms
    results[rank] = (slowest, bench.whole_job_value(ctx.world, 21.0, slowest))
    ctx.close()


def test_two_ranks_take_the_slowest_rank():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        for rank in range(world):
            slowest, value = results[rank]
            assert slowest == 2.0
            assert value == pytest.approx(2 * 21.0 / 2e-3)


def test_clock_records_are_rejected_for_thermal_or_locked_clocks():
    ok = {"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert not bench.clocks_rejected(ok)
    assert bench.clocks_rejected({**ok, "reasons": ["hw_thermal_slowdown"]})
    assert bench.clocks_rejected({"sm_mhz": 900, "sm_max_mhz": 1965, "reasons": []})
    assert not bench.clocks_rejected({"sm_mhz": 900, "sm_max_mhz": 1965,
                                      "reasons": ["sw_power_cap"]})


def test_profile_traffic_goes_stale_when_the_kernel_changes(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "transformer_attention_causal_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "prefill_tcgen05.cuh").write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    sha = bench.kernel_source_sha("tcgen05")
    prof = tmp_path / "profiles" / "tcgen05_w.md"
    prof.write_text(f"dram_bytes_per_launch: 1234\ntensor_pipe_active_pct: 45.5\n"
                    f"kernel_source_sha256_16: {sha}\n")
    got = bench.profiled("tcgen05", "w")
    assert got["dram_bytes_per_launch"] == 1234.0 and got["tensor_pipe_active_pct"] == 45.5
    assert got["source"] == "profiles/tcgen05_w.md" and "dram_throughput_pct" not in got
    w = {"kind": "prefill", "dtype": "bf16", "B": 1, "H": 2, "Hkv": 1, "T": 256, "d": 64}
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    line = bench.roofline(w, 1.0, "tcgen05", "w", peaks, "measured")
    assert line["traffic"] == 1234.0 and line["ncu"]["tensor_pipe_active_pct"] == 45.5
    (csrc / "prefill_tcgen05.cuh").write_text("kernel v2")
    assert bench.profiled("tcgen05", "w") == {}
    line = bench.roofline(w, 1.0, "tcgen05", "w", peaks, "measured")
    assert line["traffic"] is None and "ncu" not in line


def test_spread_of_per_call_times():
    s = bench.spread([5, 1, 4, 2, 3, 6, 7, 8, 9, 10])
    assert s == {"median_ms": 5.5, "p10_ms": 1, "p90_ms": 9}
    assert bench.spread([2.0]) == {"median_ms": 2.0, "p10_ms": 2.0, "p90_ms": 2.0}
    assert bench.spread([]) is None
