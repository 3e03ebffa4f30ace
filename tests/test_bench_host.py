"""Host-side logic of bench.py: accounting, the multi-rank reduction (gloo,
world size 2, CPU), and the oracle reference arm's JSON line."""
import contextlib
import io
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from gated_delta_rule_67_b200.workloads import TINY_F32


def test_accounting_matches_hand_count():
    # C=64, d=128: A_kk 516096 + A_qk 532480 + W,U,A_qk V' 1597440 + inverse 83328 + state 6291456 per chunk
    assert bench.prefill_flops_per_token_head(128) == pytest.approx(9020800 / 64)
    # per token and head: q,k,g,v read + beta + o written, bf16
    assert bench.prefill_bytes(1, 1, 1, 128, 128, 2, False, False) == 1282
    assert bench.prefill_bytes(1, 0, 1, 128, 128, 2, True, True) == 2 * 128 * 128 * 4
    assert bench.decode_bytes(256, 32, 128, 128) == 256 * 32 * (2 * 65536 + 1282)
    # the prep kernel alone reads q, k, g, v and beta: 1282 B less the 256 B of o
    assert bench.prep_input_bytes(1, 1, 1, 128, 128) == 1026


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    mine = 1.5 + rank  # rank 1 is the slow one
    mx = bench.reduce_max(mine)
    val = bench.weak_scaling_value(1000.0, world, mx)
    out[rank] = (mx, val)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        mx, val = out[r]
        assert mx == 2.5
        assert val == pytest.approx(2000.0 / 2.5)


def test_reference_arm_line():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", TINY_F32.name])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_silent_on_other_ranks(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"]) == 0
    assert buf.getvalue() == ""


def test_warmup_floor():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_reference_arm_config_keys_match_ours():
    """Both arms describe the workload with the same config keys."""
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", TINY_F32.name])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["config"] == bench.bench_config(TINY_F32, 1)
    assert {"workload", "l2", "parallelism"} <= set(line["config"])


def test_hbm_fractions_flag_readings_above_the_measured_copy():
    peaks = {"hbm_gbs": 6000.0}
    assert bench.hbm_fracs(3000.0, peaks) == {"frac": 0.5, "frac_nominal": 3000.0 / bench.NOMINAL_HBM_GBS}
    assert bench.hbm_fracs(6500.0, peaks)["above_measured_peak"] is True
