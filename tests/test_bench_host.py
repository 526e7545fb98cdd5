"""Host-side logic of bench.py (CPU only): the max-over-ranks timing reduction
and barrier with world size 2 over gloo, clock-sample parsing, FLOP and byte
accounting, and the reference arm's JSON line and rank-0-only rule."""
import json
import os
import socket

import numpy as np
import pytest

import bench
from tiled_attention_23_b200 import synthetic as syn


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        m = bench.max_over_ranks(float(10 + 5 * rank))
        bench.barrier()
        q.put((rank, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def test_parse_clocks():
    text = "\n".join([
        "0, 1845 MHz, 1965 MHz, 700.00 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1850 MHz, 1965 MHz, 710.00 W, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1300 MHz, 1965 MHz, 990.00 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ])
    c = bench.parse_clocks(text)
    assert c["samples"] == 3
    assert c["sm_mhz"] == 1845.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert bench.parse_clocks("")["samples"] == 0


def test_flop_and_byte_accounting():
    w = syn.LLAMA_PREFILL
    assert w.flops == 4 * 32 * 32 * 4096 * 4096 * 128 / 2
    lens = np.array([512, 1000], np.int32)
    assert bench.decode_flops(lens) == 4.0 * 32 * 128 * 1512
    d = syn.DECODE
    assert d.kv_bytes(lens) == 1512 * 8 * 128 * 2 * 2
    assert bench.step_flops(lens) == w.flops + bench.decode_flops(lens)


def test_load_peaks_fallback(tmp_path):
    peaks, src = bench.load_peaks(str(tmp_path / "missing.json"))
    assert src == "fallback" and peaks["bf16_tflops"] > 0
    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0, "bf16_tflops_sustained": 3.0}))
    peaks, src = bench.load_peaks(str(p))
    assert src == "measured" and peaks == {"hbm_gbs": 1.0, "bf16_tflops": 2.0, "bf16_tflops_sustained": 3.0}


def test_reference_arm_line_and_rank_rule(monkeypatch, capsys):
    # small stand-ins so the test is quick; the arm's logic is what is checked
    monkeypatch.setattr(bench, "PREFILL", syn.LLAMA_PREFILL.with_(B=1, Lq=256, Lk=256, Hq=2, Hkv=2))
    monkeypatch.setattr(bench, "DECODE", syn.DECODE.with_(B=2, len_hi=600))
    args = bench.parse_args(["--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-step-seconds", "0.05"])
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""          # non-zero ranks do no work
    bench.run_reference(args, rank=0, world=2)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["higher_is_better"] is True


def test_warmup_minimum_enforced():
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])


def test_traffic_key_ignores_comments_only():
    src = "int f(int x) {  // twice\n  return 2 * x; /* doubled */\n}\n"
    same = "// a new header line\nint f(int x) {\n  return 2 * x;   // doubled\n}\n"
    other = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench._code_only(src) == bench._code_only(same)
    assert bench._code_only(src) != bench._code_only(other)

