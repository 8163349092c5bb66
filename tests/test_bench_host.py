"""Host-side logic of bench.py (CPU only): the byte model, clock summaries,
the DRAM-traffic record, max-over-ranks across two gloo processes, and the
reference arm (the CPU oracle) on the tiny workload."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import dcn4_inputs as gen  # noqa: E402


def test_byte_model_matches_the_compulsory_bytes():
    bm = bench.byte_model(gen.WORKLOADS["stage1_f16"])
    assert bm["fwd"] == 25_690_112 + 44_957_696 + 25_690_112
    assert bm["bwd"] == 166_985_728
    bm5 = bench.byte_model(gen.WORKLOADS["train_bf16_k8"])
    assert bm5["fwd"] == 89_915_392 and bm5["bwd"] == 154_140_672
    assert bench.byte_model(gen.WORKLOADS["tiny_f32"])["fwd"] == 22_528


def test_summarize_clocks():
    rows = [(1.0, ["0", "1965", "1965", "500", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]),
            (2.0, ["0", "1900", "1965", "900", "0x4", "Not Active", "Not Active", "Not Active", "Active"]),
            (9.0, ["0", "120", "1965", "90", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"])]
    c = bench.summarize_clocks(rows, 0.5, 2.5)
    assert c["sm_mhz"] == 1932.5 and c["sm_max_mhz"] == 1965.0 and c["reasons"] == ["sw_power_cap"]
    assert c["window"] == "timed loop" and c["samples"] == 2
    c = bench.summarize_clocks(rows, 5.0, 6.0)
    assert c["samples"] == 3 and c["window"].startswith("whole run")


def test_kernel_sources_sha_covers_the_kernels_own_sources():
    shas = {k: bench.kernel_sources_sha(k) for k in bench.KERNELS.values()}
    assert shas["samples_kernel"] == shas["value_kernel"]          # one translation unit
    assert shas["forward_kernel"] != shas["value_kernel"]
    assert all(len(v) == 64 for v in shas.values())


def test_recorded_traffic_needs_matching_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    sha = bench.kernel_sources_sha("value_kernel")
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# kernel workload bytes sources_sha256\n"
        f"value_kernel stage1_f16 123456 {sha}\n"
        "forward_kernel stage1_f16 99 0000\n")
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda kernel: sha)
    assert bench.recorded_traffic("value_kernel", "stage1_f16") == 123456
    assert bench.recorded_traffic("forward_kernel", "stage1_f16") is None   # other sources
    assert bench.recorded_traffic("samples_kernel", "stage1_f16") is None   # not captured


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        out[rank] = bench.max_over_ranks(10.0 * (rank + 1))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_processes():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn")
        assert dict(out) == {0: 20.0, 1: 20.0}


def test_reference_arm_tiny():
    import time
    t0 = time.time()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_f32", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=300)
    wall = time.time() - t0
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "us/call" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    # the whole batch fits the budget: no scaling, and the measured steps fit the run
    assert line["config"]["images_per_step"] == 1
    assert abs(line["value"] - line["ms_per_step"] * 1e3) <= 1e-3 * line["value"] + 0.1
    assert line["ms_per_step"] * (line["steps"] + line["warmup"]) / 1e3 <= wall
    assert line["cpu_baseline"]["cores"] == 1          # one image: one thread does the work


def test_config_record_fractions():
    w = gen.WORKLOADS["stage1_f16"]
    rec = bench.config_record(w, {"fwd": 100.0, "bwd_offset_mask": 150.0, "bwd_value": 50.0},
                              {"hbm_gbs": 6000.0})
    assert rec["fwd_us"] == 100.0 and rec["bwd_us"] == 200.0
    assert rec["fwd_gbs"] == round(96_337_920 / 100e-6 / 1e9, 1)
    assert rec["bwd_frac_hbm"] == round(166_985_728 / 200e-6 / 1e9 / 6000.0, 4)
    assert rec["fwd_frac_8tbs"] == round(96_337_920 / 100e-6 / 1e9 / 8000.0, 4)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_f32", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=300,
                       env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_attn_byte_model():
    w = gen.ATTN_WORKLOADS["attn_enc_f16"]
    bm = bench.attn_byte_model(w)
    value, ref, ol, out = 8 * 64 * 64 * 256 * 2, 8 * 4096 * 8, 8 * 4096 * 96 * 2, 8 * 4096 * 256 * 2
    assert bm["fwd"] == value + ref + ol + out
    assert bm["bwd"] == value + ref + ol + out + value + ol
