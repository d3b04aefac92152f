"""Host-side logic of bench.py without a GPU: the max-over-ranks reduction and the job
throughput with two gloo ranks, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [1.0 + rank, 10.0 - rank]           # rank 1 is slower on the first entry
        dist.barrier()
        res = bench.max_over_ranks(local, dist, torch.device("cpu"))
        out[rank] = res + [bench.job_throughput(world, 8, res[0])]
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    for r in range(world):
        assert res[r][:2] == [2.0, 10.0]            # max over ranks, on every rank
        assert res[r][2] == pytest.approx(2 * 8 / 2e-3)


def test_single_rank_passthrough():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.job_throughput(1, 8, 0.1) == pytest.approx(80000.0)


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = [l for l in r.stdout.splitlines() if l.startswith("{")][-1]
    d = json.loads(line)
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["metric"] == json.load(open(os.path.join(ROOT, "BASELINE.json")))["metric"]


def test_ffn_kernel_name_follows_the_library_rule():
    from expert_routed_ffn_softmax_b200 import build
    build.build()
    # the default form is the dynamic FFN with an A slot of the smallest of 8..128 rows >= T
    assert bench.ffn_kernel_name(1, "auto") == "expert_ffn_dynamic_kernel<8>"
    assert bench.ffn_kernel_name(9, "auto") == "expert_ffn_dynamic_kernel<16>"
    assert bench.ffn_kernel_name(64, "prefill") == "expert_ffn_dynamic_kernel<64>"
    assert bench.ffn_kernel_name(65, "auto") == "expert_ffn_dynamic_kernel<128>"
    assert bench.ffn_kernel_name(32768, "auto") == "expert_ffn_dynamic_kernel<128>"
    assert bench.ffn_kernel_name(32768, "pairs") == "expert_ffn_pair_kernel"      # CTA pairs
    assert "+" in bench.ffn_kernel_name(4096, "unfused")          # two launches
    assert bench.ffn_kernel_name(8, "fused").endswith(",1>")       # 8-row A slots
    assert bench.ffn_kernel_name(8, "decode").startswith("grouped_gemm_decode_kernel")


def test_nvfp4_expert_bytes_are_the_formats():
    """Per expert: three projections of H x I codes at 4 bits, one E4M3 byte per 16 of them,
    three fp32 tensor scales."""
    H, I = 2816, 704
    assert bench.FP4_EXPERT_BYTES == 3 * H * I // 2 + 3 * H * I // 16 + 3 * 4 == 3_345_420


def test_nvfp4_entry_arithmetic():
    from expert_routed_ffn_softmax_b200 import workloads as wl
    cfg = wl.CONFIGS["decode"]
    m = {"active": 57, "ffn_ms": 0.060, "ms": 0.087, "stages": {"expert_ffn": 0.060},
         "clocks": {}, "kernels": 4, "_steps": 20}
    e = bench.nvfp4_entry(cfg, m, 1, {"hbm_gbs": 6544.7})
    gbs = 57 * 3_345_420 / 60e-6 / 1e9
    assert e["expert_ffn"]["algorithmic_bytes"] == 57 * 3_345_420
    assert abs(e["expert_ffn"]["achieved_gbs"] - gbs) < 1e-6 * gbs
    assert abs(e["expert_ffn"]["frac_of_hbm"] - gbs / 6544.7) < 1e-9
    assert abs(e["value"] - 8 / 0.087e-3) < 1e-6 * e["value"]       # tokens/s of one rank
    assert e["gpu_launches"] == 80
    e2 = bench.nvfp4_entry(cfg, m, 2, {"hbm_gbs": 6544.7})
    assert abs(e2["value"] - 2 * e["value"]) < 1e-6 * e["value"]    # the whole job


def test_tensor_bound_entry_arithmetic():
    from expert_routed_ffn_softmax_b200 import workloads as wl
    cfg = wl.CONFIGS["skewed"]
    acc = {"gemm1_flops": 1.0e12, "gemm2_flops": 0.5e12, "step_flops": 1.6e12,
           "active_experts": 63}
    m = {"acc": acc, "stages": {"expert_ffn": 1.5}, "ms": 2.0, "rstats": {}, "clocks": {},
         "kernels": 4, "_steps": 20, "_tiles": "auto"}
    pk = {"bf16_tflops": 1662.1, "bf16_tflops_sustained": 1394.8}
    e = bench.tensor_bound_entry(cfg, m, 1, pk)
    tf = 1.5e12 / 1.5e-3 / 1e12
    assert abs(e["expert_ffn"]["achieved_tflops"] - tf) < 1e-9 * tf
    assert abs(e["expert_ffn"]["frac_of_burst"] - tf / 1662.1) < 1e-12
    assert abs(e["expert_ffn"]["frac_of_sustained"] - tf / 1394.8) < 1e-12
    assert abs(e["step_tensor_frac"] - (1.6e12 / 2.0e-3) / 1662.1e12) < 1e-12
    assert "router bias" in e["workload"]


def test_kernel_source_hashes_are_per_family():
    a, b = bench.kernel_source_sha("bf16"), bench.kernel_source_sha("nvfp4")
    assert a != b and len(a) == len(b) == 16
    assert a == bench.kernel_source_sha("bf16")
