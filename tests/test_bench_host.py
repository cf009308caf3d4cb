"""Host-side logic of bench.py, on CPU: the max-over-ranks reduction with two
gloo ranks, the reference arm under torchrun (rank 0 alone prints), the
algorithmic byte and FLOP counts behind the roofline, weight cloning for the
L2 rotation, the ncu traffic lookup and the clock-sample summary."""
import json
import os
import subprocess
import sys
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from w4a4_diffusion_model_b200 import synth  # noqa: E402


def _max_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q.put((rank, bench.aggregate_max(10.0 + 7.0 * rank, world)))
    finally:
        dist.destroy_process_group()


def test_aggregate_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 17.0, 1: 17.0}
    assert bench.aggregate_max(3.5, 1) == 3.5


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={30500 + os.getpid() % 1000}",
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1",
           "--workload", synth.TINY.name]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(s) for s in out.stdout.splitlines() if s.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_algorithmic_bytes_and_flops():
    w = synth.FLUX_QKV
    # X read, inv_lambda, L1p read; codes, scales (rows padded to 128), T written
    assert bench.quantize_bytes(w) == (2 * 4608 * 3072 + 4 * 3072 + 2 * 32 * 3072 + 4608 * 1536 + 4608 * 192
                                       + 2 * 4608 * 32)
    assert bench.gemm_flops(w) == 2 * 4608 * 9216 * 3072 + 2 * 4608 * 32 * 9216
    assert w.flops() == bench.gemm_flops(w) + 2 * 4608 * 32 * 3072
    w1 = w.with_(M=200)
    assert bench.quantize_bytes(w1) - bench.quantize_bytes(w1.with_(M=199)) == 2 * 3072 + 1536 + 2 * 32
    assert bench.quantize_bytes(w1.with_(M=256)) - bench.quantize_bytes(w1) > 56 * (2 * 3072 + 1536)


def test_clone_weights_copies_every_buffer():
    from w4a4_diffusion_model_b200 import svdq as S
    P = S.PreparedWeights(S.LayerShape(0, 128, 128, 16), torch.arange(8, dtype=torch.uint8),
                          torch.ones(4, dtype=torch.uint8), torch.zeros(16, 128, dtype=torch.bfloat16),
                          torch.zeros(128, 16, dtype=torch.bfloat16), torch.ones(128), torch.ones(128))
    C = bench.clone_weights(P)
    for f in ("Qr", "Sr", "L1p", "L2t", "lam", "inv_lam"):
        a, b = getattr(P, f), getattr(C, f)
        assert torch.equal(a, b) and a.data_ptr() != b.data_ptr()
    assert bench.weight_bytes(P) == 8 + 4 + 2 * 16 * 128 * 2 + 2 * 128 * 4
    P0 = S.PreparedWeights(S.LayerShape(0, 128, 128, 0), P.Qr, P.Sr, None, None, P.lam, P.inv_lam)
    assert bench.clone_weights(P0).L1p is None


def test_profiled_traffic_needs_the_current_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "w4a4_diffusion_model_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.GEMM_SOURCES:
        (csrc / name).write_text(f"// {name}\n")
    (tmp_path / "profiles").mkdir()
    h = bench.kernel_source_hash(bench.GEMM_SOURCES)
    (tmp_path / "profiles" / "k.md").write_text(f"x\ntraffic_bytes_per_launch: 12345 {h}\n")
    assert bench.profiled_traffic("k.md", bench.GEMM_SOURCES) == 12345.0
    (csrc / bench.GEMM_SOURCES[0]).write_text("// changed\n")
    assert bench.profiled_traffic("k.md", bench.GEMM_SOURCES) is None
    assert bench.profiled_traffic("missing.md", bench.GEMM_SOURCES) is None


def test_clock_summary_keeps_the_timed_window(tmp_path):
    s = bench.ClockSampler("0")
    s.proc = object()
    s.path = str(tmp_path / "clocks.csv")
    base = time.time()

    def row(t, mhz, cap):
        stamp = time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(t)) + f".{int((t % 1) * 1000):03d}"
        return f"{stamp}, 0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, {cap}\n"

    with open(s.path, "w") as f:
        f.write(row(base - 5.0, 800, "Not Active"))            # before load: ignored
        for i in range(5):
            f.write(row(base + 0.2 * i, 1800 + i, "Active"))
    d = s.summary(base - 0.1, base + 1.0, base - 1.0)
    assert d["samples"] == 5 and d["sm_mhz"] == 1802 and d["sm_max_mhz"] == 1965
    assert d["reasons"] == ["sw_power_cap"] and d["window"] == "timed region"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device failure")
def test_our_arm_fails_loudly_without_a_device():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "1", "--warmup", "3",
                          "--workload", synth.TINY.name, "--no-extras"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode != 0
    assert not any(s.startswith("{") for s in out.stdout.splitlines())


def test_reference_arm_int4_codec():
    """`--codec int4` times the oracle's INT4 per-call path (the same line
    contract as the NVFP4 reference arm)."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--codec", "int4", "--steps", "2",
           "--warmup", "1", "--workload", synth.TINY.name]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    d = [json.loads(s) for s in out.stdout.splitlines() if s.startswith("{")][-1]
    assert d["impl"] == "reference" and d["value"] > 0
    assert "int4" in d["cpu_baseline"]["sample"]


def test_int4_quantize_bytes():
    w = synth.FLUX_QKV
    # X read, inv_lambda, L1p read; one byte per code, fp32 scales per 64 (rows padded to 128), T written
    assert bench.quantize_bytes_int4(w) == (2 * 4608 * 3072 + 4 * 3072 + 2 * 32 * 3072 + 4608 * 3072
                                            + 4608 * 48 * 4 + 2 * 4608 * 32)
    assert bench.quantize_bytes_int4(w.with_(M=130)) - bench.quantize_bytes_int4(w.with_(M=129)) == 2 * 3072 + 3072 + 64


def test_scale_group_stats_classes():
    """E4M3 scale bytes: 0 (zero / underflow), exponent field 0 with a nonzero
    mantissa (subnormal), 0x7E (448, saturated), the rest normal."""
    class FakeS:
        @staticmethod
        def svdq_scales_to_canonical(native, rows, K):
            return native.view(rows, K // 16)
    b = torch.tensor([[0x00, 0x01, 0x07, 0x08, 0x38, 0x7E, 0x7E, 0x00]], dtype=torch.uint8)
    st = bench.scale_group_stats(FakeS, b, 1, 128)
    assert st == {"groups": 8, "zero": 2, "subnormal": 2, "saturated": 2}
