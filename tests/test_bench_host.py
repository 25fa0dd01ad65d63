"""Host-side logic of bench.py: argument defaults, the work accounting, and
the max-over-ranks timing on two gloo ranks (CPU only)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from bit_gemm_quant_b200 import roofline, synth


def test_defaults_and_workloads():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.impl == "w4" and a.workload == "decode" and a.warmup >= 3
    keys = [k for k, _ in bench.problems_for("decode")]
    assert len(keys) == 3 and len(set(keys)) == 3
    assert {k for k, _ in bench.problems_for("prefill")} == {"prefill_W"}


def test_algorithmic_bytes():
    # decode N=4096, K=4096, asym g=128: codes 8 MiB, 32 groups/row of fp16 scales, 4 zp words/row
    assert roofline.packed_bytes(4096, 4096, 128, 1) == 4096 * 2048 + 4096 * 64 + 4096 * 16
    assert roofline.gemm_bytes(1, 4096, 4096, 128, 1) == 8732672
    assert roofline.gemm_flops(2048, 14336, 4096) == 2 * 2048 * 14336 * 4096
    assert roofline.quant_pack_bytes(28672, 8192, 128, 0) == 2 * 28672 * 8192 + 28672 * 4096 + 2 * 28672 * 64
    # bf16 in, two E2M1 codes per byte, one scale byte per block
    assert roofline.fp4_quant_bytes(28672, 8192, 16) == 28672 * 8192 * 2 + 28672 * 4096 + 28672 * 512
    assert roofline.fp4_quant_bytes(1, 32, 32) == 64 + 16 + 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms, units = bench.aggregate(10.0 + 5 * rank, 100 * (rank + 1))
    bench.barrier()
    q.put((rank, ms, units))
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, units in res:
        assert ms == 15.0 and units == 300.0


@pytest.mark.parametrize("workload", ["decode", "decodequant", "awq", "fp4quant", "mxdecode", "smallbatch"])
def test_reference_arm_prints_one_complete_line(workload):
    """`bench.py --impl reference` (the CPU oracle on a bounded sample) prints
    one JSON line with the base contract's keys and the same workload
    description as the library's arm."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"), "--impl",
                          "reference", "--workload", workload, "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["value"] > 0 and d["warmup"] >= 3
    assert d["unit"] == "GB/s" and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    want = (bench.WORKLOAD_DESC[workload] if workload != "awq" else
            bench.awq_desc(bench.AWQ_SHAPE["M"], bench.AWQ_SHAPE["N"], bench.AWQ_SHAPE["K"],
                           bench.AWQ_SHAPE["group"], bench.AWQ_SHAPE["n_alpha"]))
    assert d["config"]["workload"] == want


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun with N > 1 the reference arm runs on rank 0 alone: the
    other ranks exit 0 without work or output, and rank 0's line counts N."""
    import json
    import subprocess
    import sys
    script = os.path.join(os.path.dirname(bench.__file__), "bench.py")
    cmd = [sys.executable, script, "--impl", "reference", "--workload", "decode", "--gpus", "2", "--steps", "1",
           "--warmup", "3"]
    for rank in (1, 0):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2")
        out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env)
        assert out.returncode == 0, out.stderr[-2000:]
        lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
        if rank:
            assert out.stdout.strip() == ""
        else:
            assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2


@pytest.mark.parametrize("workload", ["decode", "decodequant"])
def test_cpu_baseline_reports_single_thread_and_all_cores(workload):
    """The oracle timed single-threaded (the reported value) and, as a labelled
    variant, with its row slices on every host core: the product for the
    product workloads (weights quantized by the oracle beforehand), the
    quantization for the quantizer workloads."""
    plist = bench.problems_for(workload)
    keys = list(dict.fromkeys(k for k, _ in plist))
    qp = {k: p for k, p in reversed(plist)}
    host_W = {k: [synth.weights(qp[k].seed, qp[k].N, qp[k].K, qp[k].w_std, *qp[k].w_outlier)] for k in keys}
    host_s = {k: qp[k].s() for k in keys}
    host_X = {p.name: [p.X()] for _, p in plist if p.M > 0}
    quant = workload in bench.QUANT_WORKLOADS
    cpu = bench.cpu_baseline(workload, plist, keys, qp, host_W, host_X, host_s, 0.3, quant)
    assert cpu["kind"] == "oracle" and cpu["cores"] == 1 and cpu["value"] > 0 and cpu["unit"] == "GB/s"
    assert ("fold+quantize+pack" in cpu["sample"]) == quant
    if (os.cpu_count() or 1) > 1:
        mc = cpu["all_cores"]
        assert mc["cores"] == os.cpu_count() and mc["value"] > 0 and mc["unit"] == "GB/s"
