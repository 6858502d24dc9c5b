"""Host-side checks of bench.py: the multi-process (one process per GPU) path,
exercised on the CPU with two gloo ranks (the barrier, the max-over-ranks timing and
the whole-job rate under weak scaling: each rank its own batch, no data-path
collective), and the roofline numerators against closed forms."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    my_ms = [2.0, 5.0][rank]                       # rank 1 is the slow one
    ms = bench.max_over_ranks(world, my_ms)
    rate = bench.whole_job_rate(world, 1e12, ms)   # 1 TFLOP of work per rank
    result_q.put((rank, ms, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, rate in res:
        assert ms == pytest.approx(5.0)             # both ranks see the max
        assert rate == pytest.approx(2 * 1e12 / 5e-3)


def test_bench_accounting_matches_the_closed_forms():
    """The roofline numerators of bench.py: flops per causal pair (B-space contraction,
    a_Q a_K weighting, values), causal pair counts, projection flops and factor bytes,
    against values worked out by hand for the benchmark shapes."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from tensor_product_attention_b200 import inputs as I
    c2 = I.WORKLOADS["prefill_b8_s2048_d1024"]
    c5 = I.WORKLOADS["layer_prefill_b4_s8192_d2048"]
    # 2*6*2*64 + 2*16*6*2 + 2*16*64 = 1536 + 384 + 2048
    assert bench.attn_flops_per_pair(c2) == 3968
    assert bench.attn_flops_per_pair(c5) == 2 * 6 * 2 * 128 + 2 * 16 * 6 * 2 + 2 * 16 * 128 == 7552
    assert bench.causal_pairs(8, 2048) == 8 * 2048 * 2049 // 2 == 16785408
    # (R_Q+R_K+R_V)(h+d_h) = 10 * 80 = 800 output columns, 2 T N D flops
    assert bench.proj_flops(c2, 16384) == 2 * 16384 * 800 * 1024
    assert bench.cache_bytes_per_token(I.WORKLOADS["decode_b64_ctx32k"]) == (2 + 2) * (16 + 128) * 2 == 1152
    sb = I.WORKLOADS["shared_basis_decode_b64_ctx32k"]
    assert bench.cache_bytes_per_token(sb) == (2 + 2) * 16 * 2 == 128
    # shared basis: W_B_k and W_B_v are not projected
    assert bench.proj_flops(I.custom("p", c2, shared_basis=True), 10) == 2 * 10 * (800 - 4 * 64) * 1024


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference times the fp64 oracle on the host cores and prints one
    JSON line with the bench contract's keys (no GPU involved)."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["config"]["workload"] == "prefill_b8_s2048_d1024"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]
