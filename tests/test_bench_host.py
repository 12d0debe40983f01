"""Host-side logic of bench.py that runs without a GPU: the max-over-ranks time of the
multi-GPU (replica) path on world-size-2 gloo ranks, and the reference arm's rank
gating and JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out_q.put((rank, bench.max_over_ranks(values[rank], "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    values = [3.25, 7.5]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 7.5, 1: 7.5}


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "linear", "--steps", "1", "--warmup", "0"],
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_only_rank0_prints():
    r1 = _run_reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0, 2)
    assert r0.returncode == 0
    lines = [ln for ln in r0.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "linear_m128_n1024_k1024"


def test_pair_gemm_l2_stream_bytes():
    """The L2 -> SM operand bytes the bench reports for the CTA-pair GEMM: per 256 x 256
    tile and 256-wide K stage, each CTA brings 128 A rows and 128 B rows of 128 bytes, A's
    four 512-byte scale atoms and both 128-row halves of B's (eight atoms)."""
    sys.path.insert(0, ROOT)
    import bench
    per_cta = 128 * 128 + 128 * 128 + 4 * 512 + 8 * 512
    assert bench.PAIR_STAGE_L2_BYTES == 2 * per_cta == 77824
    # MLP gate|up at 32768 tokens: 128 x 136 pair tiles, 20 K stages
    assert bench.pair_gemm_l2_bytes(32768, 34816, 5120) == 128 * 136 * 20 * 77824
    # down projection: 128 x 20 tiles, 68 K stages
    assert bench.pair_gemm_l2_bytes(32768, 5120, 17408) == 128 * 20 * 68 * 77824
    # a ragged last M tile still loads a whole pair tile
    assert bench.pair_gemm_l2_bytes(300, 256, 256) == 2 * 1 * 1 * 77824
