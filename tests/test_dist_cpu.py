"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

The path shards by tokens with no collective on the data path; the only
cross-rank steps are the barrier and the max over ranks of the timed region.
These tests run them on gloo (world size 2) without a GPU.
"""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench._max_over_ranks(local_ms[rank], True, device="cpu")
        value, ms = bench.job_throughput(got, 10, world, 1e12)
        dist.barrier()
        q.put((rank, got, value, ms))
    finally:
        dist.destroy_process_group()


def _run(world, local_ms):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_max_over_ranks_two_gloo_ranks():
    out = _run(2, [12.5, 40.0])
    for rank, got, value, ms in out:
        assert got == 40.0  # every rank sees the slowest rank's time
        assert ms == pytest.approx(4.0)
        # two ranks each did 1e12 FLOP per step in 4 ms per step
        assert value == pytest.approx(2 * 1e12 / 4e-3 / 1e12)


def test_single_rank_passthrough():
    import bench
    assert bench._max_over_ranks(3.25, False) == 3.25
    value, ms = bench.job_throughput(50.0, 5, 1, 2e9)
    assert ms == 10.0 and value == pytest.approx(2e9 / 1e-2 / 1e12)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-rows", "16"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-rows", "16"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "config", "cpu_baseline", "e2e"):
        assert k in d
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_bench_kernel_models_add_up_to_the_step():
    # the per-launch FLOP models of the c2 step's kernels sum to the step's
    # executed FLOPs (so a kernel's roofline and the step's value agree), and
    # so do the groups of back-to-back launches
    import torch
    import bench
    from associative_algebra_block_b200 import inputs
    wl = bench.WORKLOADS["c2"]()
    st = inputs.Stream(100)
    wl.sets = [{"dec": [{"pos": torch.from_numpy(st.positions(B, wl.seq_len))}
                        for B in wl.decode_batches]}]
    total = 0
    for name, _ in wl.timing_slots():
        flops, byts = wl.kernel_model(name)
        assert byts > 0
        total += flops
    assert total == wl.exec_flops
    assert sum(wl.group_model(g)[0] for g in wl.group_names()) == wl.exec_flops
    # c4-swiglu: the six timed launches are a subset of the step's work
    w4 = bench.WORKLOADS["c4-swiglu"]()
    assert sum(w4.kernel_model(n)[0] for n, _ in w4.timing_slots()) < w4.exec_flops


@pytest.mark.parametrize("law,q", [("Q", 1), ("Q", 2), ("Q", 5), ("Q", 32), ("Q2xQ2", 4)])
def test_bench_work_accounting_matches_the_oracle_table(law, q):
    # the bench counts FLOPs from closed forms (it never loads libaal or the
    # oracle on the GPU arm); they must agree with the oracle's table
    import bench
    import oracle
    S = oracle.block_table(law, q)
    for t in range(q):
        for k in range(q):
            assert bench._members(law, q, t, k) == tuple(S[t][k])
    assert bench._per_row(law, q) == oracle.block_product_count(law, q, True)
    assert bench._square_count(law, q) == oracle.block_product_count(law, q, False)


def test_reference_arm_never_loads_libaal():
    code = ("import sys; sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', "
            "'--warmup', '0', '--ref-rows', '16']\n"
            "import bench\n"
            "bench.main()\n"
            "maps = open('/proc/self/maps').read()\n"
            "print('LIBAAL_MAPPED' if 'libaal' in maps else 'LIBAAL_NOT_MAPPED')\n")
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                       env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip().splitlines()[-1] == "LIBAAL_NOT_MAPPED"


@pytest.mark.parametrize("config", ["c4", "c5", "c4-swiglu"])
def test_reference_arm_other_workloads(config):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", config, "--steps", "1", "--warmup", "0", "--ref-rows", "32"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"


def _shard_worker(rank, world, port, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        import oracle
        from associative_algebra_block_b200 import inputs
        from associative_algebra_block_b200.sharding import token_shard
        law, q, L, M, din, dout = "Q2xQ2", 4, 12, 5 * 12 + 7, 8, 12
        s = inputs.Stream(70)
        X = s.integers(M, din, -3, 3, "f32").f64
        W = s.integers(din, dout, -3, 3, "f32").f64
        dY = s.integers(M, dout, -3, 3, "f32").f64
        r0, r1 = token_shard(M, L, world, rank)
        # the position rule is unchanged on the shard: it starts at a sequence start
        types = oracle.row_types(law, q, inputs.packed_positions(r1 - r0, L))
        Y = oracle.project(law, q, types, X[r0:r1], W)
        dX, dW = oracle.project_bwd(law, q, types, X[r0:r1], W, dY[r0:r1])
        # forward: no exchange; the rows are gathered here only to check them
        parts = [None] * world
        dist.all_gather_object(parts, (r0, r1, Y, dX))
        # backward: the weight gradient is a sum over tokens -> one all-reduce
        t = torch.from_numpy(dW.copy())
        dist.all_reduce(t)
        q_out.put((rank, parts, t.numpy()))
    finally:
        dist.destroy_process_group()


def test_token_shards_reassemble_the_single_rank_result():
    import numpy as np
    import oracle
    from associative_algebra_block_b200 import inputs
    world = 2
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q_out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    law, q, L, M, din, dout = "Q2xQ2", 4, 12, 5 * 12 + 7, 8, 12
    s = inputs.Stream(70)
    X = s.integers(M, din, -3, 3, "f32").f64
    W = s.integers(din, dout, -3, 3, "f32").f64
    dY = s.integers(M, dout, -3, 3, "f32").f64
    types = oracle.row_types(law, q, inputs.packed_positions(M, L))
    Y = oracle.project(law, q, types, X, W)
    dX, dW = oracle.project_bwd(law, q, types, X, W, dY)
    for rank, parts, dW_sum in out:
        covered = sorted((r0, r1) for r0, r1, _, _ in parts)
        assert covered[0][0] == 0 and covered[-1][1] == M
        assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))
        for r0, r1, Ys, dXs in parts:
            assert r0 % L == 0  # shards start at a sequence start
            assert np.array_equal(Ys, Y[r0:r1]) and np.array_equal(dXs, dX[r0:r1])
        assert np.array_equal(dW_sum, dW)  # exact on small integers


@pytest.mark.parametrize("rows,seq_len,world", [(0, 4, 2), (10, 4, 3), (12, 4, 3), (12288, 1536, 8),
                                                (7, 10, 4)])
def test_token_shard_covers_rows_by_whole_sequences(rows, seq_len, world):
    from associative_algebra_block_b200.sharding import token_shard
    spans = [token_shard(rows, seq_len, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == rows
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    for r0, r1 in spans:
        assert r0 <= r1 and (r0 % seq_len == 0 or r0 == rows)
