"""N > 1 host logic on CPU: world-size-2 gloo process groups (no GPU).

The data path shards into independent replicas with no collective; the only
cross-rank steps are the barrier and the max-over-ranks timing reduction,
which are exercised here, plus a rank that fails is seen by the other rank
as an error, not a hang.
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

from activation_epilogue_tcgen05_b200.replicas import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _spawn(body: str, world=2, timeout=120, extra_env=None):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), PYTHONPATH=ROOT)
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", textwrap.dedent(body)], env=env,
                                      cwd=ROOT, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                      text=True))
    outs = []
    for p in procs:
        try:
            out, _ = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            p.kill()
            out, _ = p.communicate()
        outs.append((p.returncode, out))
    return outs


def test_shard_covers_units_exactly():
    for units in (0, 1, 5, 8, 13, 1000):
        for world in (1, 2, 3, 8):
            got = [list(shard(units, world, r)) for r in range(world)]
            flat = [u for part in got for u in part]
            assert flat == list(range(units))
            sizes = [len(p) for p in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def test_barrier_and_max_over_ranks_gloo():
    outs = _spawn("""
        from activation_epilogue_tcgen05_b200 import replicas
        rank, world, _ = replicas.env_rank()
        assert replicas.init("gloo", timeout_s=60)
        replicas.barrier()
        mx = replicas.max_over_ranks(1.5 + rank)
        total = replicas.sum_over_ranks(10.0)
        units = list(replicas.shard(10, world, rank))
        print("RESULT", rank, mx, total, units[0], len(units), flush=True)
        replicas.finalize()
    """)
    res = {}
    for rc, out in outs:
        assert rc == 0, out
        line = [l for l in out.splitlines() if l.startswith("RESULT")][0].split()
        res[int(line[1])] = line[2:]
    assert res[0][:2] == ["2.5", "20.0"] and res[1][:2] == ["2.5", "20.0"]
    assert res[0][2:] == ["0", "5"] and res[1][2:] == ["5", "5"]


def test_failed_rank_is_an_error_not_a_hang():
    """Rank 1 raises before the collective; rank 0's next collective ends with an error."""
    outs = _spawn("""
        import sys
        from activation_epilogue_tcgen05_b200 import replicas
        rank, world, _ = replicas.env_rank()
        replicas.init("gloo", timeout_s=10)
        replicas.barrier()
        if rank == 1:
            sys.exit(3)
        try:
            replicas.max_over_ranks(1.0)
            replicas.barrier()
            print("NO-ERROR", flush=True)
        except Exception as e:
            print("ERROR-SEEN", type(e).__name__, flush=True)
            sys.exit(4)
    """, timeout=90)
    (rc0, out0), (rc1, _) = outs
    assert rc1 == 3
    assert "ERROR-SEEN" in out0 and rc0 == 4, out0


def test_bench_reference_arm_other_ranks_exit_quietly():
    """Under torchrun-style env with N = 2, only rank 0 runs the reference arm."""
    port = _free_port()
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
