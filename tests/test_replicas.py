"""The multi-GPU path on CPU: replicas coordinated over gloo with world size 2,
in processes started the way torchrun starts them (RANK, WORLD_SIZE,
MASTER_ADDR=127.0.0.1, MASTER_PORT in the environment)."""
import json
import os
import socket
import subprocess
import sys

import pytest

from quantized_attention_qk_b200.replicas import Replicas, head_range, whole_job_tops

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(mode, tmp_path, world=2, pg_timeout=30, wall=120):
    port = _free_port()
    procs, outs = [], []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), TEST_PG_TIMEOUT=str(pg_timeout))
        out = tmp_path / f"rank{r}.json"
        outs.append(out)
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "_replica_worker.py"), mode, str(out)],
                                      env=env))
    codes = []
    for p in procs:
        try:
            codes.append(p.wait(timeout=wall))
        except subprocess.TimeoutExpired:
            p.kill()  # the exact process this test started
            codes.append(None)
    results = [json.loads(o.read_text()) if o.exists() else None for o in outs]
    return codes, results


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    r = Replicas()
    assert (r.world, r.rank, r.is_root) == (1, 0, True)
    r.barrier()
    assert r.max(2.5) == 2.5
    r.close()


def test_whole_job_throughput_counts_every_rank():
    # 2 ranks x 4 steps x 1e12 operations in 8 ms -> 1000 TOPS
    assert whole_job_tops(2, 1e12, 4, 8.0) == pytest.approx(1000.0)
    with pytest.raises(ValueError):
        whole_job_tops(1, 1.0, 1, 0.0)


def test_bad_rank_is_rejected(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "2")
    with pytest.raises(ValueError):
        Replicas(backend="gloo")


def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path):
    codes, res = _run_ranks("max", tmp_path)
    assert codes == [0, 0]
    for r in res:
        assert r["world"] == 2
        assert r["max"] == 6.0                        # rank 1's 3 * 2 ms
        assert r["tops"] == pytest.approx(2 * 1e9 * 4 / 6e-3 / 1e12)


def test_a_rank_that_leaves_fails_the_others_instead_of_hanging(tmp_path):
    codes, res = _run_ranks("die", tmp_path, pg_timeout=5)
    assert codes[1] == 3
    assert codes[0] == 0                              # rank 0 returned (no hang)
    assert "error" in res[0]


def test_a_rank_that_never_joins_fails_the_others(tmp_path):
    codes, res = _run_ranks("never", tmp_path, pg_timeout=5)
    assert codes == [0, 0]
    assert "error" in res[0]


def test_reference_arm_does_nothing_on_other_ranks():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0
    assert p.stdout.strip() == ""


def test_head_ranges_cover_every_head_once():
    for H in (1, 2, 5, 24, 40):
        for W in (1, 2, 3, 8):
            got = [head_range(H, W, r) for r in range(W)]
            assert got[0][0] == 0 and got[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world,H", [(2, 5), (3, 5), (2, 1)])
def test_head_sharded_forward_gathers_the_whole_result(tmp_path, world, H):
    codes, res = _run_ranks(f"shard{H}", tmp_path, world=world)
    assert codes == [0] * world
    for r in res:
        assert "error" not in r, r
        assert r["gathered_equal"] and r["part_equal"], r


def test_timed_head_sharding_takes_the_slowest_rank(tmp_path):
    """bench.py --shard's timing path over two gloo ranks: both ranks time the
    same steps, report the same maximum, which is at least their own time, and
    the gathered output is the whole problem's."""
    codes, res = _run_ranks("timed_shard", tmp_path)
    assert codes == [0, 0], res
    assert all(r.get("error") is None for r in res), res
    assert all(r["gathered_equal"] for r in res)
    assert res[0]["max_ms"] == res[1]["max_ms"] == max(r["mine_ms"] for r in res)
    assert all(r["before_step_calls"] == 3 for r in res)
