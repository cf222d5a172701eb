"""One rank of a CPU (gloo) replica group, started by test_replicas.py with the
environment torchrun would give it.  Usage: _replica_worker.py MODE OUT_JSON"""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from quantized_attention_qk_b200.replicas import (Replicas, env_int, head_range, sharded_forward,  # noqa: E402
                                                  timed_sharded, whole_job_tops)


def main():
    mode, out = sys.argv[1], sys.argv[2]
    rank = env_int("RANK", 0)
    if mode == "never" and rank == 1:
        sys.exit(0)  # this rank never joins the group
    result = {"rank": rank}
    try:
        reps = Replicas(backend="gloo", timeout_s=float(os.environ.get("TEST_PG_TIMEOUT", "30")))
        result["world"] = reps.world
        if mode == "max":
            # per-rank "times": rank r took 3 (r + 1) ms for 4 steps of 1e9 operations
            t = reps.max(3.0 * (rank + 1))
            reps.barrier()
            result["max"] = t
            result["tops"] = whole_job_tops(reps.world, 1e9, 4, t)
        elif mode.startswith("shard"):
            # one problem split by heads; the compute is the oracle's exact
            # attention (the sharding and the gather are what is tested)
            import torch
            import oracle
            H = int(mode[len("shard"):])
            g = torch.Generator().manual_seed(5)
            q, k, v = (torch.randn(2, H, 40, 16, generator=g).to(torch.bfloat16) for _ in range(3))

            def attn(qs, ks, vs, sm_scale=None):
                return torch.from_numpy(oracle.attn_exact(qs, ks, vs, sm_scale))

            full = sharded_forward(q, k, v, reps, sm_scale=0.25, gather=True, attn=attn, out_dtype=torch.float64)
            part = sharded_forward(q, k, v, reps, sm_scale=0.25, gather=False, attn=attn, out_dtype=torch.float64)
            ref = attn(q, k, v, sm_scale=0.25)
            h0, h1 = head_range(H, reps.world, rank)
            result["gathered_equal"] = bool(torch.equal(full, ref))
            result["part_equal"] = bool(torch.equal(part, ref[:, h0:h1]))
            result["heads"] = [h0, h1]
        elif mode == "timed_shard":
            # the timing path of bench.py --shard on CPU: warm-up, timed steps,
            # the maximum over ranks, and the gathered output
            import torch
            import oracle
            g = torch.Generator().manual_seed(6)
            q, k, v = (torch.randn(1, 5, 32, 16, generator=g).to(torch.bfloat16) for _ in range(3))

            def attn(qs, ks, vs, sm_scale=None):
                return torch.from_numpy(oracle.attn_exact(qs, ks, vs, sm_scale))

            calls = []
            got, mine, mx = timed_sharded(q, k, v, reps, steps=3, warmup=3, sm_scale=0.25, attn=attn,
                                          out_dtype=torch.float64, before_step=lambda: calls.append(1))
            result["gathered_equal"] = bool(torch.equal(got, attn(q, k, v, sm_scale=0.25)))
            result["mine_ms"] = mine
            result["max_ms"] = mx
            result["before_step_calls"] = len(calls)
        elif mode == "die":
            if rank == 1:
                os._exit(3)  # leaves between steps, before the next collective
            reps.barrier()
            result["max"] = reps.max(1.0)
        reps.close()
    except Exception as e:  # the error a surviving rank sees
        result["error"] = type(e).__name__
    with open(out, "w") as f:
        json.dump(result, f)


if __name__ == "__main__":
    main()
