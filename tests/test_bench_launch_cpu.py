"""bench.py's `--gpus N` on CPU: without a launcher it starts N replica
processes itself (RANK / LOCAL_RANK / WORLD_SIZE set, rendezvous on
127.0.0.1), their scalars meet over gloo, and rank 0 alone prints one line
for the whole job.  Driven with the host-only allocator workload, so no GPU is
needed; a WORLD_SIZE that disagrees with --gpus is refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, env=None, timeout=300):
    e = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
        e.pop(k, None)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=e,
                          capture_output=True, text=True, timeout=timeout, cwd=ROOT)


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_two_replicas_print_one_aggregated_line():
    one = _bench(["--workload", "alloc_host", "--steps", "200"])
    two = _bench(["--gpus", "2", "--workload", "alloc_host", "--steps", "200"])
    assert one.returncode == 0 and two.returncode == 0, two.stderr
    l1, l2 = _json_lines(one.stdout), _json_lines(two.stdout)
    assert len(l1) == 1 and len(l2) == 1
    assert l1[0]["ranks"] == 1 and l2[0]["ranks"] == 2 and l2[0]["cores"] == 2
    # the same trace on each rank: twice the calls over the slower rank's time
    assert l2[0]["value"] > 0 and l2[0]["prompt_tokens_saved"] == l1[0]["prompt_tokens_saved"]


def test_world_size_that_disagrees_with_gpus_is_refused():
    r = _bench(["--gpus", "3", "--workload", "alloc_host"],
               env={"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode == 2
    assert "WORLD_SIZE" in r.stderr and not _json_lines(r.stdout)
