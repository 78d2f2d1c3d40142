"""bench.py's multi-GPU launcher on CPU: `--gpus N` without torchrun
re-launches the script under torch.distributed.run with N ranks (here over
gloo, in the launcher self-test mode that needs no GPU), rank 0 prints one
line for the whole job, and a --gpus that disagrees with the launcher's
WORLD_SIZE is refused."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=240, cwd=ROOT)


def test_gpus_2_relaunches_two_ranks():
    p = _run(["--gpus", "2", "--cpu-dry-run"])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["dry_run"] is True
    assert d["value"] > 0 and d["ms_per_step"] >= 20.0   # the slower rank sleeps 20 ms


def test_gpus_disagreeing_with_world_size_is_refused():
    p = _run(["--gpus", "2", "--cpu-dry-run"], {"WORLD_SIZE": "3", "RANK": "0", "LOCAL_RANK": "0"})
    assert p.returncode != 0
    assert "WORLD_SIZE=3" in (p.stderr + p.stdout)
