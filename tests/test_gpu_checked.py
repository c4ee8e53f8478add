"""The DQ_CHECKED build (lib/libdq_checked.so): its attention kernels count
containers whose decoder reads past the container's bytes in
dq_stats.overreads, and never trap. Host-side fault injection: a few
containers of a small cache are overwritten with a state that makes every
decode step take a byte. The default library leaves the counter at 0 and
flags the same containers through the final-state check only. Each library
runs in a child process (DQ_LIBRARY selects it)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(lib):
    from decode_attention_dq_b200 import build

    path = build.build(checked=True) if lib == "checked" else build.build()
    env = dict(os.environ, DQ_LIBRARY=path, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_probe.py")], env=env,
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_checked_build_counts_overreads():
    res = _run("checked")
    for tag in ("append", "decode_valid", "prefill_valid"):
        assert res[tag]["overreads"] == 0 and res[tag]["integrity_errors"] == 0, tag
    # decode: the 8 corrupt containers (every one is in the attended range)
    assert res["decode_corrupt"]["overreads"] == 8
    assert res["decode_corrupt"]["integrity_errors"] >= 8
    assert res["decode_corrupt_finite"]
    # prefill: the tile kernel decodes every container the chunk attends to once
    assert res["prefill_corrupt"]["overreads"] == 8
    assert res["prefill_corrupt"]["wait_timeouts"] == 0


def test_default_build_leaves_the_counter_at_zero():
    res = _run("default")
    assert res["decode_corrupt"]["overreads"] == 0
    assert res["decode_corrupt"]["integrity_errors"] >= 8
    assert res["prefill_corrupt"]["overreads"] == 0
