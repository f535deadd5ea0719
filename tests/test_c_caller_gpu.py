"""cvq_attend driven from C with no Python in the loop (tests/c_abi/attend_loop.c): the
program runs a small layer and the 128K-token layer, reports the host cost of a call, the
device time per step and an end-to-end step (codes and queries copied from pinned host
memory, out and lse read back), and exits 0 only if the device fault word stayed 0 and
the outputs are finite."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("args", [["1", "4", "1", "1", "4096", "50"],
                                  ["1", "32", "8", "1", "131072", "20"]])
def test_c_caller_runs(tmp_path, args):
    sys.path.insert(0, os.path.join(ROOT, "tests", "c_abi"))
    import build_attend_loop

    exe = build_attend_loop.build(str(tmp_path / "attend_loop"))
    r = subprocess.run([exe, *args], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["fault"] == 0 and line["outputs_finite"] == 1
    assert line["device_us_per_step"] > 0 and line["host_us_per_call"] > 0
    print(json.dumps(line))
