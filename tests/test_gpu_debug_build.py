"""The layer forward writes inside its buffers only, and the grouping it derives stays inside the
arrays it indexes: canary_run.py runs both FFN paths on ragged shapes with guard regions around
the output and after the workspace, once with libpw.so and once with libpw_debug.so (every
index the kernels derive from the grouping checked, a violation recorded as PW_ERR_BOUNDS
instead of the access).  Each variant runs in a child process because the binding loads one
library per process."""
import json
import os
import subprocess
import sys

import pytest

from any_precision_expert_pw_b200 import binding as B

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("variant", ["release", "debug"])
def test_forward_stays_inside_its_buffers(libpw, variant):
    env = dict(os.environ)
    env.pop("PW_LIB_VARIANT", None)
    if variant == "debug":
        env["PW_LIB_VARIANT"] = "debug"
        assert os.path.exists(os.path.join(os.path.dirname(B.LIB_PATH), "libpw_debug.so"))
    r = subprocess.run([sys.executable, os.path.join(HERE, "canary_run.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    lines = [json.loads(s) for s in r.stdout.splitlines() if s.startswith("{")]
    assert r.returncode == 0, (r.stdout[-4000:], r.stderr[-4000:])
    cases = [x for x in lines if "case" in x]
    assert len(cases) == 9 and all(x["ok"] for x in cases), lines
    assert ("debug" in lines[0]["library"]) == (variant == "debug")
