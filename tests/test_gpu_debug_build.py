"""The debug build (libswa_debug.so, -DSWA_DEBUG) checks the tile, row and
slot indices of every kernel on the device and records SWA_ERR_INTERNAL
instead of trapping; compute-sanitizer is not available on this hardware's
pool, so this is the bounds check.  Every compute call runs through it in a
fresh process (SWA_DEBUG=1 selects the library) and must match the oracle
with no check firing."""
import os
import subprocess
import sys

import pytest

from decode_swa_prefill_b200 import build as swa_build

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_every_call_through_the_debug_build():
    swa_build.build(debug=True)
    env = dict(os.environ, SWA_DEBUG="1", PYTHONPATH=os.pathsep.join([os.path.dirname(HERE), HERE]))
    out = subprocess.run([sys.executable, os.path.join(HERE, "debug_build_cases.py")], capture_output=True,
                         text=True, timeout=900, env=env, cwd=HERE)
    print(out.stdout[-4000:])
    assert out.returncode == 0, out.stderr[-4000:]
    assert "all cases ok" in out.stdout
