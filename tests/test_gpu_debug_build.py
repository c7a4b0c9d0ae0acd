"""The range-checked build (libtq_debug.so, compiled with TQ_DEBUG): the
parity suites of the decode, gated decode, Monarch step with promotion,
compress, Tensor Cache and Self-Indexing paths run against it in a child
process (TQ_LIB=debug selects it), on their smaller cases.  Every parity test
checks the context's error word after each call, so an index outside its
array (TQ_ERR_RANGE, the access skipped) fails the run; the results must
match the oracle as with the release build."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suites_pass_on_the_range_checked_build():
    import compressed_kv_decode_b200 as tq
    from compressed_kv_decode_b200 import build

    build.build(debug=True)
    env = dict(os.environ, TQ_LIB="debug")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "tests/test_gpu_decode.py", "tests/test_gpu_gate.py", "tests/test_gpu_promotion.py",
           "tests/test_gpu_tensor_cache.py", "tests/test_gpu_self_index.py",
           "tests/test_gpu_compress.py",
           "-k", "not 32k and not 4m and not 1m and not end_to_end and not 70000 and not 60000"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    import re
    m = re.search(r"(\d+) passed", r.stdout)
    assert m and int(m.group(1)) >= 40, r.stdout[-2000:]
    # the child really loaded the debug library
    probe = subprocess.run([sys.executable, "-c", "import compressed_kv_decode_b200 as t; t.lib(); print(t.LIB_PATH)"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.stdout.strip().endswith("libtq_debug.so"), probe.stdout + probe.stderr
    assert tq.status_string(tq.TQ_ERR_RANGE) != "unknown status"
