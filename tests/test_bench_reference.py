"""bench.py's reference arm (the float64 oracle on the host cores) for the
striped and HyenaND passes prints one well-formed JSON line (CPU only)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("args,metric_word,unit", [
    (["--pass", "striped"], "StripedHyena", "1e9 B*D*L/s"),
    (["--pass", "nd", "--nd-config", "0"], "HyenaND", "1e9 B*D*grid/s"),
])
def test_reference_arm_line(args, metric_word, unit):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3", *args],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and metric_word in d["metric"] and d["unit"] == unit
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
