"""The bandwidth profile ("FreeToken gguf": `ft bench bw`; "FreeToken linux", setup:
measure the machine's PCIe bandwidth rather than trust the specification) written
end to end on a GPU: the module's command line runs the pinned host<->device link
probe and the host memcpy probe and writes one JSON file."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bwprofile_writes_the_profile_file(tmp_path):
    out = tmp_path / "bw_profile.json"
    r = subprocess.run([sys.executable, "-m", "moe_expert_offload_top_b200.bwprofile", "--out", str(out),
                        "--bytes", str(64 << 20), "--iters", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    prof = json.loads(out.read_text())
    for key in ("library", "bytes", "iters", "host_memcpy_gbs_1_thread", "host_memcpy_gbs_all_threads",
                "host_threads", "h2d_gbs", "d2h_gbs"):
        assert key in prof, key
    assert prof["bytes"] == 64 << 20 and prof["iters"] == 3
    # a PCIe or faster host link, and a host memcpy that moves bytes: positive, finite, and
    # below any physical bound of these links (1 TB/s)
    for key in ("h2d_gbs", "d2h_gbs", "host_memcpy_gbs_1_thread", "host_memcpy_gbs_all_threads"):
        assert 1.0 < prof[key] < 1000.0, (key, prof[key])
    # the printed line is the file's content
    assert json.loads(r.stdout.strip().splitlines()[-1]) == prof
