"""Bandwidth profile of this machine for the expert cache: the pinned host<->device link
the slot fills use, and host memory copy bandwidth, written as one JSON file.

    python -m moe_expert_offload_top_b200.bwprofile [--out bw_profile.json] [--host-only]

Method ("FreeToken linux", setup: measure the PCIe bandwidth of the machine instead of
trusting the specification): the link is timed with CUDA events over pinned copies of
`--bytes` each way (ft_probe_host_link); host memory with timed memcpy passes
(ft_probe_host_memory) on 1 thread and on every core.
"""
import argparse
import json
import os
import sys

from moe_expert_offload_top_b200 import ft_probe_host_link, ft_probe_host_memory, ft_version


def profile(bytes_=256 << 20, iters=5, host_only=False):
    cores = os.cpu_count() or 1
    out = {"library": ft_version(), "bytes": bytes_, "iters": iters,
           "host_memcpy_gbs_1_thread": ft_probe_host_memory(bytes_, 1, iters),
           "host_memcpy_gbs_all_threads": ft_probe_host_memory(bytes_, cores, iters),
           "host_threads": cores}
    if not host_only:
        h2d, d2h = ft_probe_host_link(bytes_, iters)
        out.update({"h2d_gbs": h2d, "d2h_gbs": d2h})
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--out", default="bw_profile.json")
    ap.add_argument("--bytes", type=int, default=256 << 20)
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--host-only", action="store_true", help="skip the GPU link (no device needed)")
    a = ap.parse_args(argv)
    prof = profile(a.bytes, a.iters, a.host_only)
    with open(a.out, "w") as f:
        json.dump(prof, f, indent=1)
    print(json.dumps(prof))
    return 0


if __name__ == "__main__":
    sys.exit(main())
