"""The DRAM-traffic captures under profiles/ that bench.py reports beside its
rooflines belong to the kernel sources as they stand: each records the
sha256 of its kernel's source file, and bench.py drops a capture whose
kernel changed since it was taken.  A kernel edit without a fresh capture
fails here instead of silently reporting no traffic."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("kda_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_captures_match_kernel_sources():
    bench = _bench()
    assert set(bench.TRAFFIC_PROFILES) == {"kda_fwd_tc_kernel", "kda_decode_kernel", "kda_spec_kernel"}
    for kernel, (profile, source) in bench.TRAFFIC_PROFILES.items():
        kv = bench.read_kv(os.path.join(ROOT, "profiles", profile))
        assert kv["kernel_source_sha256"] == bench.source_sha(source), (kernel, profile)
        # the capture scales: bytes per unit are positive and finite
        per_launch = bench.scaled_traffic(profile, source, 1000, 0.0)
        assert per_launch is not None and per_launch > 0, (kernel, profile)
        assert int(kv["capture_units"]) > 0 and float(kv["gpu_time_ns"]) > 0
