"""Host logic of the bench's decode roofline object (no GPU): the dominant
kernel's achieved bandwidth is the algorithmic bytes of the layers whose
one-token call is a single k_stream launch over the sum of their per-call
times; with no such layer it falls back to the whole M = 1 set, and the
ncu traffic record is quoted only for the k_stream form."""
import bench


def _inputs():
    specs = bench.HEAD_SPECS
    per_layer = {s.name: {"1": {"us": 10.0 + i}} for i, s in enumerate(specs)}
    return specs, per_layer, {"1": {"GB/s": 1234.5}}


def test_roofline_over_single_launch_layers():
    specs, per_layer, per_m = _inputs()
    launches = {s.name: (2 if s.name.endswith((".k", ".v")) else 1) for s in specs}
    rec = {"bytes_per_launch": 123, "workload": "w", "summary": "s"}
    r = bench.decode_roofline(specs, launches, per_layer, per_m, 6543.4, "measured", rec, 3)
    ks = [s for s in specs if launches[s.name] == 1]
    b = sum(bench.algorithmic_bytes(s.K, s.N, s.r, 1) for s in ks)
    us = sum(per_layer[s.name]["1"]["us"] for s in ks)
    assert r["achieved"] == round(b / (us * 1e-6) / 1e9, 1)
    assert r["frac"] == round(r["achieved"] / 6543.4, 4)
    assert r["traffic"] == 123 and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert all(s.name in r["kernel"] for s in ks)
    assert not any(s.name in r["kernel"] for s in specs if launches[s.name] != 1)


def test_roofline_falls_back_to_the_set():
    specs, per_layer, per_m = _inputs()
    r = bench.decode_roofline(specs, {s.name: 2 for s in specs}, per_layer, per_m, 6543.4, "measured",
                              {"bytes_per_launch": 1, "workload": "w", "summary": "s"}, 3)
    assert r["achieved"] == 1234.5 and r["traffic"] is None and r["traffic_source"] is None
