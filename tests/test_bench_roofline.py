"""Host logic of the bench's measurement units and decode roofline object
(no GPU).  The per-call units are pinned to values summed by hand from their
definitions (vals N K / 4 + meta N K / 8 + scales 2 N K / 128 + L 2 K r +
R 2 r N + X 2 M K + Y 2 M N bytes; kept FLOPs 2 M N K / 2 + adapter
2 M r (K + N); 4-bit adapters: 1056-byte blocks of 16 columns x 128 K for L,
16-row tiles of r / 2 bytes a row plus a 2-byte scale per 128 of r for R).
The dominant kernel's achieved bandwidth is the algorithmic bytes of the
layers whose one-token call is a single k_stream launch over the sum of
their per-call times; with no such layer it falls back to the whole M = 1
set, and the ncu traffic record is quoted only for the k_stream form."""
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


def test_units_by_hand():
    # 70B gate (8192 -> 28672, r = 256), one token:
    # 58720256 + 29360128 + 3670016 + 4194304 + 14680064 + 16384 + 57344
    assert bench.algorithmic_bytes(8192, 28672, 256, 1) == 110698496
    # 70B k (8192 -> 1024): 2097152 + 1048576 + 131072 + 4194304 + 524288 + 16384 + 2048
    assert bench.algorithmic_bytes(8192, 1024, 256, 1) == 8013824
    # the same with 4-bit adapters: weights 3276800, L 16 x 64 blocks of 1056 B,
    # R 64 tiles of (16 x 128 + 2 x 32) B, X 16384, Y 2048
    assert bench.algorithmic_bytes_q4(8192, 1024, 256, 1) == 3276800 + 1081344 + 135168 + 16384 + 2048
    # 70B gate, 4096 tokens: 2 x 4096 x 28672 x 4096 kept + 2 x 4096 x 256 x 36864 adapter
    assert bench.kept_flops(8192, 28672, 256, 4096) == 962072674304 + 77309411328
