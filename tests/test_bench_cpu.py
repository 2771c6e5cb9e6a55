"""bench.py's host-side arithmetic on the CPU: algorithmic bytes against
hand counts for the encoder and decoder shapes, the out-of-map statistics against a
closed form, the touched-bytes count against brute force, the clock
summary's reason decoding and the headline timing's entries."""
import numpy as np

import bench
from scale_deformable_attention_msdeformattn_b200 import workloads as wl


def test_algorithmic_bytes_match_hand_counts():
    # encoder float32: forward 79.65 MB, backward 136.54 MB (value + loc + A +
    # out; grad_out + value + loc + A + grad_value + grad_loc + grad_attn)
    nb = bench.algorithmic_bytes(wl.WORKLOADS["detr_encoder_f32"])
    assert abs(nb["forward"] / 1e6 - 79.65) < 0.01
    assert abs(nb["backward"] / 1e6 - 136.54) < 0.01
    # decoder bf16 with the value counted whole: 95.94 MB forward
    nb = bench.algorithmic_bytes(wl.WORKLOADS["detr_decoder_bf16"])
    assert abs(nb["forward"] / 1e6 - 95.94) < 0.01


def test_out_of_map_shares_closed_form():
    """One level, every sample a quarter pixel right of and below its own
    query's pixel centre: every sample is inside; exactly those in the last
    column or the last row have a corner outside, (H + W - 1) of H*W."""
    H, W = 7, 11
    w = wl.custom("stats", 2, [(H, W)], None, 3, 8, 2, "f32", "pixel_centre", 0.0)
    x = wl.generate(w, with_nonfused=False)
    x.sampling_offsets[...] = 0.25  # pixels of the level
    st = bench._input_stats(w, x)
    assert st["fully_outside"] == 0.0
    assert abs(st["any_corner_outside"] - (H + W - 1) / (H * W)) < 1e-4
    # every value row is touched (each pixel is its own query's corner)
    assert st["value_bytes_touched"] == st["value_bytes_whole"]


def test_touched_bytes_brute_force():
    w = wl.custom("touch", 1, [(9, 13), (5, 6)], 17, 2, 16, 3, "bf16", "uniform", 3.0)
    x = wl.generate(w, with_nonfused=False)
    st = bench._input_stats(w, x)
    rows = set()
    for q in range(w.num_queries):
        for m in range(w.M):
            for l, (H, W) in enumerate(w.levels):
                for k in range(w.K):
                    ref = x.reference_points[0, q].astype(np.float64)
                    off = x.sampling_offsets[0, q, m, l, k].astype(np.float64)
                    px = (ref[0] + off[0] / W) * W - 0.5
                    py = (ref[1] + off[1] / H) * H - 0.5
                    x0, y0 = int(np.floor(px)), int(np.floor(py))
                    for dy in (0, 1):
                        for dx in (0, 1):
                            xi, yi = x0 + dx, y0 + dy
                            if 0 <= xi < W and 0 <= yi < H:
                                rows.add((int(x.level_start_index[l]) + yi * W + xi) * w.M + m)
    row_bytes = w.D * 2
    sectors = {(r * row_bytes + b) // 32 for r in rows for b in range(0, row_bytes, 32)}
    assert st["value_bytes_touched"] == 32 * len(sectors)


def test_clock_summary_decodes_reasons():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.ok, c.max_mhz = True, 1965
    c.samples = [(1965, 0x1), (1950, 0x4), (1965, 0x4 | 0x40)]
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["sm_mhz_min"] == 1950
    assert set(s["reasons"]) == {"sw_power_cap", "hw_thermal_slowdown"}  # gpu_idle dropped


def test_dcn_workload_sizes_agree_with_the_oracle_and_the_library():
    """Output grid of each DCNv3 workload: the workload table, the oracle and
    the C ABI's msda_dcn_output_size agree; the draws are reproducible."""
    import ctypes

    import oracle
    from scale_deformable_attention_msdeformattn_b200 import _lib, build
    build.build()
    lib = _lib.load()
    for w in wl.DCN_WORKLOADS.values():
        ho, wo = w.out_hw
        assert (ho, wo) == oracle.dcn_output_size(w.H, w.W, w.kernel, w.stride, w.pad, w.dil)
        p = _lib.DcnProblem(w.N, w.H, w.W, w.G, w.C, w.kernel[0], w.kernel[1], w.stride[0],
                            w.stride[1], w.pad[0], w.pad[1], w.dil[0], w.dil[1], _lib.MSDA_F32, 0)
        a, b = ctypes.c_int64(0), ctypes.c_int64(0)
        assert lib.msda_dcn_output_size(ctypes.byref(p), ctypes.byref(a), ctypes.byref(b)) == 0
        assert (a.value, b.value) == (ho, wo)
    w = wl.custom_dcn("repro", 1, 6, 7, 2, 8, (3, 3))
    x1, x2 = wl.generate_dcn(w), wl.generate_dcn(w)
    assert np.array_equal(x1.offset, x2.offset) and np.array_equal(x1.mask, x2.mask)
    np.testing.assert_allclose(x1.mask.sum(-1), 1.0, rtol=1e-5)


def test_headline_timing_and_the_other_entry():
    """`value` times the graph-replayed step by default; the line carries the
    launched step beside it, or says that the capture failed."""
    assert bench.parse_args([]).headline == "graph"
    launched = (7.4, 38.0, [0.38, 0.37, 0.39])
    graph = (7.7, 37.0, [0.37, 0.37, 0.37])
    e = bench._other_timing("graph", True, 100, launched, graph)
    assert set(e) == {"launched"} and e["launched"]["value"] == 7.4
    assert e["launched"]["ms_per_step"] == 0.38 and e["launched"]["step_ms_p10_p50_p90"][1] == 0.38
    e = bench._other_timing("launched", True, 100, launched, graph)
    assert set(e) == {"graph"} and e["graph"]["value"] == 7.7
    e = bench._other_timing("launched", False, 100, launched, launched)
    assert "unavailable" in e["graph"]
