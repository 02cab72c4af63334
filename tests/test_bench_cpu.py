"""bench.py's host-side arithmetic (no GPU): the algorithmic work that the
rooflines divide by, the guard that ties the reported DRAM traffic to the
sources it was captured on, and the choice of peak denominators."""

import json

import bench


def test_forward_and_backward_flops_count_every_product():
    # forward: x W^T (m n k), x A^T (m k r), u' B^T (m r n) multiply-adds
    # backward: dY W (m n k), dY B (m n r), v' A (m r k), dA = v'^T x (m r k), dB = dY^T u' (m n r)
    m, n, k, r = 3, 5, 7, 2
    assert bench.fwd_flops(m, n, k, r) == 2 * (m * n * k + m * k * r + m * r * n)
    assert bench.bwd_flops(m, n, k, r) == 2 * (m * n * k + m * n * r + m * r * k + m * r * k + m * n * r)


def test_7b_mlp_step_figures():
    # the 7B-MLP projection (d_out 11008, d_in 4096), 4096 tokens, r 64: the
    # figures quoted beside the measurements
    f = bench.fwd_flops(4096, 11008, 4096, 64)
    b = bench.bwd_flops(4096, 11008, 4096, 64)
    assert round(f / 1e9, 2) == 377.29
    assert round((f + b) / 1e9, 1) == 762.5
    # quantizer: 2 B read + 0.5 B codes + 1/64 B scale codes + 4 B per 256 blocks written, per weight
    assert bench.quant_bytes(11008, 4096) == 2 * 11008 * 4096 + 11008 * 4096 // 2 + 11008 * 64 + 4 * 2752
    assert round(bench.quant_bytes(11008, 4096) / 1e6, 1) == 113.4


def test_decode_and_merge_bytes():
    # packed W + scale codes + group constants + A + B + x + y of one decode call
    assert bench.gemv_bytes(4096, 4096, 64) == 9_719_808
    assert bench.gemv_bytes(22016, 8192, 64) == 96_966_656
    # merge: packed W + scale codes + group constants + A + B read, bf16 W written
    assert bench.merge_bytes(11008, 4096, 64) == 115_370_752


def test_traffic_is_reported_only_for_the_sources_it_was_captured_on(monkeypatch):
    digest = bench.fwd_sources_digest()
    monkeypatch.setitem(bench.FWD_TRAFFIC, "sources_sha256", digest)
    monkeypatch.setitem(bench.FWD_TRAFFIC, "bytes", 123456)
    assert bench.fwd_traffic() == 123456
    monkeypatch.setitem(bench.FWD_TRAFFIC, "sources_sha256", "0" * 64)
    assert bench.fwd_traffic() is None
    monkeypatch.setitem(bench.FWD_TRAFFIC, "sources_sha256", digest)
    monkeypatch.setitem(bench.FWD_TRAFFIC, "bytes", None)
    assert bench.fwd_traffic() is None


def test_source_digest_follows_every_listed_source(monkeypatch, tmp_path):
    # a copy of the listed sources digests the same; changing one byte of any
    # of them changes the digest
    csrc = tmp_path / "bit_nf4_quantized_06_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.FWD_SOURCES:
        with open(bench.os.path.join(bench.ROOT, "bit_nf4_quantized_06_b200", "csrc", f), "rb") as src:
            (csrc / f).write_bytes(src.read())
    ref = bench.fwd_sources_digest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.fwd_sources_digest() == ref
    for f in bench.FWD_SOURCES:
        p = csrc / f
        orig = p.read_bytes()
        p.write_bytes(orig + b" ")
        assert bench.fwd_sources_digest() != ref, f
        p.write_bytes(orig)
    assert bench.fwd_sources_digest() == ref


def test_peaks_from_the_measured_file_else_the_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6540.2, "bf16_tflops": 1639.1}))
    peaks, src = bench.load_peaks()
    assert src == "measured"
    assert peaks == {"hbm_gbs": 6540.2, "bf16_tflops": 1639.1, "bf16_tflops_sustained": 1639.1}
