"""The synthetic workloads have the sizes the pages print (CPU only).

tests/golden/cache_sizes.txt holds the printed numbers with their citations:
the Qwen3-32B cache of the TTAS-X2 page ("3. Experiments", "4. Memory
Analysis") and the live-migration block of the QATQ page ("Measured
evidence"). The workloads' shapes are pinned to them, as is the reading of
their units (GB = 10^9 bytes of keys plus values; "ratio vs raw" = coded bytes
over raw bytes, the inverse of the compression ratio this codec reports).
"""
import os

import kvgen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    out = {}
    for line in open(os.path.join(GOLDEN, "cache_sizes.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split("=", 1)
            out[k] = v
    return out


def test_qwen3_32b_cache_sizes():
    g = _golden()
    L, H, D = int(g["ttas_layers"]), int(g["ttas_kv_heads"]), int(g["ttas_head_dim"])
    for T in (4096, 16384, 32768, 65536):
        raw = 2 * L * H * T * D * 2  # keys and values, 2 bytes a value
        assert f"{raw / 1e9:.2f}" == g[f"ttas_fp16_gb_{T}"], T
    for name in ("transform-64x8x32768x128-bf16", "lossless-64x8x32768x128-bf16"):
        w = kvgen.WORKLOADS[name]
        assert (w.n_layers, w.n_heads, w.head_dim, w.n_tokens) == (L, H, D, 32768)
        assert f"{w.raw_bytes / 1e9:.2f}" == g["ttas_fp16_gb_32768"]
        assert w.slices_per_frame * w.n_tokens * w.head_dim * 2 == 64 << 20  # 64 MiB frames


def test_ttas_table_ratio_and_bits_disagree():
    """The page's 32k row: its ratio follows from the sizes, its bits per
    weight do not (16 / 1.59 is about 10, not 6.3). This codec reports both
    its allocated code bits and its total bits per value for that reason."""
    g = _golden()
    ratio = float(g["ttas_fp16_gb_32768"]) / float(g["ttas_compressed_gb_32768"])
    assert round(ratio, 1) == float(g["ttas_ratio"])
    assert abs(16.0 / float(g["ttas_bpw"]) - ratio) > 3.0


def test_migration_block_bytes_and_ratio_column():
    """The block is the workload's size exactly; the table's ratio column is
    transferred over raw bytes, within one unit of its last printed digit (the
    page truncates LZ4's 0.570997 to 0.5709 but rounds QATQ's 0.278254 to
    0.2783), and its reductions (43.0, 59.5, 72.2%) are one minus that,
    within a tenth of a point (LZ4's is 42.90%)."""
    g = _golden()
    raw = int(g["qatq_raw_bytes"])
    assert kvgen.WORKLOADS["lossless-8x8x1536x128-bf16"].raw_bytes == raw
    for codec, reduction in (("qatq_lz4", 43.0), ("qatq_zstd", 59.5), ("qatq", 72.2)):
        r = int(g[codec + "_bytes"]) / raw
        assert abs(r - float(g[codec + "_ratio"])) < 1e-4, codec
        assert abs(100 * (1 - r) - reduction) <= 0.1 + 1e-9, codec
