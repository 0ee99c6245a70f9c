"""Host-side pieces of Int4KVCache (no GPU): the compression ratio it reports is the
pages' 3.56x for int4 codes with one fp16 scale per 32 channels ("When Quantization
Is Free", gist.science/de/paper/2605.05699, "Wichtige Ergebnisse": 3.0-3.56x; 3.56 =
16 / (4 + 16/32)), 3.2x with groups of 16, and agrees with the oracle's byte count."""
import pytest

import oracle


def test_compression_ratio_matches_pages_and_oracle():
    from rotated_int4_kv_b200 import Int4KVCache

    assert Int4KVCache.compression_ratio(128, 32) == pytest.approx(16 / (4 + 16 / 32))
    assert Int4KVCache.compression_ratio(256, 32) == pytest.approx(3.5556, abs=1e-4)
    assert Int4KVCache.compression_ratio(128, 16) == pytest.approx(3.2)
    # int8 codes: 2D / (D + 2D/G)
    assert Int4KVCache.compression_ratio(128, 32, 8) == pytest.approx(256 / 136)
    assert Int4KVCache.compression_ratio(256, 16, 8) == pytest.approx(2 * 256 / oracle.compressed_bytes_per_vector(256, 16, 8))
    for D in (128, 256):
        for G in (16, 32):
            assert Int4KVCache.compression_ratio(D, G) == pytest.approx(2 * D / oracle.compressed_bytes_per_vector(D, G))


def test_cache_rejects_bad_sizes_before_touching_a_device():
    from rotated_int4_kv_b200 import Int4KVCache

    with pytest.raises(ValueError):
        Int4KVCache(0, 1, 1, 128, 16, ([1] * 128, [1.0] * 128), ([1] * 128, [1.0] * 128), device="cpu")
