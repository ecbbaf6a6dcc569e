"""The decode benchmark's algorithmic HBM bytes per step, against a count
done by hand for the 350M workload (bf16 weights, 20 layers, d 1024, 16 heads
of 64, SwiGLU 2730, vocab 32000, batch 8)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_decode_bytes_350m():
    import bench
    from synth import get_config
    cfg = get_config("c5")
    total, weights, kv = bench.decode_bytes(cfg, 1023)
    d, L, h, V, B = 1024, 20, 2730, 32000, 8
    per_layer = d * 3 * d + d * d + 2 * d * h + h * d  # q|k|v, o, W1|W3, W2
    assert weights == (L * per_layer + d * V) * 2
    # keys and values of positions 0..1023 read, the new row of q|k|v written
    assert kv == L * B * (1024 * 2 * d + 3 * d) * 2
    assert total == weights + kv + B * d * 4 + (2 * L + 1) * d * 4 + B * V * 4
