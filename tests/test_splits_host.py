"""The token-split count the library picks (CPU: read back through the encode's
workspace size, which holds one fp32 partial of M x (D + 2) per split and head).

The count minimises (waves of the SMs' CTA slots) x (tiles per CTA + a fixed
per-CTA cost): on the million-token step it stays at 37 splits per head
(592 CTAs, four full waves of 148 SMs); with few heads it does not round up
past a wave boundary (32 heads: 4 splits, 128 CTAs in one wave, where 5
splits would be 160 CTAs = 1.08 waves)."""
import pytest

import rank_latent_attention_b200 as flare


def _align256(x):
    return (x + 255) // 256 * 256


def _encode_splits(B, H, N, M, D):
    ws = flare.flare_encode_workspace_size(B, H, N, M, D, 1)
    for P in range(1, 4097):
        rows = B * H * P * M
        if _align256(rows * D * 4) + 2 * _align256(rows * 4) == ws:
            return P
    raise AssertionError(f"no split count matches workspace {ws}")


@pytest.mark.parametrize("shape,splits", [
    ((1, 16, 1 << 20, 256, 64), 37),   # million-token step: 592 CTAs, 4 waves
    ((4, 8, 11271, 128, 32), 4),       # 32 heads: one wave of 128 CTAs
    ((8, 8, 972, 64, 16), 2),          # 64 heads, 16 tiles: 128 CTAs
    ((32, 8, 4096, 256, 32), 1),       # 256 heads: 1.73 waves whatever the split
])
def test_encode_split_count(shape, splits):
    assert _encode_splits(*shape) == splits
    # the host query reports the same count (1: the encode writes its result, no merge)
    B, H, N = shape[:3]
    assert flare.flare_encode_splits(B, H, N) == splits


def test_split_query_rejects_empty_shapes():
    assert flare.flare_encode_splits(0, 1, 10) == 0
    assert flare.flare_encode_splits(1, 0, 10) == 0
    assert flare.flare_encode_splits(1, 1, 0) == 0


def test_override_wins_and_is_clamped():
    old = flare.flare_set_split_override(3)
    try:
        assert _encode_splits(4, 8, 11271, 128, 32) == 3
        assert _encode_splits(1, 1, 100, 16, 16) == 2  # 2 tiles of 64 tokens
        assert flare.flare_encode_splits(4, 8, 11271) == 3
        assert flare.flare_encode_splits(1, 1, 100) == 2
    finally:
        flare.flare_set_split_override(old)
