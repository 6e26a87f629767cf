"""Host logic of the tactic table (the measured per-shape tile choice): shape
classes, overwrite, validation and clearing.  No GPU needed: lookup, store
and clear never touch the device."""
import pytest

import fp8_block_scaled_route_b200 as moe


@pytest.fixture(autouse=True)
def _clean_table():
    moe.moe_tactic_clear()
    yield
    moe.moe_tactic_clear()


def test_empty_table_misses():
    assert moe.moe_tactic_lookup(300, 512, 1024, 8, False) is None


def test_store_and_bucket_boundaries():
    # ceil(300 / 8) = 38 rows per expert: bucket (32, 64]
    moe.moe_tactic_store(300, 512, 1024, 8, False, 64)
    assert moe.moe_tactic_lookup(300, 512, 1024, 8, False) == 64
    assert moe.moe_tactic_lookup(257, 512, 1024, 8, False) == 64   # 33 rows per expert
    assert moe.moe_tactic_lookup(512, 512, 1024, 8, False) == 64   # 64 rows per expert
    assert moe.moe_tactic_lookup(256, 512, 1024, 8, False) is None  # 32: the bucket below
    assert moe.moe_tactic_lookup(513, 512, 1024, 8, False) is None  # 65: the bucket above
    # every other part of the class must match too
    assert moe.moe_tactic_lookup(300, 1024, 1024, 8, False) is None
    assert moe.moe_tactic_lookup(300, 512, 2048, 8, False) is None
    assert moe.moe_tactic_lookup(300, 512, 1024, 16, False) is None
    assert moe.moe_tactic_lookup(300, 512, 1024, 8, True) is None


def test_small_groups_share_one_bucket():
    moe.moe_tactic_store(8, 512, 1024, 8, True, 16)    # 1 row per expert
    assert moe.moe_tactic_lookup(64, 512, 1024, 8, True) == 16  # 8 rows per expert
    assert moe.moe_tactic_lookup(65, 512, 1024, 8, True) is None


def test_overwrite_and_clear():
    moe.moe_tactic_store(4096, 4096, 7168, 256, True, 64)
    moe.moe_tactic_store(4096, 4096, 7168, 256, True, 128)
    assert moe.moe_tactic_lookup(4096, 4096, 7168, 256, True) == 128
    moe.moe_tactic_clear()
    assert moe.moe_tactic_lookup(4096, 4096, 7168, 256, True) is None


def test_invalid_tiles_refused():
    assert moe.moe_tactic_store(300, 512, 1024, 8, False, 48, check=False) == moe.MOE_ERR_NO_TILE_CONFIG
    # a swapped tile stages K/128 x tile_m activation scales on chip: K too large for it
    big_k = 1 << 20
    assert moe.moe_tactic_store(300, 512, big_k, 8, False, 16, check=False) == moe.MOE_ERR_NO_TILE_CONFIG
    assert moe.moe_tactic_store(300, 512, big_k, 8, False, 128) == 0
    assert moe.moe_tactic_store(300, 0, 1024, 8, False, 64, check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_tactic_lookup(300, 512, 1024, 8, False) is None
