"""Plant plausible mistakes in the oracle's FP8 mode (per-tile dequantisation
and the attention over it) and show that its pins catch each one (CPU only;
the oracle module is patched for the duration of one test)."""
import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

_real_tiles = oracle.dequant_e4m3_tiles
_real_fp8 = oracle.sdpa_fp8


def _tiles_off_by_one(raw, scales, tile=128):
    val = oracle.dequant_e4m3(raw)
    sc = np.asarray(scales, dtype=np.float64)
    tok_tile = np.minimum(np.arange(val.shape[2]) // (tile - 1), sc.shape[2] - 1)
    return val * sc[:, :, tok_tile][..., None]


def _tiles_first_head_only(raw, scales, tile=128):
    val = oracle.dequant_e4m3(raw)
    sc = np.asarray(scales, dtype=np.float64)
    tok_tile = np.arange(val.shape[2]) // tile
    return val * sc[:, :1, tok_tile][..., None]


def _tiles_first_tile_only(raw, scales, tile=128):
    val = oracle.dequant_e4m3(raw)
    sc = np.asarray(scales, dtype=np.float64)
    return val * sc[:, :, :1, None]


def _fp8_value_scale_ignored(q8, k8, v8, q_scale, k_scale, v_scale, causal, scale, tile=128, **kw):
    return _real_fp8(q8, k8, v8, q_scale, k_scale, np.ones_like(np.asarray(v_scale, dtype=np.float64)),
                     causal, scale, tile, **kw)


def _fp8_query_scale_on_keys(q8, k8, v8, q_scale, k_scale, v_scale, causal, scale, tile=128, **kw):
    q = oracle.dequant_e4m3(q8)
    k = _real_tiles(k8, k_scale, tile) * np.asarray(q_scale, dtype=np.float64).max()
    v = _real_tiles(v8, v_scale, tile)
    return oracle.sdpa(q, k, v, causal, scale)


MUTANTS = [
    ("tile_index_off_by_one", "dequant_e4m3_tiles", _tiles_off_by_one),
    ("scale_of_first_head_for_all", "dequant_e4m3_tiles", _tiles_first_head_only),
    ("scale_of_first_tile_for_all", "dequant_e4m3_tiles", _tiles_first_tile_only),
    ("value_scale_ignored", "sdpa_fp8", _fp8_value_scale_ignored),
    ("query_scale_moved_to_keys", "sdpa_fp8", _fp8_query_scale_on_keys),
]


@pytest.mark.parametrize("name,attr,fn", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_fp8_oracle_mutant_is_caught(monkeypatch, name, attr, fn):
    monkeypatch.setattr(oracle, attr, fn)
    caught = 0
    for pin in (pins.test_dequant_e4m3_tiles, pins.test_sdpa_fp8_scaling_and_tiles):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"mutant {name} passed every FP8 pin"


def test_fp8_pins_pass_on_the_real_oracle():
    pins.test_dequant_e4m3_tiles()
    pins.test_sdpa_fp8_scaling_and_tiles()
