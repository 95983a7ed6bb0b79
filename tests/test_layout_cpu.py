"""The value-code layout of wushkv.h (16-position groups laid out for the decode's PV
operand), as the test harness converts it: a bijection between (group position, 16-bit
chunk) and the group's 16-bit halves; the four words a decode lane loads pair positions
(t4, t4 + 8) and (t4 + 4, t4 + 12) and sit together, lanes in order; round trips."""
import numpy as np
import pytest

from tests import harness as H


@pytest.mark.parametrize("bits", [2, 4])
def test_value_group_index_is_a_bijection(bits):
    idx = H._vgroup_index(bits)
    assert idx.shape == (16, 8 * bits)
    assert sorted(idx.ravel().tolist()) == list(range(16 * 8 * bits))


@pytest.mark.parametrize("bits", [2, 4])
def test_decode_lane_words_are_adjacent(bits):
    idx = H._vgroup_index(bits)
    for g in range(8):
        for t4 in range(4):
            for ws in range(2 if bits == 4 else 1):
                c = 4 * g + 2 * ws if bits == 4 else 2 * g
                first_word = (512 * ws + 64 * g + 16 * t4) // 4
                # words: (pair t4, chunk c), (pair t4+4, chunk c), (pair t4, c+1), (pair t4+4, c+1)
                for k, (t, cc) in enumerate([(t4, c), (t4 + 4, c), (t4, c + 1), (t4 + 4, c + 1)]):
                    assert idx[t, cc] == 2 * (first_word + k)          # position t: low half
                    assert idx[t + 8, cc] == 2 * (first_word + k) + 1  # position t + 8: high half


@pytest.mark.parametrize("bits", [2, 4])
def test_value_layout_round_trip(bits):
    rng = np.random.default_rng(bits)
    rows = rng.integers(0, 256, (2, 3, 128, 16 * bits), dtype=np.uint8)
    groups = H.v_groups_from_rows(rows, bits)
    assert groups.shape == rows.shape
    assert np.array_equal(H.v_rows_from_groups(groups, bits), rows)
    # one record changed -> only its own group changes
    rows2 = rows.copy()
    rows2[1, 2, 37] ^= 0xFF
    diff = np.nonzero((H.v_groups_from_rows(rows2, bits) != groups).any(axis=-1))
    assert set(diff[2].tolist()) <= set(range(32, 48))
