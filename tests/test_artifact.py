"""Offline reference-score artifact: per-pair sums joined by pair index, metadata
record checked before use (host logic, no GPU)."""
import json
import os

import numpy as np
import pytest

from preference_alignment_b200 import artifact as A


def _meta(**kw):
    m = A.metadata(d=4096, V=128256, L=2048, dtype="bf16", weights_fingerprint=0x1234abcd,
                   lib_version=100, dataset="synthetic", split="train")
    m.update(kw)
    return m


@pytest.mark.parametrize("layout", ["halves", "adjacent"])
def test_roundtrip_by_pair_index(tmp_path, layout):
    seq = -np.arange(1, 9, dtype=np.float64) * 10.5        # 4 pairs
    A.save(str(tmp_path), seq, layout, _meta())
    back = A.load(str(tmp_path), _meta(), layout=layout)
    np.testing.assert_array_equal(back, seq)
    # a subset of pairs, in another order, comes back joined by index
    rows = A.pair_rows(4, layout)
    sub = A.load(str(tmp_path), _meta(), pairs=[3, 1], layout=layout)
    c3, r3 = rows[3]
    c1, r1 = rows[1]
    sub_rows = A.pair_rows(2, layout)
    assert sub[sub_rows[0][0]] == seq[c3] and sub[sub_rows[0][1]] == seq[r3]
    assert sub[sub_rows[1][0]] == seq[c1] and sub[sub_rows[1][1]] == seq[r1]


def test_append_batches_and_refuse_a_different_setup(tmp_path):
    A.save(str(tmp_path), [-1.0, -2.0], "halves", _meta(), pair_offset=0)
    A.save(str(tmp_path), [-3.0, -4.0], "halves", _meta(), pair_offset=1, append=True)
    np.testing.assert_array_equal(A.load(str(tmp_path), _meta()), [-1.0, -3.0, -2.0, -4.0])
    with pytest.raises(A.ArtifactMismatch):
        A.save(str(tmp_path), [-5.0, -6.0], "halves", _meta(L=1024), pair_offset=2, append=True)


@pytest.mark.parametrize("change", [dict(weights_fingerprint="00000000deadbeef"), dict(L=4096),
                                    dict(dtype="f32"), dict(libdpo_version=101),
                                    dict(split="test")])
def test_mismatch_is_refused(tmp_path, change):
    A.save(str(tmp_path), [-1.0, -2.0], "halves", _meta())
    with pytest.raises(A.ArtifactMismatch):
        A.load(str(tmp_path), _meta(**change))


def test_missing_pairs_are_refused(tmp_path):
    A.save(str(tmp_path), [-1.0, -2.0], "halves", _meta())
    with pytest.raises(A.ArtifactMismatch):
        A.load(str(tmp_path), _meta(), pairs=[0, 5])


def test_files_are_plain_json(tmp_path):
    A.save(str(tmp_path), [-1.25, -2.5], "halves", _meta())
    lines = open(os.path.join(tmp_path, A.SCORES)).read().splitlines()
    assert json.loads(lines[0]) == {"pair": 0, "chosen": -1.25, "rejected": -2.5}
    meta = json.load(open(os.path.join(tmp_path, A.META)))
    assert meta["weights_fingerprint"] == "000000001234abcd" and meta["d"] == 4096
