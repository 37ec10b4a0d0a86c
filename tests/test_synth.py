"""The seeded input generator: published SplitMix64 outputs and the recipe."""
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        seed, vals = line.split(":")
        out[int(seed)] = [int(v) for v in vals.split()]
    return out


def test_splitmix64_published_outputs():
    for seed, vals in _golden().items():
        assert synth.splitmix64(seed, len(vals)) == vals


def test_counter_form_matches_sequential():
    k = synth.key(7, 1)
    seq = synth.splitmix64(k, 100)
    assert synth.u64_stream(k, 100).tolist() == seq


def test_trit_distribution_and_determinism():
    T = synth.trits(0, 300, 1000, p0=0.2)
    assert T.dtype == np.int8 and set(np.unique(T).tolist()) <= {-1, 0, 1}
    f0 = (T == 0).mean()
    assert abs(f0 - 0.2) < 0.01
    assert abs((T == 1).mean() - (T == -1).mean()) < 0.01
    assert np.array_equal(T, synth.trits(0, 300, 1000, p0=0.2))
    assert not np.array_equal(T, synth.trits(1, 300, 1000, p0=0.2))
    # a strided destination holds the same values
    buf = np.full((300, 1024), 9, dtype=np.int8)
    synth.trits(0, 300, 1000, p0=0.2, out=buf)
    assert np.array_equal(buf[:, :1000], T) and (buf[:, 1000:] == 9).all()


def test_normals_recipe():
    X = synth.normals(3, 64, 1001)
    assert abs(X.mean()) < 0.01 and abs(X.std() - 1.0) < 0.01
    # thread split does not change values: generate as one row and compare
    flat = synth.normals(3, 1, 64 * 1001).reshape(64, 1001)
    assert np.array_equal(flat, X)
    H = synth.activations(3, 64, 1001)
    assert H.dtype == np.float16 and np.array_equal(H, X.astype(np.float16))


def test_alpha_range():
    a = [synth.alpha_for(s) for s in range(200)]
    assert min(a) >= 0.01 and max(a) < 0.05
    assert synth.alpha_for(0, 0.02) == 0.02
