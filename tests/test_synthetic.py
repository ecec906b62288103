"""The seeded input generators: host twins agree bit for bit, and the inputs
have the structure the workloads call for (CPU only)."""
import numpy as np

import synthetic


def test_fast_host_generator_matches_numpy_definition():
    for sigma in (1.0, 0.02):
        for start in (0, 12345, 1 << 33):
            a = synthetic.gaussian_bf16(5, 3, (1 << 17,), sigma=sigma, start=start)
            b = synthetic.gaussian_bf16(5, 3, (1 << 17,), sigma=sigma, start=start, reference=True)
            assert np.array_equal(a, b)


def test_fast_path_with_outliers_matches_numpy_definition():
    a = synthetic.gaussian_bf16(0, 1, (512, 512), outlier_frac=0.001)
    b = synthetic.gaussian_bf16(0, 1, (512, 512), outlier_frac=0.001, reference=True)
    assert np.array_equal(a, b)
    a = synthetic.gaussian_bf16(2, 4, (256, 1024), sigma=0.02, outlier_frac=0.001)
    b = synthetic.gaussian_bf16(2, 4, (256, 1024), sigma=0.02, outlier_frac=0.001, reference=True)
    assert np.array_equal(a, b)


def test_normal_moments_and_slices():
    z = synthetic.normal_z(0, 1, 0, 1 << 20)
    assert abs(z.mean()) < 5e-3 and abs(z.var() - 1.0) < 5e-3
    full = synthetic.gaussian_bf16(1, 2, (1000,), reference=True)
    part = synthetic.gaussian_bf16(1, 2, (100,), start=400, reference=True)
    assert np.array_equal(full[400:500], part)


def test_outliers_exact_count():
    x = synthetic.gaussian_bf16(0, 1, (128, 512), outlier_frac=0.001)
    pos = synthetic.outlier_positions(0, 128 * 512)
    assert len(pos) == 65 and len(np.unique(pos)) == 65
    f = synthetic.bf16_bits_to_f32(x).reshape(-1)
    base = synthetic.bf16_bits_to_f32(synthetic.gaussian_bf16(0, 1, (128 * 512,), reference=True))
    assert np.array_equal(np.delete(f, pos), np.delete(base, pos))


def test_topk_routing_structure():
    r = synthetic.route_topk_softmax(0, 512, 64, 10)
    e = r["experts"]
    assert all(len(set(row)) == 10 for row in e)
    assert r["offsets"][-1] == 5120 and (np.diff(r["offsets"]) >= 0).all()
    for g in range(64):
        toks = r["row_index"][r["offsets"][g]:r["offsets"][g + 1]]
        assert (np.diff(toks) > 0).all()                     # ascending token id
        assert all(g in e[t] for t in toks)
    assert np.allclose(r["weights"].sum(1), 1.0)


def test_zipf_routing_is_skewed():
    r = synthetic.route_zipf_gumbel(7, 64, 384, 10)
    c = np.diff(r["offsets"])
    assert c.sum() == 640 and (c == 0).sum() > 100 and c.max() > 20
    assert all(len(set(row)) == 10 for row in r["experts"])


def test_mxfp4_generators():
    q = synthetic.mxfp4_codes(0, 9, 1 << 16)
    nib = np.concatenate([q & 15, q >> 4])
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.9 * counts.mean()
    e = synthetic.mxfp4_exponents(0, 10, 1 << 16, lo=-10)
    assert e.min() == 117 and e.max() == 124
