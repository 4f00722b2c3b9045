"""Pins for the oracle's skin check and the synthetic dynamics stand-in."""
import numpy as np


def test_no_motion_no_rebuild(oracle):
    pos = np.random.default_rng(1).random((100, 3)).astype(np.float32) * 30
    m, rb = oracle.skin_check(pos, pos, [30.0, 30.0, 30.0], 1.0)
    assert m == 0.0 and rb is False


def test_exactly_half_skin_is_not_a_rebuild(oracle):
    # skin 1.0 -> h = 0.5, h^2 = 0.25 exactly; the rule is strict (>).
    ref = np.full((10, 3), 1.0, np.float32)
    pos = ref.copy()
    pos[3, 0] = 1.5
    m, rb = oracle.skin_check(pos, ref, [10.0, 10.0, 10.0], 1.0)
    assert m == 0.25 and rb is False
    pos[3, 0] = float(np.nextafter(np.float32(1.5), np.float32(2)))
    m, rb = oracle.skin_check(pos, ref, [10.0, 10.0, 10.0], 1.0)
    assert m > 0.25 and rb is True


def test_displacement_across_the_boundary_is_min_image(oracle):
    ref = np.array([[9.9, 5.0, 5.0]], np.float32)
    pos = np.array([[0.2, 5.0, 5.0]], np.float32)  # moved +0.3 through the face
    m, rb = oracle.skin_check(pos, ref, [10.0, 10.0, 10.0], 1.0)
    assert abs(m - 0.09) < 1e-5 and rb is False


def test_max_over_atoms(oracle):
    rng = np.random.default_rng(2)
    ref = rng.random((500, 3)).astype(np.float32) * 20
    d = rng.uniform(-0.2, 0.2, (500, 3)).astype(np.float32)
    pos = (ref + d).astype(np.float32)
    m, rb = oracle.skin_check(pos, ref, [20.0, 20.0, 20.0], 1.0)
    exact = ((pos.astype(np.float64) - ref) ** 2).sum(axis=1).max()
    assert abs(m - exact) < 1e-6 and rb is False


def test_displacement_statistics_and_determinism(oracle):
    sig = 0.02
    vals = np.array([oracle.displacement(1234, 7, a, ax, sig)
                     for a in range(4000) for ax in range(3)])
    assert abs(vals.mean()) < 3 * sig / np.sqrt(vals.size) * 1.5
    assert abs(vals.std() / sig - 1.0) < 0.03
    # Irwin-Hall(4) support: |g| <= 2*65535 units of A
    A = float(np.float32(sig * np.sqrt(3.0) / 65536.0))
    assert np.abs(vals).max() <= 131070 * A * (1 + 1e-6)
    assert oracle.displacement(1234, 7, 5, 1, sig) == oracle.displacement(1234, 7, 5, 1, sig)
    assert oracle.displacement(1234, 7, 5, 1, sig) != oracle.displacement(1234, 8, 5, 1, sig)
    # every value is fl(g * A) for an integer g (exact integer sum, one product)
    import fp32model as m32
    for v in vals[:500]:
        g = round(v / A)
        assert abs(g) <= 131070 and m32.mul(float(g), A) == float(np.float32(v))


def test_md_loop_first_rebuild_in_expected_range(oracle):
    """Sanity (not a pin): for 59k atoms at sigma 0.02, the first rebuild
    comes when the largest 3-D walk passes 0.5 A, around step 20-40."""
    from neighbor_list_construction_b200 import workloads
    w = workloads.make("lattice60k")
    dec, final, ref = oracle.md_decisions(w.pos, w.box, w.skin, 99, 0.02, 50)
    first = int(np.argmax(dec)) + 1 if dec.any() else None
    assert first is not None and 12 <= first <= 45
    # after the last rebuild ref holds the positions of that step
    last = int(np.nonzero(dec)[0][-1]) + 1
    p = w.pos.copy()
    for t in range(1, last + 1):
        p = oracle.displace(p, 99, t, 0.02)
    np.testing.assert_array_equal(ref[:, :3], p[:, :3])
    np.testing.assert_array_equal(final[:, :3], _walk(oracle, w.pos, 99, 50)[:, :3])


def _walk(oracle, pos, seed, steps):
    p = pos.copy()
    for t in range(1, steps + 1):
        p = oracle.displace(p, seed, t, 0.02)
    return p
