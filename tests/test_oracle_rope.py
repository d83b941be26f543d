"""Pins of the RoPE / LoL-jitter oracle against closed forms and identities.

LoL review, 'Prerequisites: RoPE' (rotation matrix, theta_i = theta^(-2i/d),
relative-position identity) and 'Method steps' (per-head jittered base)."""
import math

import numpy as np
import pytest

import swa_workloads as W
from oracle import rope


def test_frequency_closed_forms(golden):
    g = golden("rope_frequencies.json")
    for c in g["cases"]:
        om = rope.band_frequencies(g["theta0"], c["pairs"])
        assert om[c["i"]] == pytest.approx(c["omega"], rel=1e-13)


def test_frequencies_geometric():
    # consecutive ratios are base^(-2/d) and the first entry is exactly 1
    for base, P in [(10000.0, 22), (2000.0, 21), (18000.0, 64)]:
        om = rope.band_frequencies(base, P)
        assert om[0] == 1.0
        r = om[1:] / om[:-1]
        assert np.allclose(r, base ** (-2.0 / (2 * P)), rtol=1e-13)
        assert np.all(np.diff(om) < 0)


def test_jitter_points_and_bounds(golden):
    g = golden("jitter.json")
    for c in g["cases"]:
        assert rope.jittered_base(g["theta0"], g["sigma"], [c["eps"]])[0] == pytest.approx(c["theta_hat"], rel=1e-15)
    eps = W.jitter_eps(12345, 4096).astype(np.float64)
    th = rope.jittered_base(g["theta0"], g["sigma"], eps)
    lo, hi = g["bounds"]
    assert th.min() >= lo and th.max() <= hi
    # eps ~ U[-1,1]: mean ~ 0, variance ~ 1/3
    assert abs(eps.mean()) < 0.05 and abs(eps.var() - 1 / 3) < 0.02


def test_splitmix64_known_answers():
    # published SplitMix64 reference outputs (state seeded with 1234567)
    s = 1234567
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    for w in want:
        s, z = W.splitmix64(s)
        assert z == w


def test_jitter_regenerated_from_seed():
    e1 = W.jitter_eps(7, 12)
    e2 = W.jitter_eps(7, 12)
    assert np.array_equal(e1, e2)
    # by hand from the generator definition: u = (z >> 11) * 2^-53, eps = 2u - 1
    s, z = W.splitmix64(7)
    assert e1[0] == np.float32(2.0 * ((z >> 11) * 2.0 ** -53) - 1.0)
    om = rope.head_frequencies(12, (22, 21, 21), 10000.0, 0.8, e1)
    for h in range(12):
        base = 10000.0 * (1 + 0.8 * float(e1[h]))
        assert om[h, 1] == pytest.approx(base ** (-2.0 / 44), rel=1e-13)
        # spatial bands keep theta0
        assert om[h, 22 + 1] == pytest.approx(10000.0 ** (-2.0 / 42), rel=1e-13)


def test_rotation_golden(golden):
    for c in golden("rope_rotation.json")["cases"]:
        y = rope.rotate_pairs(np.array(c["x"]), np.array([c["angle"]]))
        assert np.allclose(y, c["y"], atol=1e-14)


def test_rotation_is_complex_multiplication():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 16))
    ang = rng.uniform(-50, 50, (5, 8))
    y = rope.rotate_pairs(x, ang)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * ang)
    assert np.allclose(y[:, 0::2], z.real, atol=1e-12)
    assert np.allclose(y[:, 1::2], z.imag, atol=1e-12)


@pytest.mark.parametrize("sigma", [0.0, 0.8])
def test_relative_position_identity_3d(sigma):
    """<R(m)q, R(n)k> = <q, R(n-m)k> for every axis offset, per head."""
    rng = np.random.default_rng(1)
    H, D, pairs = 3, 64, (12, 10, 10)
    eps = W.jitter_eps(3, H) if sigma else None
    om = rope.head_frequencies(H, pairs, 10000.0, sigma, eps)
    q = rng.standard_normal((1, H, D))
    k = rng.standard_normal((1, H, D))
    for (m, n) in [((5, 1, 2), (2005, 3, 0)), ((0, 0, 0), (7, 29, 51)), ((131, 4, 4), (201, 4, 4))]:
        qm = rope.rope_3d(q, [m[0]], [m[1]], [m[2]], om, pairs)
        kn = rope.rope_3d(k, [n[0]], [n[1]], [n[2]], om, pairs)
        kd = rope.rope_3d(k, [n[0] - m[0]], [n[1] - m[1]], [n[2] - m[2]], om, pairs)
        lhs = np.einsum("thd,thd->h", qm, kn)
        rhs = np.einsum("thd,thd->h", q, kd)
        assert np.allclose(lhs, rhs, rtol=1e-10, atol=1e-10)


def test_norm_preserved_and_zero_position_identity():
    rng = np.random.default_rng(2)
    om = rope.head_frequencies(2, (22, 21, 21), 10000.0)
    x = rng.standard_normal((7, 2, 128))
    pos = rng.integers(0, 3000, (3, 7))
    y = rope.rope_3d(x, pos[0], pos[1], pos[2], om, (22, 21, 21))
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    y0 = rope.rope_3d(x, np.zeros(7), np.zeros(7), np.zeros(7), om, (22, 21, 21))
    assert np.array_equal(y0, x)


def test_sigma_zero_is_plain_rope():
    eps = W.jitter_eps(9, 4)
    a = rope.head_frequencies(4, (12, 10, 10), 10000.0, 0.0, eps)
    b = rope.head_frequencies(4, (12, 10, 10), 10000.0, 0.8, np.zeros(4))
    c = rope.head_frequencies(4, (12, 10, 10), 10000.0)
    assert np.array_equal(a, c) and np.array_equal(b, c)


def test_band_layout_by_hand():
    """Only the t band moves with t, only the h band with the row, only w with the column."""
    pairs = (12, 10, 10)
    om = rope.head_frequencies(1, pairs, 10000.0)
    x = np.ones((1, 1, 64))
    base = rope.rope_3d(x, [0], [0], [0], om, pairs)
    for axis, sl in [(0, slice(0, 24)), (1, slice(24, 44)), (2, slice(44, 64))]:
        p = [[0], [0], [0]]
        p[axis] = [3]
        y = rope.rope_3d(x, *p, om, pairs)
        changed = np.nonzero(np.abs(y - base).reshape(-1) > 1e-15)[0]
        assert changed.min() >= sl.start and changed.max() < sl.stop
        # first pair of the band turns by exactly pos * 1 radian
        j = sl.start
        assert y[0, 0, j] == pytest.approx(math.cos(3) - math.sin(3), abs=1e-14)
        assert y[0, 0, j + 1] == pytest.approx(math.sin(3) + math.cos(3), abs=1e-14)


def test_token_positions_row_major():
    t, r, c = rope.token_positions(7, 4, 6, t_offset=2000)
    assert np.all(t == 2007)
    assert list(r[:7]) == [0, 0, 0, 0, 0, 0, 1] and list(c[:7]) == [0, 1, 2, 3, 4, 5, 0]
    assert r[-1] == 3 and c[-1] == 5


def test_rope_frames_absolute_positions():
    """Every token of a block of frames turns by its own absolute position: the
    first pair of each band has frequency 1 (i = 0), so in frame g of the block
    its t pair turns by exactly (t_offset + g) * t_scale radians and its h and w
    pairs by the token's row and column, written out with math.cos / math.sin."""
    pairs = (12, 10, 10)
    H, gh, gw = 2, 2, 3
    N = gh * gw
    om = rope.head_frequencies(H, pairs, 10000.0)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((2, 3 * N, H, 64))
    first, t_offset, t_scale = 5, 100, 0.5
    y = rope.rope_frames(x, first, gh, gw, om, pairs, t_offset, t_scale)
    for b in range(2):
        for fi in range(3):
            for n in range(N):
                row = fi * N + n
                for j, ang in [(0, (t_offset + first + fi) * t_scale), (2 * 12, n // gw), (2 * 22, n % gw)]:
                    x0, x1 = x[b, row, :, j], x[b, row, :, j + 1]
                    c, s_ = math.cos(ang), math.sin(ang)
                    assert np.allclose(y[b, row, :, j], c * x0 - s_ * x1, atol=1e-12)
                    assert np.allclose(y[b, row, :, j + 1], s_ * x0 + c * x1, atol=1e-12)


# ---------------------------------------------------------------- phase coherence and position interpolation
def test_phase_coherence_special_values():
    """C(0) = 1, |C| <= 1, C(-D) = conj C(D); one component is a pure phase."""
    om = rope.band_frequencies(10000.0, 22)
    d = np.arange(-300, 301, dtype=np.float64)
    c = rope.phase_coherence(om, d)
    assert c[300] == pytest.approx(1.0, abs=1e-15)
    assert np.all(np.abs(c) <= 1.0 + 1e-12)
    assert np.allclose(c[::-1], np.conj(c), atol=1e-13)
    one = rope.phase_coherence(om[:1], d)
    assert np.allclose(one, np.cos(d) + 1j * np.sin(d), atol=1e-13)


def test_phase_coherence_harmonic_closed_form():
    """Components i*w0 (i = 0..K-1): the sum is a geometric series,
    C(D) = (1 - z^K) / (K (1 - z)) with z = e^{j w0 D}, and C = 1 whenever
    w0 D is a multiple of 2 pi (every component back in phase)."""
    K, w0 = 7, 0.37
    om = w0 * np.arange(K, dtype=np.float64)
    d = np.array([0.5, 1.0, 2.5, 10.0, 123.4])
    z = np.exp(1j * w0 * d)
    want = (1 - z ** K) / (K * (1 - z))
    assert np.allclose(rope.phase_coherence(om, d), want, atol=1e-13)
    period = 2 * math.pi / w0
    assert np.allclose(rope.phase_coherence(om, [period, 3 * period]), 1.0, atol=1e-12)


def test_phase_coherence_decorrelates_over_long_offsets():
    """For RoPE's geometric frequencies the components drift apart: averaged
    over many offsets, |C|^2 approaches 1/K (the components' phases behave as
    independent), far below the 1 at D = 0."""
    om = rope.band_frequencies(10000.0, 22)
    d = np.arange(1000, 200000, 7, dtype=np.float64)
    m2 = np.mean(np.abs(rope.phase_coherence(om, d)) ** 2)
    assert 0.5 / 22 < m2 < 2.0 / 22


def test_phase_coherence_jitter_breaks_alignment():
    """Heads with different jittered bases (LoL "Method steps") have different
    C(D) away from D = 0; with sigma = 0 every head has the same curve."""
    eps = W.jitter_eps(3, 4).astype(np.float64)
    om = rope.head_frequencies(4, (22, 21, 21), 10000.0, 0.8, eps)
    om0 = rope.head_frequencies(4, (22, 21, 21), 10000.0, 0.0, None)
    d = np.arange(1, 500, dtype=np.float64)
    cj = [rope.phase_coherence(om[h, :22], d) for h in range(4)]
    c0 = [rope.phase_coherence(om0[h, :22], d) for h in range(4)]
    assert all(np.array_equal(c0[0], c) for c in c0[1:])
    assert all(np.max(np.abs(cj[0] - c)) > 0.1 for c in cj[1:])


def test_position_interpolation_pins():
    """t_scale = 1 is plain RoPE; with t_scale = 1/2 frame 2f sits at the
    position of frame f; the relative identity holds at scaled positions."""
    rng = np.random.default_rng(5)
    pairs = (12, 10, 10)
    om = rope.head_frequencies(2, pairs, 10000.0)
    x = rng.standard_normal((1, 24, 2, 64))
    a = rope.rope_frames(x, 7, 4, 6, om, pairs)
    b = rope.rope_frames(x, 7, 4, 6, om, pairs, t_scale=1.0)
    assert np.array_equal(a, b)
    c = rope.rope_frames(x, 14, 4, 6, om, pairs, t_scale=0.5)
    assert np.allclose(c, a, atol=1e-14)
    # <R(s m) q, R(s n) k> = <q, R(s (n - m)) k> per pair
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    s, m, n = 0.3, 11.0, 29.0
    w = om[0, 0]
    lhs = rope.rotate_pairs(q[:2], s * m * w) @ rope.rotate_pairs(k[:2], s * n * w)
    rhs = q[:2] @ rope.rotate_pairs(k[:2], s * (n - m) * w)
    assert lhs == pytest.approx(rhs, abs=1e-12)
