"""Pins of the recache and FP8 oracles.

LongLive review, 'KV Recache' (cache rebuilt from the generated frames with the
new prompt); OCP OFP8 E4M3 format for the FP8 cache."""
import numpy as np
import pytest
import torch

from oracle import fp8, recache, rope


def test_rmsnorm_textbook():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((6, 48)) * 3
    g = rng.uniform(0.5, 1.5, 48)
    y = recache.rmsnorm(x, g, 0.0)
    assert np.allclose(np.sqrt(np.mean((y / g) ** 2, axis=-1)), 1.0, rtol=1e-13)
    # library cross-check
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (48,), torch.from_numpy(g), eps=1e-6).numpy()
    assert np.allclose(recache.rmsnorm(x, g, 1e-6), ref, rtol=1e-12, atol=1e-12)
    # eps matters for small rows: the all-zero row stays zero
    assert np.all(recache.rmsnorm(np.zeros((1, 4)), np.ones(4), 1e-6) == 0)


def test_recache_frame_composition():
    rng = np.random.default_rng(1)
    H, D, gh, gw, dm = 2, 16, 2, 3, 20
    pairs = (4, 2, 2)
    om = rope.head_frequencies(H, pairs, 10000.0)
    x = rng.standard_normal((gh * gw, dm))
    wk = rng.standard_normal((dm, H * D)) / np.sqrt(dm)
    wv = rng.standard_normal((dm, H * D)) / np.sqrt(dm)
    g = rng.uniform(0.5, 1.5, H * D)
    k, v = recache.recache_frame(x, wk, wv, g, 1e-6, 41, H, D, gh, gw, om, pairs, t_offset=7)
    kp = (torch.from_numpy(x) @ torch.from_numpy(wk)).numpy()
    assert np.allclose(v.reshape(gh * gw, -1), (torch.from_numpy(x) @ torch.from_numpy(wv)).numpy(), rtol=1e-12)
    kn = kp / np.sqrt((kp ** 2).mean(-1, keepdims=True) + 1e-6) * g
    # undo the rotation: R(-pos) R(pos) = I, so k rotated back equals the normalised projection
    t, r, c = rope.token_positions(41, gh, gw, 7)
    back = rope.rope_3d(k, -t, -r, -c, om, pairs)
    assert np.allclose(back.reshape(gh * gw, -1), kn, rtol=1e-12, atol=1e-12)


def test_e4m3_golden(golden):
    g = golden("e4m3.json")
    for code, val in g["codes"].items():
        assert fp8.e4m3_decode(int(code, 16)) == val
    for code in g["nan_codes"]:
        assert np.isnan(fp8.e4m3_decode(int(code, 16)))
    for c in g["encode"]:
        assert int(fp8.e4m3_encode([c["x"]])[0]) == int(c["code"], 16), c


def test_e4m3_decode_matches_library_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = fp8.e4m3_table()
    both_nan = np.isnan(lib) & np.isnan(ours)
    assert np.all(both_nan | (lib == ours))
    assert np.array_equal(np.isnan(lib), np.isnan(ours))


def test_e4m3_encode_roundtrip_and_nearest():
    tab = fp8.e4m3_table()
    finite = [c for c in range(256) if not np.isnan(tab[c])]
    # every finite code encodes back to itself (0x80 = -0.0 included)
    enc = fp8.e4m3_encode(np.array([tab[c] if c != 0x80 else -0.0 for c in finite]))
    assert list(enc) == finite
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(4000) * 50, rng.uniform(-0.02, 0.02, 2000)])
    codes = fp8.e4m3_encode(x)
    got = np.abs(fp8.e4m3_decode_array(codes) - x)
    vals = tab[finite]
    best = np.min(np.abs(x[:, None] - vals[None, :]), axis=1)
    assert np.allclose(got, np.minimum(best, got), atol=0) and np.all(got <= best + 1e-300)
    # and it agrees with the library's round-to-nearest-even cast inside the finite range
    lib = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(lib, codes)


def test_quantize_rows():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((10, 128))
    x[3] = 0.0
    codes, scale = fp8.quantize_rows(x)
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    deq = fp8.dequantize_rows(codes, scale)
    # the row max maps to exactly +-448
    i = np.argmax(np.abs(x[0]))
    assert abs(fp8.e4m3_decode(codes[0, i])) == 448.0
    # relative error bound of E4M3 (3 mantissa bits): half an ulp = 2^-4 of the value for normals
    big = np.abs(x) > 2.0 ** -6 * scale[:, None] * 8
    assert np.all(np.abs(deq - x)[big] <= 2.0 ** -4 * np.abs(x)[big] + 1e-15)
