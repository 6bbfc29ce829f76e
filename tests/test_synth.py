"""The seeded input generator: determinism, chunking independence, distribution."""
import numpy as np

from block_diffusion_lm_masked_b200 import synth
from oracle import dg_oracle as O


def test_normal_is_deterministic_and_chunk_independent(monkeypatch):
    a = synth.normal(5, 77, (3000,), 0.02, "bf16")
    monkeypatch.setattr(synth, "_CHUNK", 257)
    b = synth.normal(5, 77, (3000,), 0.02, "bf16")
    np.testing.assert_array_equal(a, b)
    c = synth.normal(5, 78, (3000,), 0.02, "bf16")
    assert (a != c).mean() > 0.9


def test_normal_moments_and_bf16_exactness():
    f = synth.normal(1234, 9, (200000,), 0.02, "f32").astype(np.float64)
    assert abs(f.mean()) < 3 * 0.02 / np.sqrt(2e5)
    assert abs(f.std() - 0.02) < 0.02 * 0.01
    bits = synth.normal(1234, 9, (200000,), 0.02, "bf16")
    wide = O.widen(bits)
    np.testing.assert_array_equal(O.round_bf16(f), O.round_bf16(wide))   # same draws, bf16-representable
    assert np.abs(wide - f).max() <= 0.02 * 6 * 2.0 ** -8


def test_tokens_uniform_in_range():
    t = synth.tokens(1235, 3, 100000, 1000)
    assert t.min() >= 0 and t.max() < 1000
    cnt = np.bincount(t, minlength=1000)
    assert cnt.min() > 40 and cnt.max() < 170


def test_mx8_experts_are_valid_deterministic_codes(monkeypatch):
    cfg = dict(n_layers=1, hidden=128, n_experts=2, expert_ffn=64)
    a = synth.mx8_experts(cfg)
    monkeypatch.setattr(synth, "_CHUNK", 1000)
    b = synth.mx8_experts(cfg)
    for name, shape in (("gate", (2, 64, 128)), ("up", (2, 64, 128)), ("down", (2, 128, 64))):
        codes, exps = a[0][name]
        assert codes.shape == shape and codes.dtype == np.uint8
        np.testing.assert_array_equal(codes, b[0][name][0])
        assert not np.isin(codes, [0x7F, 0xFF]).any()            # no NaN codes
        mag = codes & 0x7F
        assert mag.max() == 0x6F and 0.4 < (codes >> 7).mean() < 0.6
        assert exps.shape == shape[:-1] + (shape[-1] // 32,) and (exps == -12).all()
    assert (a[0]["gate"][0] != a[0]["up"][0]).mean() > 0.9


def test_nv4_experts_are_uniform_4bit_codes():
    cfg = dict(n_layers=1, hidden=128, n_experts=2, expert_ffn=64)
    a = synth.nv4_experts(cfg)
    for name, shape in (("gate", (2, 64, 128)), ("up", (2, 64, 128)), ("down", (2, 128, 64))):
        codes, sc, g = a[0][name]
        assert codes.shape == shape and codes.dtype == np.uint8 and codes.max() < 16
        cnt = np.bincount(codes.ravel(), minlength=16)
        assert cnt.min() > 0.8 * codes.size / 16 and cnt.max() < 1.2 * codes.size / 16
        assert sc.shape == shape[:-1] + (shape[-1] // 16,) and (sc == 0x28).all() and g == 2.0 ** -6
    np.testing.assert_array_equal(a[0]["gate"][0], synth.nv4_experts(cfg)[0]["gate"][0])


def test_low_precision_vocab_matrices():
    """The 8- and 4-bit output matrices: shapes, valid codes, their own streams (not the
    experts'), deterministic."""
    cfg = dict(n_layers=1, hidden=128, n_experts=2, expert_ffn=64, vocab=256)
    codes, exps = synth.mx8_vocab(cfg)
    assert codes.shape == (256, 128) and exps.shape == (256, 4) and (exps == -12).all()
    assert not np.isin(codes, [0x7F, 0xFF]).any() and (codes & 0x7F).max() == 0x6F
    np.testing.assert_array_equal(codes, synth.mx8_vocab(cfg)[0])
    c4, sc, g = synth.nv4_vocab(cfg)
    assert c4.shape == (256, 128) and c4.max() < 16 and sc.shape == (256, 8) and (sc == 0x28).all()
    cnt = np.bincount(c4.ravel(), minlength=16)
    assert cnt.min() > 0.8 * c4.size / 16 and cnt.max() < 1.2 * c4.size / 16
    # distinct streams from the experts' codes of the same shape
    e8 = synth.mx8_experts(dict(cfg, n_experts=1, expert_ffn=256))[0]["down"][0]   # [1][128][256]
    assert (e8[0].T != codes).mean() > 0.9
