"""The seeded input generator: determinism, slicing and the workload recipe's
distributions (q, V ~ N(0,1); K = N(0,1) * exp(0.5 N(0,1)) per channel with 4
outlier channels x10 per KV head; ragged lengths uniform in [lo, hi])."""
import numpy as np
import torch

from quantized_attention_kvq_b200 import synth


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: published first outputs of the generator
    assert synth.u64(0, 1) == 0xE220A8397B1DCDAF
    assert synth.u64(0, 2) == 0x6E789E6AA1B965F4
    assert synth.u64(0, 3) == 0x06C45D188009454F


def test_deterministic_and_sliceable():
    s = synth.Synth(5, 2, 4, 2, 128, 64, "bf16")
    full = s.k_full()
    np.testing.assert_array_equal(full, synth.Synth(5, 2, 4, 2, 128, 64, "bf16").k_full())
    np.testing.assert_array_equal(full[1, 1, 10:30], s.k_slice(1, 1, 10, 20))
    np.testing.assert_array_equal(s.v_full()[0, 1, 5:9], s.v_slice(0, 1, 5, 4))
    assert not np.array_equal(full, synth.Synth(6, 2, 4, 2, 128, 64, "bf16").k_full())


def test_normal_moments():
    x = synth.normals(synth.stream_key(1, 1), 0, 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    assert abs((x ** 4).mean() - 3) < 0.1


def test_bf16_is_round_to_nearest_even_of_fp32():
    key = synth.stream_key(2, 3)
    f = synth.normals(key, 0, 10000, "f32")
    b = synth.normals(key, 0, 10000, "bf16")
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(b, want)


def test_key_channel_scales_and_outliers():
    s = synth.Synth(7, 1, 8, 8, 128, 16, "f32")
    for h in range(8):
        c = s.chscale[h]
        base = synth.channel_scales(synth.u64(synth.stream_key(7, synth.TAG_CHSCALE), h + 1), 128, n_outliers=0)
        out = np.nonzero(c != base)[0]
        assert len(out) == 4
        np.testing.assert_allclose(c[out], base[out] * 10, rtol=1e-15)
    logc = np.log(np.concatenate([s.chscale[h][s.chscale[h] == synth.channel_scales(
        synth.u64(synth.stream_key(7, synth.TAG_CHSCALE), h + 1), 128, n_outliers=0)] for h in range(8)]))
    assert abs(logc.std() - 0.5) < 0.06


def test_lengths_in_range():
    s = synth.Synth(9, 64, 64, 8, 128, 16384, "bf16", (1024, 16384))
    assert s.lens.min() >= 1024 and s.lens.max() <= 16384
    assert len(set(s.lens.tolist())) > 50


def test_dual_pair_inputs_are_seeded_inverse_transposes():
    tq, tk = synth.dual_pair(8, 3)
    tq2, tk2 = synth.dual_pair(8, 3)
    assert np.array_equal(tq, tq2) and np.array_equal(tk, tk2)  # same seed, same matrices
    assert not np.array_equal(tq, synth.dual_pair(9, 3)[0])
    assert tq.dtype == np.float32 and tq.shape == (3, 128, 128)
    for h in range(3):
        t = tq[h].astype(np.float64)
        # T^T T^-T = I up to the fp32 rounding of T^-T
        assert np.abs(t.T @ tk[h].astype(np.float64) - np.eye(128)).max() < 1e-5
        assert not np.allclose(t, t.T)  # a general pair, not an orthogonal one
        assert np.linalg.cond(t) < 20


def test_rope_frequencies():
    f = synth.rope_inv_freq(1.0e6)
    assert f.dtype == np.float32 and f.shape == (64,)
    assert f[0] == 1.0 and np.all(np.diff(f) < 0)
    np.testing.assert_allclose(f[32], 1.0e6 ** -0.5, rtol=1e-7)
