"""Pins of the oracle's log-mel front-end against library routines, closed
forms and invariants (CPU only).

The front-end is defined by the MOSS-Transcribe-preview-2B-GGUF card,
Architecture table "Audio" row (16 kHz, 128 mel bins, n_fft=400, hop=160,
matching WhisperFeatureExtractor), and its Non-obvious gotchas (trailing STFT
frame dropped, n_samples/hop frames).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def test_dft_matches_numpy_rfft():
    rng = np.random.default_rng(7)
    for n_samples in (1600, 16000 + 160 * 3):
        x = rng.normal(size=n_samples)
        p = oracle.power_spectrum(x, 400, 160)
        frames = oracle.frame_signal(x, 400, 160)[:-1] * oracle.hann_periodic(400)
        ref = np.abs(np.fft.rfft(frames, axis=1)) ** 2
        assert p.shape == ref.shape == (n_samples // 160, 201)
        np.testing.assert_allclose(p, ref, rtol=1e-10, atol=1e-9)


def test_hann_is_periodic_numpy():
    # numpy.hanning is the symmetric window of length N+1; its first N points
    # are the periodic window of length N.
    np.testing.assert_allclose(oracle.hann_periodic(400), np.hanning(401)[:-1], atol=1e-15)
    np.testing.assert_allclose(oracle.hann_periodic(400),
                               torch.hann_window(400, periodic=True, dtype=torch.float64).numpy(),
                               atol=1e-15)


def test_parseval_one_sided():
    # sum (w x)^2 = (1/N) (|X_0|^2 + 2 sum_{k=1}^{N/2-1} |X_k|^2 + |X_{N/2}|^2)
    rng = np.random.default_rng(3)
    x = rng.normal(size=3200)
    p = oracle.power_spectrum(x, 400, 160)
    wx = oracle.frame_signal(x, 400, 160)[:-1] * oracle.hann_periodic(400)
    lhs = (wx ** 2).sum(axis=1)
    rhs = (p[:, 0] + 2.0 * p[:, 1:200].sum(axis=1) + p[:, 200]) / 400.0
    np.testing.assert_allclose(lhs, rhs, rtol=1e-11)


def test_bin_centred_cosine_stays_in_main_lobe():
    # A unit cosine at exactly bin k0 under a periodic Hann window has all of
    # its one-sided energy in bins k0-1, k0, k0+1: |X|^2 = (N/8)^2, (N/4)^2, (N/8)^2.
    k0, n = 37, 400
    t = np.arange(16000)
    x = np.cos(2 * math.pi * k0 * t / n)
    p = oracle.power_spectrum(x, n, 160)
    mid = p[p.shape[0] // 2]
    assert mid[k0] == pytest.approx((n / 4) ** 2, rel=1e-9)
    assert mid[k0 - 1] == pytest.approx((n / 8) ** 2, rel=1e-9)
    assert mid[k0 + 1] == pytest.approx(mid[k0 - 1], rel=1e-9)
    others = np.delete(mid, [k0 - 1, k0, k0 + 1])
    assert others.max() < 1e-18 * mid[k0] + 1e-12


def test_frame_count_is_n_over_hop():
    for n in (16000, 480000, 16000 * 7):
        x = np.zeros(n)
        x[::97] = 1.0
        assert oracle.power_spectrum(x, 400, 160).shape[0] == n // 160
        assert oracle.log_mel(x, 128).shape == (128, n // 160)


@pytest.mark.parametrize("n_mels", [128, 80])
def test_filterbank_matches_torchaudio(n_mels):
    import torchaudio
    ref = torchaudio.functional.melscale_fbanks(201, 0.0, 8000.0, n_mels, 16000,
                                                norm="slaney", mel_scale="slaney").double().numpy()
    fb = oracle.mel_filterbank(201, n_mels)
    np.testing.assert_allclose(fb, ref, atol=1e-6)
    assert (fb > 0).sum(axis=0).min() >= 1          # no empty filter
    nnz = int((fb > 0).sum())
    assert nnz == {128: 394, 80: 391}[n_mels]


def test_slaney_scale_closed_forms():
    assert oracle.hz_to_mel_slaney(1000.0) == pytest.approx(15.0)
    assert oracle.hz_to_mel_slaney(600.0) == pytest.approx(9.0)
    assert oracle.hz_to_mel_slaney(6400.0) == pytest.approx(15.0 + 27.0)
    m = np.linspace(0, 60, 41)
    np.testing.assert_allclose(oracle.hz_to_mel_slaney(oracle.mel_to_hz_slaney(m)), m, atol=1e-12)


@pytest.mark.parametrize("n_mels,seed,n", [(128, 0, 16000), (80, 5, 32000), (128, 11, 48000)])
def test_log_mel_matches_whisper_feature_extractor(n_mels, seed, n):
    from transformers import WhisperFeatureExtractor
    x = synth.pcm_clip(n, seed)
    fe = WhisperFeatureExtractor(feature_size=n_mels)
    ref = fe(x, sampling_rate=16000, return_tensors="np", padding="longest")["input_features"][0]
    out = oracle.log_mel(x, n_mels)
    assert out.shape == ref.shape == (n_mels, n // 160)
    assert np.abs(out - ref).max() < 1e-4
    ref64 = fe._np_extract_fbank_features(x[None].astype(np.float64), "cpu")[0]
    assert np.abs(out - ref64).max() < 1e-6


def test_log_mel_clamp_and_scale():
    x = synth.pcm_clip(16000, 2)
    out = oracle.log_mel(x, 128)
    m = (out.max() * 4.0) - 4.0              # clip max of log10 mel
    assert out.min() >= (m - 8.0 + 4.0) / 4.0 - 1e-12


def test_silent_frames_equal_clamp_floor():
    # Speech-like long form: fully silent frames sit at the clamp, (m - 4) / 4.
    x = synth.pcm_clip(16000 * 20, 3000, speech_like=True)
    out = oracle.log_mel(x, 128)
    m = out.max() * 4.0 - 4.0
    frames = oracle.frame_signal(x, 400, 160)[:-1]
    silent = np.where(np.all(frames == 0.0, axis=1))[0]
    assert silent.size > 0
    np.testing.assert_array_equal(out[:, silent], np.full((128, silent.size), (m - 8.0 + 4.0) / 4.0))
