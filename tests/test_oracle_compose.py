"""Pin of the oracle's composition from PCM (encode_clip, forward) against an
independent float64 torch composition (CPU).

The reference side never calls the oracle: the log-mel comes from
transformers.WhisperFeatureExtractor (the routine the MOSS-Transcribe-
preview-2B-GGUF card, Architecture "Audio" row, names), the stems from torch
conv2d / conv1d, the positions from a torch restatement of the sinusoid
table, and the tower, head and adapter from torch layer_norm / linear /
scaled_dot_product_attention / gelu / silu over the WHOLE clip with an
explicit window mask.  The oracle instead maps each attention window to the
conv chunks it needs and slices tokens out of them (encode_clip), so an
off-by-one in that mapping, in the window partition or in the batch stacking
(forward) fails here.  Architecture: MOSS card, Architecture table ("Audio
encoder" windowed block-diagonal attention, "Conv front-end", "Encoder head",
"Adapter"); the whisper-style stem: CrisperWhisper ONNX-export page, "What
this exports instead" and "Results".
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


# The feature extractor's own filterbank and STFT agree with the oracle's
# log-mel to ~1e-7 (tests/test_oracle_frontend.py); that difference, carried
# through the stem and tower, is the only one expected here.  A slicing or
# partition mistake moves rows by O(1).
RTOL = ATOL = 1e-6


def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def _fe_mel(x, n_mels):
    from transformers import WhisperFeatureExtractor
    fe = WhisperFeatureExtractor(feature_size=n_mels)
    return fe._np_extract_fbank_features(np.asarray(x, np.float64)[None], "cpu")[0]


def _sinusoids(length, d):
    half = d // 2
    inv = torch.exp(-math.log(10000.0) * torch.arange(half, dtype=torch.float64) / (half - 1))
    ang = torch.arange(length, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cat([torch.sin(ang), torch.cos(ang)], dim=1)


def _stem2d(mel, W, g):
    T = lambda n: W[n].double()
    outs = []
    for c0 in range(0, mel.shape[1], g.chunk_frames):
        x = _t(mel[:, c0:c0 + g.chunk_frames])[None, None]
        for i in (1, 2, 3):
            x = F.gelu(F.conv2d(x, T(f"conv{i}.w"), T(f"conv{i}.b"), stride=2, padding=1))
        _, c, f, t = x.shape
        y = F.linear(x[0].permute(2, 0, 1).reshape(t, c * f), T("conv_out.w"))
        outs.append(y + _sinusoids(t, g.d_model))
    return torch.cat(outs)


def _stem1d(mel, W, g):
    T = lambda n: W[n].double()
    x = F.gelu(F.conv1d(_t(mel)[None], T("conv1.w"), T("conv1.b"), stride=1, padding=1))
    x = F.gelu(F.conv1d(x, T("conv2.w"), T("conv2.b"), stride=2, padding=1))[0].T
    return x + _sinusoids(x.shape[0], g.d_model)


def _windows(n_tokens, w):
    w = w if w else n_tokens
    return [(a, min(a + w, n_tokens)) for a in range(0, n_tokens, w)]


def _tower(x, W, g, wins):
    T = lambda n: W[n].double()
    wid = torch.empty(x.shape[0], dtype=torch.long)
    for j, (a, b) in enumerate(wins):
        wid[a:b] = j
    mask = wid[:, None] == wid[None, :]
    H, dh = g.n_heads, g.head_dim
    sp = lambda z: z.reshape(-1, H, dh).transpose(0, 1)
    for l in range(g.n_layers):
        p = f"layers.{l}."
        h = F.layer_norm(x, (g.d_model,), T(p + "ln1.g"), T(p + "ln1.b"), g.ln_eps)
        q, k, v = (F.linear(h, T(p + n + ".w"), T(p + n + ".b")) for n in "qkv")
        a = F.scaled_dot_product_attention(sp(q), sp(k), sp(v), attn_mask=mask).transpose(0, 1).reshape(-1, g.d_model)
        x = x + F.linear(a, T(p + "o.w"), T(p + "o.b"))
        h = F.layer_norm(x, (g.d_model,), T(p + "ln2.g"), T(p + "ln2.b"), g.ln_eps)
        x = x + F.linear(F.gelu(F.linear(h, T(p + "fc1.w"), T(p + "fc1.b"))), T(p + "fc2.w"), T(p + "fc2.b"))
    h = F.layer_norm(x, (g.d_model,), T("ln_post.g"), T("ln_post.b"), g.ln_eps)
    if g.proj1_out:
        h = F.linear(F.gelu(F.linear(h, T("proj1.w"), T("proj1.b"))), T("proj2.w"), T("proj2.b"))
    if g.adapter_hidden:
        h = F.linear(F.silu(F.linear(h, T("adapter.gate.w"))) * F.linear(h, T("adapter.up.w")), T("adapter.down.w"))
    return h.numpy()


def torch_clip(pcm, W, g):
    """Whole-clip forward from PCM, composed of library routines only."""
    mel = _fe_mel(pcm, g.n_mels)
    x = _stem2d(mel, W, g) if g.stem == 0 else _stem1d(mel, W, g)
    return _tower(x, W, g, _windows(x.shape[0], g.window_tokens))


def _geom(**kw):
    base = synth.GEOMETRIES["tiny"].as_dict()
    base.update(dict(conv_ch=8, d_model=64, n_heads=2, head_dim=32, d_ffn=96, n_layers=1, proj1_out=64,
                     proj2_out=48, adapter_hidden=80, adapter_out=40))
    base.update(kw)
    return synth.Geometry(**base)


CASES = {
    # windows of two whole chunks
    "conv2d_w26": (_geom(window_tokens=26), 5),
    # windows that cut chunks (20 = 13 + 7): the chunk-to-token slicing is exercised
    "conv2d_w20": (_geom(window_tokens=20, n_layers=2), 5),
    # the MOSS window of 104 tokens over a 10 s clip (104 + 26)
    "conv2d_w104": (_geom(window_tokens=104), 10),
    # whisper-style stem, full attention and windowed
    "conv1d_full": (_geom(stem=1, n_mels=80, pos_mode=1, window_tokens=0, proj1_out=0, proj2_out=0,
                          adapter_hidden=0, adapter_out=0), 2),
    "conv1d_w30": (_geom(stem=1, n_mels=80, pos_mode=1, window_tokens=30), 2),
    # a short last chunk (730 frames: 7 chunks and 30 frames -> 95 tokens)
    "conv2d_short_chunk": (_geom(window_tokens=20, n_layers=2), 7.3),
    # a length that is not a whole number of hops (the extra samples only
    # enter the last frames through the reflect padding)
    "conv2d_odd_length": (_geom(window_tokens=26), 3.4567),
}


@pytest.mark.parametrize("case", list(CASES))
def test_encode_clip_from_pcm_matches_torch_composition(case):
    g, secs = CASES[case]
    W = synth.make_weights(g, 31, affine=True, std=0.1)
    pcm = synth.pcm_clip(int(round(16000 * secs)), 41)
    ref = torch_clip(pcm, W, g)
    full = oracle.encode_clip(pcm, W, g)
    assert full.shape == ref.shape
    np.testing.assert_allclose(full, ref, rtol=RTOL, atol=ATOL)
    # every window computed alone gives that window's rows of the whole clip
    for j, (a, b) in enumerate(_windows(ref.shape[0], g.window_tokens)):
        part = oracle.encode_clip(pcm, W, g, windows=[j])
        np.testing.assert_allclose(part, ref[a:b], rtol=RTOL, atol=ATOL)


def test_forward_stacks_independent_clips():
    g = _geom(window_tokens=20)
    W = synth.make_weights(g, 32, affine=True, std=0.1)
    pcm = np.stack([synth.pcm_clip(48000, 50), synth.pcm_clip(48000, 51)])
    out = oracle.forward(pcm, W, g)
    assert out.shape == (2, 39, g.adapter_out)
    for b in range(2):
        np.testing.assert_allclose(out[b], torch_clip(pcm[b], W, g), rtol=RTOL, atol=ATOL)


def _torch_stream(pcm, W, g):
    """Streaming reference from library routines: torch.stft (centred,
    reflect, periodic Hann, trailing frame dropped) and the torchaudio Slaney
    filterbank, each window's log-mel normalised by its own maximum, then the
    torch stem and tower over the window."""
    import torchaudio
    x = _t(pcm)
    spec = torch.stft(x, 400, 160, window=torch.hann_window(400, periodic=True, dtype=torch.float64),
                      center=True, pad_mode="reflect", return_complex=True)[:, :-1]
    fb = torchaudio.functional.melscale_fbanks(201, 0.0, 8000.0, g.n_mels, 16000, norm="slaney",
                                               mel_scale="slaney").double()
    lg = torch.log10(torch.clamp((spec.abs() ** 2).T @ fb, min=1e-10))     # [F, M]
    wf = g.window_tokens // 13 * g.chunk_frames
    outs = []
    for f0 in range(0, lg.shape[0], wf):
        w = lg[f0:f0 + wf]
        w = torch.maximum(w, w.max() - 8.0)
        xs = _stem2d(((w + 4.0) / 4.0).T.numpy(), W, g)
        outs.append(_tower(xs, W, g, _windows(xs.shape[0], 0)))
    return np.concatenate(outs)


def test_encode_stream_one_window_equals_encode_clip():
    # a stream that fits in one window has the clip's maximum: the offline result
    g = _geom(window_tokens=26)                     # windows of 2 chunks = 200 frames
    W = synth.make_weights(g, 33, affine=True, std=0.1)
    pcm = synth.pcm_clip(31000, 42)                 # 193 frames
    np.testing.assert_allclose(oracle.encode_stream(pcm, W, g), oracle.encode_clip(pcm, W, g), rtol=1e-12, atol=1e-12)


def test_encode_stream_matches_torch_composition():
    g = _geom(window_tokens=26, n_layers=2)         # windows of 200 frames
    W = synth.make_weights(g, 34, affine=True, std=0.1)
    pcm = synth.pcm_clip(16000 * 5 + 1234, 43, speech_like=True)  # 507 frames: windows 200, 200, 107
    out = oracle.encode_stream(pcm, W, g)
    assert out.shape[0] == 26 + 26 + 13 + 1
    np.testing.assert_allclose(out, _torch_stream(pcm, W, g), rtol=RTOL, atol=ATOL)
