"""Pins of the oracle's convolution, attention, layer, head and adapter steps
against float64 torch library routines, closed forms and brute force (CPU).

Architecture: MOSS-Transcribe-preview-2B-GGUF card, Architecture table
("Audio encoder", "Conv front-end", "Encoder head", "Adapter" rows); the
whisper-small variant: CrisperWhisper ONNX-export page, "What this exports
instead" and "Results".
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def test_conv2d_matches_torch():
    rng = np.random.default_rng(0)
    for c_in, c_out, h, w in [(1, 8, 16, 10), (5, 7, 9, 13), (3, 4, 128, 100)]:
        x = rng.normal(size=(c_in, h, w))
        wt = rng.normal(size=(c_out, c_in, 3, 3))
        b = rng.normal(size=c_out)
        ref = F.conv2d(_t(x)[None], _t(wt), _t(b), stride=2, padding=1)[0].numpy()
        out = oracle.conv2d(x, wt, b)
        assert out.shape == ref.shape
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_conv1d_matches_torch():
    rng = np.random.default_rng(1)
    for stride in (1, 2):
        x = rng.normal(size=(6, 31))
        wt = rng.normal(size=(9, 6, 3))
        b = rng.normal(size=9)
        ref = F.conv1d(_t(x)[None], _t(wt), _t(b), stride=stride, padding=1)[0].numpy()
        np.testing.assert_allclose(oracle.conv1d(x, wt, b, stride=stride), ref, rtol=1e-12, atol=1e-12)


def test_elementwise_match_torch():
    x = np.linspace(-9, 9, 1001)
    np.testing.assert_allclose(oracle.gelu(x), F.gelu(_t(x)).numpy(), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(oracle.silu(x), F.silu(_t(x)).numpy(), rtol=1e-14, atol=1e-15)
    assert oracle.gelu(0.0) == 0.0
    rng = np.random.default_rng(2)
    y = rng.normal(size=(7, 33)) * 3 + 1.5
    g, b = rng.normal(size=33), rng.normal(size=33)
    np.testing.assert_allclose(oracle.layer_norm(y, g, b, 1e-5),
                               F.layer_norm(_t(y), (33,), _t(g), _t(b), 1e-5).numpy(), rtol=1e-12, atol=1e-12)


def test_sinusoids_closed_forms():
    for d in (256, 768, 1280):
        pe = oracle.sinusoids(1500, d)
        np.testing.assert_array_equal(pe[0], np.r_[np.zeros(d // 2), np.ones(d // 2)])
        np.testing.assert_allclose((pe ** 2).sum(axis=1), d / 2, rtol=1e-12)
        p = np.arange(1500)
        np.testing.assert_allclose(pe[:, 0], np.sin(p), atol=1e-12)            # first frequency 1
        np.testing.assert_allclose(pe[:, d // 2 - 1], np.sin(p * 1e-4), atol=1e-12)  # last 1/10000
        np.testing.assert_allclose(pe[:, d - 1], np.cos(p * 1e-4), atol=1e-12)


def test_token_counts_closed_form():
    g = synth.GEOMETRIES["moss"]
    for sec in (1, 2, 30, 600):
        assert oracle.token_count(g, 16000 * sec) == 13 * sec
    w = synth.GEOMETRIES["whisper_small"]
    for sec in (1, 30):
        assert oracle.token_count(w, 16000 * sec) == 16000 * sec // 320
    # a short last chunk of L frames gives ceil(ceil(ceil(L/2)/2)/2) tokens;
    # samples past the last whole hop add no frame
    assert oracle.token_count(g, 16000 + 160) == 13 + 1            # 101 frames
    assert oracle.token_count(g, 116800) == 7 * 13 + 4             # 730 frames: 30 -> 15 -> 8 -> 4
    assert oracle.token_count(g, 192160) == 12 * 13 + 1            # 1201 frames
    assert oracle.token_count(g, 16000 + 159) == 13
    assert oracle.token_count(w, 16000 + 160) == 51                # 101 frames -> ceil(101 / 2)
    with pytest.raises(ValueError):
        oracle.token_count(g, 200)                                 # reflect padding needs > 200 samples


def test_golden_shape_pins():
    with open(os.path.join(GOLDEN, "shape_pins.json")) as f:
        pins = json.load(f)["pins"]
    g, w = synth.GEOMETRIES["moss"], synth.GEOMETRIES["whisper_small"]
    by = {p["name"]: p["value"] for p in pins}
    # conv_out input width: 480 channels x 16 frequency rows
    assert synth.weight_specs(g)[6] == ("conv_out.w", (1280, by["conv_out_in"]), "w")
    assert oracle.token_count(w, 480000) == by["whisper_encoder_frames_30s"]
    assert oracle.token_count(g, 16000) == by["tokens_per_chunk"]
    assert oracle.token_count(g, 480000) == by["tokens_30s"]
    assert oracle.power_spectrum(np.ones(16000) * 0.1, 400, 160).shape[0] == by["mel_frames_1s"]


@pytest.mark.parametrize("name,n,batch,expect", [
    ("moss", 480000, 1, [0, 104, 208, 312, 390]),
    ("moss", 16000, 2, [0, 13, 26]),
    ("tiny", 16000, 1, [0, 13]),
])
def test_window_partition(name, n, batch, expect):
    assert oracle.window_partition(synth.GEOMETRIES[name], n, batch).tolist() == expect


def test_window_partition_counts():
    g = synth.GEOMETRIES["moss"]
    cu = oracle.window_partition(g, 480000, 16)
    assert len(cu) - 1 == 16 * 4 and cu[-1] == 6240
    cu = oracle.window_partition(g, 9600000, 1)
    assert len(cu) - 1 == 75 and set(np.diff(cu).tolist()) == {104}
    cu = oracle.window_partition(synth.GEOMETRIES["whisper_small"], 480000, 32)
    assert len(cu) - 1 == 32 and set(np.diff(cu).tolist()) == {1500}


def test_attention_blockdiag_equals_masked_and_sdpa():
    rng = np.random.default_rng(4)
    t, h, dh = 61, 3, 16
    q, k, v = (rng.normal(size=(t, h * dh)) for _ in range(3))
    cu = np.array([0, 13, 26, 40, 57, 61], dtype=np.int32)
    a = oracle.attention_windows(q, k, v, cu, h)
    mask = oracle.window_mask(cu, t)
    b = oracle.attention_masked(q, k, v, mask, h)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    qt, kt, vt = (_t(z).reshape(t, h, dh).transpose(0, 1) for z in (q, k, v))
    ref = F.scaled_dot_product_attention(qt[None], kt[None], vt[None], attn_mask=torch.from_numpy(mask))[0]
    np.testing.assert_allclose(a, ref.transpose(0, 1).reshape(t, h * dh).numpy(), rtol=1e-11, atol=1e-12)
    # A window of one token returns its own value row.
    cu1 = np.arange(t + 1, dtype=np.int32)
    np.testing.assert_allclose(oracle.attention_windows(q, k, v, cu1, h), v, atol=1e-14)


def _torch_encoder(x, W, g, cu):
    """float64 torch composition of library ops (layer_norm, linear, SDPA, gelu)."""
    T = lambda n: W[n].double()
    x = _t(x)
    mask = torch.from_numpy(oracle.window_mask(cu, x.shape[0]))
    H, dh = g.n_heads, g.head_dim
    for l in range(g.n_layers):
        p = f"layers.{l}."
        h = F.layer_norm(x, (g.d_model,), T(p + "ln1.g"), T(p + "ln1.b"), g.ln_eps)
        q, k, v = (F.linear(h, T(p + n + ".w"), T(p + n + ".b")) for n in "qkv")
        sp = lambda z: z.reshape(-1, H, dh).transpose(0, 1)
        a = F.scaled_dot_product_attention(sp(q), sp(k), sp(v), attn_mask=mask)
        a = a.transpose(0, 1).reshape(-1, g.d_model)
        x = x + F.linear(a, T(p + "o.w"), T(p + "o.b"))
        h = F.layer_norm(x, (g.d_model,), T(p + "ln2.g"), T(p + "ln2.b"), g.ln_eps)
        x = x + F.linear(F.gelu(F.linear(h, T(p + "fc1.w"), T(p + "fc1.b"))), T(p + "fc2.w"), T(p + "fc2.b"))
    h = F.layer_norm(x, (g.d_model,), T("ln_post.g"), T("ln_post.b"), g.ln_eps)
    if g.proj1_out:
        h = F.linear(F.gelu(F.linear(h, T("proj1.w"), T("proj1.b"))), T("proj2.w"), T("proj2.b"))
    if g.adapter_hidden:
        h = F.linear(F.silu(F.linear(h, T("adapter.gate.w"))) * F.linear(h, T("adapter.up.w")),
                     T("adapter.down.w"))
    return h.numpy()


def _small_geom(**kw):
    base = synth.GEOMETRIES["tiny"].as_dict()
    base.update(dict(conv_ch=8, d_model=64, n_heads=2, head_dim=32, d_ffn=96, proj1_out=64,
                     proj2_out=48, adapter_hidden=80, adapter_out=40))
    base.update(kw)
    return synth.Geometry(**base)


@pytest.mark.parametrize("layers", [1, 2])
def test_tiny_encoder_matches_torch_composition(layers):
    g = _small_geom(n_layers=layers)
    W = synth.make_weights(g, 99, affine=True, std=0.1)
    rng = np.random.default_rng(5)
    x = rng.normal(size=(50, g.d_model))
    cu = np.array([0, 13, 26, 39, 50], dtype=np.int32)
    out = oracle.encode_tokens(x, W, g, cu)
    ref = _torch_encoder(x, W, g, cu)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)


def test_whisper_style_encoder_matches_torch_composition():
    g = _small_geom(n_layers=1, proj1_out=0, proj2_out=0, adapter_hidden=0, adapter_out=0,
                    window_tokens=0, stem=1, pos_mode=1)
    W = synth.make_weights(g, 7, affine=True, std=0.1)
    x = np.random.default_rng(6).normal(size=(40, g.d_model))
    cu = np.array([0, 40], dtype=np.int32)
    np.testing.assert_allclose(oracle.encode_tokens(x, W, g, cu), _torch_encoder(x, W, g, cu),
                               rtol=1e-10, atol=1e-11)


def _torch_stem_conv2d(mel, W, g):
    T = lambda n: W[n].double()
    outs = []
    for c0 in range(0, mel.shape[1], g.chunk_frames):
        x = _t(mel[:, c0:c0 + g.chunk_frames])[None, None]
        for i in (1, 2, 3):
            x = F.gelu(F.conv2d(x, T(f"conv{i}.w"), T(f"conv{i}.b"), stride=2, padding=1))
        b, c, f, t = x.shape
        x = x.permute(0, 3, 1, 2).reshape(t, c * f)
        y = F.linear(x, T("conv_out.w"))
        outs.append(y.numpy() + oracle.sinusoids(t, g.d_model))
    return np.concatenate(outs)


def test_conv2d_stem_matches_torch():
    g = _small_geom()
    W = synth.make_weights(g, 3, affine=True, std=0.1)
    mel = oracle.log_mel(synth.pcm_clip(32000, 9), g.n_mels)
    out = oracle.stem_conv2d_chunked(mel, W, g)
    assert out.shape == (26, g.d_model)
    np.testing.assert_allclose(out, _torch_stem_conv2d(mel, W, g), rtol=1e-10, atol=1e-11)


def test_conv1d_stem_matches_torch():
    g = _small_geom(stem=1, n_mels=80, pos_mode=1, window_tokens=0)
    W = {"conv1.w": torch.randn(g.d_model, 80, 3, dtype=torch.float64) * 0.1,
         "conv1.b": torch.randn(g.d_model, dtype=torch.float64) * 0.1,
         "conv2.w": torch.randn(g.d_model, g.d_model, 3, dtype=torch.float64) * 0.1,
         "conv2.b": torch.randn(g.d_model, dtype=torch.float64) * 0.1}
    mel = oracle.log_mel(synth.pcm_clip(16000, 4), 80)
    x = F.gelu(F.conv1d(_t(mel)[None], W["conv1.w"], W["conv1.b"], padding=1))
    x = F.gelu(F.conv1d(x, W["conv2.w"], W["conv2.b"], stride=2, padding=1))[0].T.numpy()
    ref = x + oracle.sinusoids(x.shape[0], g.d_model)
    out = oracle.stem_conv1d(mel, W, g)
    assert out.shape == (50, g.d_model)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-11)


def test_window_sampling_is_exact():
    # Running only some windows of a clip gives exactly those rows of the full run.
    g = _small_geom(n_layers=1, window_tokens=26)
    W = synth.make_weights(g, 11, affine=True, std=0.1)
    pcm = synth.pcm_clip(16000 * 5, 21)
    full = oracle.encode_clip(pcm, W, g)
    cu = oracle.window_partition(g, pcm.shape[0], 1)
    part = oracle.encode_clip(pcm, W, g, windows=[1, 2])
    np.testing.assert_allclose(part, full[cu[1]:cu[3]], rtol=1e-12, atol=1e-12)


def test_splice_hand_example():
    # MOSS card, Architecture "Audio injection": placeholder rows take the
    # adapter frames in order, every other row its token embedding.
    P = 9
    table = np.arange(10 * 3, dtype=np.float64).reshape(10, 3)
    frames = np.array([[100.0, 101.0, 102.0], [200.0, 201.0, 202.0], [300.0, 301.0, 302.0]])
    ids = [3, P, P, 1, P, 0]
    out = oracle.splice_embeddings(ids, P, table, frames)
    expect = np.array([[9, 10, 11], [100, 101, 102], [200, 201, 202], [3, 4, 5], [300, 301, 302], [0, 1, 2]],
                      dtype=np.float64)
    np.testing.assert_array_equal(out, expect)
    with pytest.raises(ValueError):
        oracle.splice_embeddings([3, P, 1], P, table, frames)        # 1 placeholder, 3 frames
    with pytest.raises(ValueError):
        oracle.splice_embeddings([3, 12, P, P, P], P, table, frames)  # id 12 is not a row
