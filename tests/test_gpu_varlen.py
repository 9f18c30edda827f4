"""Variable-length batches (asr_enc_forward_varlen) against the oracle (GPU).

Each clip has its own length; its frames are cut into 100-frame chunks with
a short last chunk, its log-mel maximum and its attention windows are its
own ("MOSS-Transcribe-preview-2B-GGUF", Architecture table: "Audio encoder"
windowed attention, "Conv front-end" per-chunk stem).  Every clip is compared
with oracle.encode_clip run on that clip alone, at the encoder tolerance
(per-row cosine >= 0.999, max row relative L2 <= 2e-2); token counts are
bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_encoder_parity

pytestmark = pytest.mark.gpu

sra = pytest.importorskip("speech_recognition_audio_b200")


def _encoder(g, seed, affine=False):
    W = synth.make_weights(g, seed, affine=affine)
    return sra.Encoder(g, {k: v.cuda() for k, v in W.items()}), W


def _packed(lengths, seed0):
    clips = [synth.pcm_clip(n, seed0 + i) for i, n in enumerate(lengths)]
    return clips, torch.from_numpy(np.concatenate(clips)).cuda()


def test_tiny_varlen_affine():
    # Non-zero biases: a short chunk's padded conv rows would hold GELU(bias)
    # if they were not zeroed; lengths with short chunks of 37, 1 and 50
    # frames, a clip of whole chunks, and one that is not a whole number of hops.
    g = synth.GEOMETRIES["tiny"]
    enc, W = _encoder(g, 91, affine=True)
    lengths = [21920, 16160, 32000, 8000, 16077]
    clips, pcm = _packed(lengths, 800)
    out, toks = enc.forward_varlen(pcm, lengths)
    enc.sync_status()
    assert toks == [oracle.token_count(g, n) for n in lengths] == [18, 14, 26, 7, 13]
    got = out.cpu().numpy()
    row = 0
    for n, pcm_b, t in zip(lengths, clips, toks):
        ref = oracle.encode_clip(pcm_b, W, g)
        assert ref.shape[0] == t
        assert_encoder_parity(got[row:row + t], ref, f"tiny varlen clip of {n} samples")
        row += t
    assert row == got.shape[0]
    host, toks_h = enc.forward_host_varlen(pcm.cpu().pin_memory(), lengths)
    assert toks_h == toks
    np.testing.assert_array_equal(host.numpy(), got)
    enc.close()


def test_moss_varlen_7_30_12s():
    g = synth.GEOMETRIES["moss"]
    enc, W = _encoder(g, 1239)
    lengths = [116800, 480000, 192160]              # 7.3 s, 30 s, 12.01 s
    clips, pcm = _packed(lengths, 900)
    out, toks = enc.forward_varlen(pcm, lengths)
    enc.sync_status()
    assert toks == [95, 390, 157]
    got = out.cpu().numpy()
    offs = np.cumsum([0] + toks)
    # 7.3 s and 12.01 s whole; 30 s through its first and last windows
    for b, windows in ((0, None), (1, [0, 3]), (2, None)):
        cu = oracle.window_partition(g, lengths[b], 1)
        sel = [None] if windows is None else windows
        for j in sel:
            ref = oracle.encode_clip(clips[b], W, g, windows=None if j is None else [j])
            rows = slice(offs[b], offs[b + 1]) if j is None else slice(offs[b] + cu[j], offs[b] + cu[j + 1])
            assert_encoder_parity(got[rows], ref, f"moss varlen clip {b} window {j}")
    enc.close()


def test_uniform_api_with_short_chunks_and_whole_chunk_equivalence():
    g = synth.GEOMETRIES["tiny"]
    enc, W = _encoder(g, 92)
    # B clips of one length that is not whole chunks: the uniform call runs
    # the variable-length path
    pcm = np.stack([synth.pcm_clip(23456, 40 + b) for b in range(3)])
    out = enc.forward(torch.from_numpy(pcm).cuda())
    enc.sync_status()
    T = oracle.token_count(g, 23456)
    assert out.shape == (3, T, g.adapter_out)
    assert_encoder_parity(out.cpu().numpy(), oracle.forward(pcm, W, g), "uniform call, short chunks")
    # whole chunks: the variable-length path gives the uniform path's bits
    pcm2 = np.stack([synth.pcm_clip(32000, 50 + b) for b in range(2)])
    a = enc.forward(torch.from_numpy(pcm2).cuda()).cpu().numpy()
    b, toks = enc.forward_varlen(torch.from_numpy(pcm2.reshape(-1)).cuda(), [32000, 32000])
    enc.sync_status()
    assert toks == [26, 26]
    np.testing.assert_array_equal(a.reshape(-1, a.shape[-1]), b.cpu().numpy())
    enc.close()


def test_varlen_rejections():
    enc, _ = _encoder(synth.GEOMETRIES["tiny"], 93)
    pcm = torch.zeros(16000 + 200, device="cuda")
    with pytest.raises(sra.AsrError) as ei:
        enc.forward_varlen(pcm, [16000, 200])       # a clip too short for the reflect padding
    assert ei.value.code == 2
    enc.close()
    w = synth.GEOMETRIES["whisper_small"]
    encw, _ = _encoder(w, 94)
    with pytest.raises(sra.AsrError) as ei:         # the conv1d stem takes whole-hop batches only
        encw.forward_varlen(torch.zeros(32000, device="cuda"), [16000, 16000])
    assert ei.value.code == 2
    encw.close()
