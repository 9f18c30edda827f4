"""Streaming encoder (asr_stream_*) against the oracle's streaming definition (GPU).

Live input is encoded one attention window at a time ("MOSS-Transcribe-
preview-2B-GGUF", Architecture, "Audio encoder": windowed, block-diagonal
attention); each window is normalised by its own log-mel maximum and its
frames use the stream's real samples across window boundaries
(oracle.encode_stream).  Pushes of irregular sizes must give the same rows,
at the encoder tolerance, as the oracle on the whole stream.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_encoder_parity

pytestmark = pytest.mark.gpu

sra = pytest.importorskip("speech_recognition_audio_b200")


def _stream_rows(enc, pcm, pieces):
    st = sra.Stream(enc)
    x = torch.from_numpy(pcm).cuda()
    rows, pos = [], 0
    for n in pieces:
        rows.append(st.push(x[pos:pos + n].contiguous()))
        pos += n
    assert pos == pcm.shape[0]
    rows.append(st.finish())
    enc.sync_status()
    st.close()
    return torch.cat(rows).cpu().numpy(), [r.shape[0] for r in rows]


def test_tiny_stream_irregular_pushes():
    g = synth.GEOMETRIES["tiny"]                          # windows of 104 tokens = 800 frames (8 s)
    W = synth.make_weights(g, 95, affine=True)
    enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
    pcm = synth.pcm_clip(325000, 77, speech_like=True)    # 2031 frames: windows 800, 800, 431
    pieces = [11200, 80000, 37000, 1, 90000, 106799]
    got, counts = _stream_rows(enc, pcm, pieces)
    ref = oracle.encode_stream(pcm, W, g)
    assert got.shape == ref.shape
    assert sum(counts[:-1]) == 2 * 104 and counts[-1] == ref.shape[0] - 208
    assert_encoder_parity(got, ref, "tiny stream")
    # one push of everything: the same windows
    got2, _ = _stream_rows(enc, pcm, [pcm.shape[0]])
    assert_encoder_parity(got2, ref, "tiny stream, one push")
    enc.close()


def test_short_stream_equals_offline_clip():
    g = synth.GEOMETRIES["tiny"]
    W = synth.make_weights(g, 96)
    enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
    pcm = synth.pcm_clip(77777, 78)                       # under one window: the clip's own maximum
    got, _ = _stream_rows(enc, pcm, [30000, 47777])
    assert_encoder_parity(got, oracle.encode_clip(pcm, W, g), "short stream vs offline clip")
    enc.close()


def test_moss_stream_17s():
    g = synth.GEOMETRIES["moss"]
    W = synth.make_weights(g, 1240)
    enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
    pcm = synth.pcm_clip(272000, 79)                      # 1700 frames: windows 800, 800, 100
    got, counts = _stream_rows(enc, pcm, [100000, 100000, 72000])
    ref = oracle.encode_stream(pcm, W, g)
    assert got.shape == ref.shape == (104 + 104 + 13, 2048)
    assert_encoder_parity(got, ref, "moss stream 17 s")
    enc.close()
