"""Audio-embedding splice (asr_splice_embeddings) against the oracle (GPU).

MOSS-Transcribe-preview-2B-GGUF card, Architecture table: "Audio injection"
(placeholder positions take the adapter output frames) and "Prompt" (ChatML
user turn with the audio between the audio start and end markers).  Rows are
compared bit for bit: table rows are copied, frames are converted to the
output type with round-to-nearest-even on both sides.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_encoder_parity

pytestmark = pytest.mark.gpu

sra = pytest.importorskip("speech_recognition_audio_b200")

PH, IM_START, IM_END, AUDIO_START, AUDIO_END, USER, ASSISTANT, NL = 7, 1, 2, 3, 4, 5, 6, 8


def _prompt(n_audio):
    return [IM_START, USER, NL, AUDIO_START] + [PH] * n_audio + [AUDIO_END, IM_END, NL, IM_START, ASSISTANT, NL]


def _expect(ids, table, frames, dtype):
    ref = oracle.splice_embeddings(ids, PH, table.float().numpy(), frames.numpy())
    return torch.from_numpy(ref).to(dtype)


@pytest.mark.parametrize("tdt,odt", [(torch.bfloat16, torch.bfloat16), (torch.float16, torch.float16),
                                     (torch.float32, torch.float32), (torch.float16, torch.float32),
                                     (torch.bfloat16, torch.float16)])
@pytest.mark.parametrize("D", [2048, 40])
def test_splice_matches_oracle(tdt, odt, D):
    g = torch.Generator().manual_seed(D + 3)
    vocab = 1000
    table = (torch.randn(vocab, D, generator=g) * 0.05).to(tdt)
    lens = [13, 390, 1]
    ids = sum((_prompt(t) for t in lens), []) + [11, 999, 0]
    ids += list(torch.randint(9, vocab, (50,), generator=g).tolist())
    frames = torch.randn(sum(lens), D, generator=g) * 3.0
    out = sra.splice_embeddings(torch.tensor(ids, dtype=torch.int32).cuda(), PH, table.cuda(), frames.cuda(),
                                out_dtype=odt)
    ref = _expect(ids, table, frames, odt)
    assert out.dtype == odt and out.shape == (len(ids), D)
    assert torch.equal(out.cpu(), ref)


def test_splice_reports_errors():
    table = torch.zeros(16, 64, dtype=torch.bfloat16).cuda()
    frames = torch.ones(3, 64).cuda()
    with pytest.raises(sra.AsrError) as ei:   # two placeholders, three frames
        sra.splice_embeddings(torch.tensor(_prompt(2), dtype=torch.int32).cuda(), PH, table, frames)
    assert ei.value.code == 1 and "count" in str(ei.value)
    with pytest.raises(sra.AsrError) as ei:   # id 16 is outside the table
        sra.splice_embeddings(torch.tensor(_prompt(3) + [16], dtype=torch.int32).cuda(), PH, table, frames)
    assert ei.value.code == 1 and "vocab" in str(ei.value)


def test_forward_then_splice_matches_oracle():
    # The path end to end: two clips through the tiny encoder, their adapter
    # frames spliced into a packed pair of prompts.
    w = synth.WORKLOADS["tiny_1x1s"]
    gm = synth.GEOMETRIES[w.geometry]
    W = synth.make_weights(gm, w.weight_seed)
    enc = sra.Encoder(gm, {k: v.cuda() for k, v in W.items()})
    pcm = np.stack([synth.pcm_clip(32000, 61), synth.pcm_clip(32000, 62)])
    frames = enc.forward(torch.from_numpy(pcm).cuda())            # [2, 26, 512]
    enc.sync_status()
    T = frames.shape[1]
    ids = _prompt(T) + _prompt(T)
    table = (torch.randn(100, gm.adapter_out, generator=torch.Generator().manual_seed(5)) * 0.05).to(torch.float16)
    out = sra.splice_embeddings(torch.tensor(ids, dtype=torch.int32).cuda(), PH, table.cuda(),
                                frames.reshape(-1, gm.adapter_out), out_dtype=torch.float32)
    ref_frames = oracle.forward(pcm, W, gm).reshape(-1, gm.adapter_out)
    ref = oracle.splice_embeddings(ids, PH, table.float().numpy(), ref_frames)
    audio = np.array([i == PH for i in ids])
    got = out.cpu().numpy()
    np.testing.assert_array_equal(got[~audio], ref[~audio])
    assert_encoder_parity(got[audio], ref[audio], "splice of the tiny encoder's frames")
    enc.close()
