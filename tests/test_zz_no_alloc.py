"""The log-mel entry point that allocates nothing (asr_op_log_mel_noalloc).

Callers that cannot call cudaMalloc (a plugin in a host that owns device
memory, a real-time audio thread) use this variant; its scratch is a fixed
array inside the library.  It runs the same kernels on the same tables as the
entry point with a caller-supplied workspace, so its output must be
bit-identical to that entry point's, call after call, and within the log-mel
tolerance of the oracle.  This file is collected last so that, if it fails,
a run that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

sra = pytest.importorskip("speech_recognition_audio_b200")


def _noalloc(pcm, n_mels, stream=None):
    B, n = pcm.shape
    mel = torch.empty((B, n_mels, n // 160), dtype=torch.float32, device=pcm.device)
    st = stream if stream is not None else torch.cuda.current_stream()
    rc = sra.lib.asr_op_log_mel_noalloc(ctypes.c_void_p(pcm.data_ptr()), n, B, n_mels, ctypes.c_void_p(mel.data_ptr()),
                                        ctypes.c_void_p(st.cuda_stream))
    assert rc == 0, sra.lib.asr_enc_last_error(None)
    return mel


@pytest.mark.parametrize("n_mels,batch,secs", [(128, 3, 2), (80, 2, 1), (128, 1, 3)])
def test_noalloc_log_mel_matches_workspace_entry_point(n_mels, batch, secs):
    pcm_np = np.stack([synth.pcm_clip(16000 * secs, 300 + b) for b in range(batch)])
    pcm = torch.from_numpy(pcm_np).cuda()
    ref = sra.log_mel(pcm, n_mels)          # existing entry point, workspace from the caller
    first = _noalloc(pcm, n_mels)
    second = _noalloc(pcm, n_mels)          # the shared scratch keeps the last call's contents
    torch.cuda.synchronize()
    for got in (first, second):
        assert got.shape == ref.shape
        assert torch.equal(got, ref)
    for b in range(batch):
        assert np.abs(first[b].cpu().numpy() - oracle.log_mel(pcm_np[b], n_mels)).max() <= 1e-3


def test_noalloc_alternating_mel_counts_on_one_stream():
    # Calls with different n_mels, queued back to back on one stream with no
    # host synchronisation between them: each call rebuilds the shared tables
    # in stream order, so none may see another call's tables.
    pcm = torch.from_numpy(np.stack([synth.pcm_clip(32000, 700 + b) for b in range(2)])).cuda()
    ref = {m: sra.log_mel(pcm, m) for m in (128, 80, 40)}
    torch.cuda.synchronize()
    order = [128, 80, 128, 40, 80, 128]
    outs = [_noalloc(pcm, m) for m in order]
    torch.cuda.synchronize()
    for m, got in zip(order, outs):
        assert torch.equal(got, ref[m]), m


def test_noalloc_rejects_batch_over_limit():
    pcm = torch.zeros((1, 16000), device="cuda")
    mel = torch.empty((1, 128, 100), device="cuda")
    rc = sra.lib.asr_op_log_mel_noalloc(ctypes.c_void_p(pcm.data_ptr()), 16000, 4097, 128,
                                        ctypes.c_void_p(mel.data_ptr()), None)
    assert rc == 2
    assert b"4096" in sra.lib.asr_enc_last_error(None)
