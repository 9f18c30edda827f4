"""End-to-end parity of the encoder forward pass (GPU) against the oracle.

Every workload runs through the C ABI (asr_enc_create / asr_enc_forward) on
its seeded synthetic audio and random-init weights:
  tiny 1 x 1 s (fp32 weights)    whole output + every stage tap
  moss 1 x 30 s                  whole output
  moss 16 x 30 s (the benchmark launch configuration)
                                 sampled windows of several clips, exact by
                                 window independence (oracle.encode_clip)
  moss 1 x 600 s speech-like     sampled windows, including silent stretches
  whisper-small 32 x 30 s        two whole clips (full attention)
Tolerances: per-row cosine >= 0.999 and max row relative L2 <= 2e-2 for the
encoder/adapter output; log-mel max abs <= 1e-3; token counts bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_encoder_parity, MEL_ABS_MAX

pytestmark = pytest.mark.gpu

sra = pytest.importorskip("speech_recognition_audio_b200")

_CACHE = {}


def _encoder(wname, affine=False, geometry=None, seed=None):
    key = (wname, affine, geometry, seed)
    if key not in _CACHE:
        w = synth.WORKLOADS[wname]
        g = geometry or synth.GEOMETRIES[w.geometry]
        W = synth.make_weights(g, seed if seed is not None else w.weight_seed, affine=affine)
        enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
        _CACHE.clear()  # keep one large encoder resident at a time
        torch.cuda.empty_cache()
        _CACHE[key] = (enc, W, g)
    return _CACHE[key]


def _run(enc, pcm):
    out = enc.forward(torch.from_numpy(pcm).cuda())
    enc.sync_status()
    return out.cpu().numpy()


def test_tiny_full_with_taps():
    enc, W, g = _encoder("tiny_1x1s")
    w = synth.WORKLOADS["tiny_1x1s"]
    pcm = synth.pcm_batch(w)
    enc.set_taps(0b11111)
    out = _run(enc, pcm)
    taps = {}
    ref = oracle.forward(pcm, W, g, taps=taps)
    t = taps["clips"][0]
    T = out.shape[1]
    assert T == 13 == oracle.token_count(g, w.n_samples)
    mel = enc.tap(sra.TAP_MEL, (1, g.n_mels, w.n_samples // 160)).cpu().numpy()[0]
    print(f"[parity] tiny log-mel max abs {np.abs(mel - t['mel']).max():.3e}")
    assert np.abs(mel - t["mel"]).max() <= MEL_ABS_MAX
    assert_encoder_parity(enc.tap(sra.TAP_STEM, (T, g.d_model)).cpu().numpy(), t["stem"], "stem")
    assert_encoder_parity(enc.tap(sra.TAP_LAYER0, (T, g.d_model)).cpu().numpy(), t["layer0"], "layer0")
    assert_encoder_parity(enc.tap(sra.TAP_ENCODER, (T, g.d_model)).cpu().numpy(), t["encoder"], "encoder")
    assert_encoder_parity(enc.tap(sra.TAP_HEAD, (T, g.proj2_out)).cpu().numpy(), t["head"], "head")
    assert_encoder_parity(out, ref, "adapter output")
    enc.set_taps(0)


def test_tiny_fp32_weights_run_tf32_end_to_end():
    # The tiny geometry's weights are fp32: every GEMM is a kind::tf32 GEMM on
    # fp32 activations and the attention runs in fp32, so the result sits
    # well inside the bf16 tolerance tier (tf32 keeps 10 mantissa bits, bf16
    # 7; the GELU's tanh form adds up to 4.8e-4 per element either way).
    w = synth.WORKLOADS["tiny_1x1s"]
    g = synth.GEOMETRIES["tiny"]
    assert g.dtype == synth.DTYPE_F32
    enc, W, _ = _encoder("tiny_1x1s", affine=True, seed=78)
    pcm = np.stack([synth.pcm_clip(32000, 510), synth.pcm_clip(32000, 511)])
    out = _run(enc, pcm)
    ref = oracle.forward(pcm, W, g)
    cmin, rmax = assert_encoder_parity(out, ref, "tiny fp32 weights (tf32)")
    assert cmin >= 0.99995 and rmax <= 1e-2


def test_whisper_style_fp32_geometry():
    # Conv1D stem, full attention and final LN with fp32 weights (tf32 path).
    base = synth.GEOMETRIES["whisper_small"].as_dict()
    base.update(d_model=256, n_heads=4, d_ffn=1024, n_layers=2, dtype=synth.DTYPE_F32)
    g = synth.Geometry(**base)
    W = synth.make_weights(g, 79, affine=True)
    enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
    pcm = np.stack([synth.pcm_clip(48000, 520), synth.pcm_clip(48000, 521)])
    out = _run(enc, pcm)
    assert out.shape == (2, 150, 256)
    assert_encoder_parity(out, oracle.forward(pcm, W, g), "whisper-style fp32 weights (tf32)")
    enc.close()


def test_tiny_f16_weights():
    # f16 weights and activations between the GEMMs (kind::f16 with f16 operands).
    base = synth.GEOMETRIES["tiny"].as_dict()
    base.update(dtype=synth.DTYPE_F16)
    g = synth.Geometry(**base)
    W = synth.make_weights(g, 80, affine=True)
    assert W["conv1.w"].dtype == torch.float16
    enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
    pcm = np.stack([synth.pcm_clip(48000, 530), synth.pcm_clip(48000, 531)])
    out = _run(enc, pcm)
    assert_encoder_parity(out, oracle.forward(pcm, W, g), "tiny f16 weights")
    enc.close()


def test_moss_1x30s_f16_weights():
    # The MOSS tower with the F16 weights the pages' GGUF builds keep for the
    # encoder and adapter; 10 s keep the float64 oracle short.
    base = synth.GEOMETRIES["moss"].as_dict()
    base.update(dtype=synth.DTYPE_F16)
    g = synth.Geometry(**base)
    W = synth.make_weights(g, 1241)
    enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
    pcm = synth.pcm_clip(160000, 540)[None]
    out = _run(enc, pcm)
    assert out.shape == (1, 130, 2048)
    assert_encoder_parity(out, oracle.forward(pcm, W, g), "moss 1x10s f16 weights")
    enc.close()


def test_affine_biases_small_batch():
    # Non-zero biases and LayerNorm affine parameters exercise every epilogue's
    # bias path and the LN gain/shift; 2 clips x 3 s, windows of 104 > 39 tokens.
    w = synth.WORKLOADS["tiny_1x1s"]
    g = synth.GEOMETRIES["tiny"]
    enc, W, _ = _encoder("tiny_1x1s", affine=True, seed=77)
    pcm = np.stack([synth.pcm_clip(48000, 500), synth.pcm_clip(48000, 501)])
    out = _run(enc, pcm)
    ref = oracle.forward(pcm, W, g)
    assert out.shape == (2, 39, g.adapter_out)
    assert_encoder_parity(out, ref, "affine tiny")


def test_moss_1x30s_full():
    enc, W, g = _encoder("moss_1x30s")
    pcm = synth.pcm_batch(synth.WORKLOADS["moss_1x30s"])
    out = _run(enc, pcm)
    assert out.shape == (1, 390, 2048)
    ref = oracle.forward(pcm, W, g)
    assert_encoder_parity(out, ref, "moss 1x30s")


def _sampled(wname, picks, affine=False, seed=None):
    w = synth.WORKLOADS[wname]
    enc, W, g = _encoder(wname, affine=affine, seed=seed)
    pcm = synth.pcm_batch(w)
    enc.set_taps(1 << sra.TAP_MEL)
    out = _run(enc, pcm)
    mel = enc.tap(sra.TAP_MEL, (w.batch, g.n_mels, w.n_samples // 160)).cpu().numpy()
    enc.set_taps(0)
    T = oracle.token_count(g, w.n_samples)
    assert out.shape == (w.batch, T, g.d_out)
    cu = oracle.window_partition(g, w.n_samples, 1)
    for b, j in picks:
        ref_mel = oracle.log_mel(pcm[b], g.n_mels)
        print(f"[parity] {wname} clip {b} log-mel max abs {np.abs(mel[b] - ref_mel).max():.3e}")
        assert np.abs(mel[b] - ref_mel).max() <= MEL_ABS_MAX
        ref = oracle.encode_clip(pcm[b], W, g, windows=[j] if j is not None else None)
        rows = slice(int(cu[j]), int(cu[j + 1])) if j is not None else slice(0, T)
        assert_encoder_parity(out[b, rows], ref, f"{wname} clip {b} window {j}")
    return out


def test_moss_16x30s_sampled():
    _sampled("moss_16x30s", [(0, 0), (7, 3), (15, 2)])


def test_moss_1x600s_sampled():
    _sampled("moss_1x600s", [(0, 0), (0, 37), (0, 74)])


def test_whisper_small_32x30s_sampled():
    _sampled("whisper_small_32x30s", [(0, None), (31, None)])


@pytest.mark.parametrize("wname,picks", [("moss_16x30s", [(2, 1), (13, 3)]), ("whisper_small_32x30s", [(5, None)])])
def test_affine_biases_full_size_sampled(wname, picks):
    """Non-zero biases and LayerNorm gains and shifts at full size, in the
    benchmark's launch configuration: the CTA-pair tiles, the conv-box stem
    GEMMs, the split QKV projection, stream-K fc2 (d = 1280) and the flash
    attention path (whisper-small) all carry bias signal end to end."""
    _sampled(wname, picks, affine=True, seed=91)


@pytest.mark.parametrize("wname", ["moss_1x30s", "tiny_f16"])
def test_ln_fusion_matches_separate_layernorms(wname):
    """16-bit encoders can compute each block's first LayerNorm (and the
    head's) in the previous fc2's epilogue (asr_enc_set_ln_fusion; off by
    default, when the separate LayerNorm kernels run).  Both match the
    oracle, and they agree closely with each other (they differ only by the
    order in which the row statistics are summed)."""
    if wname == "tiny_f16":
        base = synth.GEOMETRIES["tiny"].as_dict()
        base.update(dtype=synth.DTYPE_F16)
        g = synth.Geometry(**base)
        W = synth.make_weights(g, 81, affine=True)
        enc = sra.Encoder(g, {k: v.cuda() for k, v in W.items()})
        pcm = np.stack([synth.pcm_clip(48000, 532), synth.pcm_clip(48000, 533)])
    else:
        enc, W, g = _encoder(wname)
        pcm = synth.pcm_batch(synth.WORKLOADS[wname])
    assert not enc.ln_fusion()
    enc.set_ln_fusion(True)
    assert enc.ln_fusion()
    fused = _run(enc, pcm)
    enc.set_ln_fusion(False)
    assert not enc.ln_fusion()
    plain = _run(enc, pcm)
    enc.set_ln_fusion(True)
    again = _run(enc, pcm)
    enc.set_ln_fusion(False)
    np.testing.assert_array_equal(fused, again)
    ref = oracle.forward(pcm, W, g)
    assert_encoder_parity(fused, ref, f"{wname} LayerNorm epilogue")
    assert_encoder_parity(plain, ref, f"{wname} separate LayerNorms")
    rel = np.linalg.norm(fused - plain) / np.linalg.norm(plain)
    print(f"[parity] {wname} fused vs separate LayerNorm rel L2 {rel:.2e}")
    assert rel < 1e-2


def test_fp32_weights_keep_separate_layernorms():
    enc, W, g = _encoder("tiny_1x1s")
    enc.set_ln_fusion(True)
    assert not enc.ln_fusion()  # kind::tf32 has no LayerNorm epilogue
    enc.set_ln_fusion(False)


def test_host_forward_matches_device_forward():
    enc, W, g = _encoder("tiny_1x1s")
    pcm = np.stack([synth.pcm_clip(32000, 900 + b) for b in range(3)])
    dev = _run(enc, pcm)
    host = enc.forward_host(torch.from_numpy(pcm).pin_memory()).numpy()
    np.testing.assert_array_equal(dev, host)


def test_forward_rejects_bad_sizes():
    import ctypes
    enc, W, g = _encoder("tiny_1x1s")
    pcm = torch.zeros((1, 200), device="cuda")    # reflect padding needs more than n_fft/2 samples
    with pytest.raises(sra.AsrError) as ei:
        enc.forward(pcm)
    assert ei.value.code == 2
    out = torch.empty((1, 1, g.adapter_out), device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    rc = sra.lib.asr_enc_forward(enc.handle, ctypes.c_void_p(pcm.data_ptr()), 200, 1, ctypes.c_void_p(out.data_ptr()),
                                 None, ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert rc == 1
    pcm = torch.zeros((1, 16000), device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(sra.AsrError) as ei:
        enc.forward(pcm, workspace=small)
    assert ei.value.code == 5


def test_repeat_forward_deterministic():
    enc, W, g = _encoder("tiny_1x1s")
    pcm = synth.pcm_batch(synth.WORKLOADS["tiny_1x1s"], batch=2)
    a = _run(enc, pcm)
    b = _run(enc, pcm)
    np.testing.assert_array_equal(a, b)


def test_graph_replay_matches_direct_launches():
    # A uniform forward is recorded as a CUDA graph for its pointers and
    # shape, then replayed: bit-identical to the direct launches, reading the
    # current data behind the same pointers, and re-recorded for new ones.
    enc, W, g = _encoder("tiny_1x1s")
    wl = synth.WORKLOADS["tiny_1x1s"]
    pcm_np = synth.pcm_batch(wl, batch=2)
    pcm = torch.from_numpy(pcm_np).cuda()
    B, n = pcm.shape
    out = torch.empty((B, enc.tokens(n), enc.d_out), device="cuda")
    ws = enc.workspace(n, B)

    def direct(x):
        enc.set_graphs(False)
        o = torch.empty_like(out)
        enc.forward(x, out=o, workspace=ws)
        enc.sync_status()
        enc.set_graphs(True)
        return o, sra.lib.asr_enc_last_launches(enc.handle)

    ref, launches = direct(pcm)
    assert launches > 10
    for _ in range(3):  # the first call records, the others replay
        out.zero_()
        enc.forward(pcm, out=out, workspace=ws)
        enc.sync_status()
        assert torch.equal(out, ref)
        assert sra.lib.asr_enc_last_launches(enc.handle) == launches
    assert_encoder_parity(out.cpu().numpy(), oracle.forward(pcm_np, W, g), "graph replay")
    # new samples behind the same pointer: the replay reads them
    pcm2_np = np.stack([synth.pcm_clip(n, 700 + b) for b in range(B)]).astype(np.float32)
    ref2, _ = direct(torch.from_numpy(pcm2_np).cuda())
    pcm.copy_(torch.from_numpy(pcm2_np))
    enc.forward(pcm, out=out, workspace=ws)
    enc.sync_status()
    assert torch.equal(out, ref2)
    # another output buffer: a new recording, same values
    out3 = torch.empty_like(out)
    enc.forward(pcm, out=out3, workspace=ws)
    enc.sync_status()
    assert torch.equal(out3, ref2)


def test_moss_16x30s_repeat_bit_identical():
    # 16 x 30 s runs fc2 with stream-K (split tiles, owner waits on flags that
    # it clears again) inside the replayed graph: repeated forwards on the
    # same buffers give the same bits, also with graphs switched off.
    w = synth.WORKLOADS["moss_16x30s"]
    enc, W, g = _encoder("moss_16x30s")
    pcm = torch.from_numpy(synth.pcm_batch(w)).cuda()
    B, n = pcm.shape
    out = torch.empty((B, enc.tokens(n), enc.d_out), device="cuda")
    ws = enc.workspace(n, B)
    runs = []
    for graphs in (True, True, True, False):
        enc.set_graphs(graphs)
        enc.forward(pcm, out=out, workspace=ws)
        enc.sync_status()
        runs.append(out.clone())
    enc.set_graphs(True)
    for r in runs[1:]:
        assert torch.equal(r, runs[0])
