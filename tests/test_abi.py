"""C-ABI checks that need no GPU: the library loads, exports every function
that include/*.h declares, and its host-only queries (token counts, window
partitions, weight order) agree bit-exactly with the oracle and the seeded
generators."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

import oracle
import synth
import speech_recognition_audio_b200 as sra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(asr_(?:enc|op)_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_function():
    declared = _declared()
    assert len(declared) >= 20
    lib = ctypes.CDLL(sra.LIB_PATH)
    missing = [n for n in sorted(declared) if not hasattr(lib, n)]
    assert not missing, missing


@pytest.mark.parametrize("gname,secs", [("tiny", 1), ("moss", 1), ("moss", 30), ("moss", 600),
                                        ("whisper_small", 30), ("whisper_small", 1)])
def test_tokens_match_oracle(gname, secs):
    g = synth.GEOMETRIES[gname]
    n = 16000 * secs
    assert sra.tokens(g, n) == oracle.token_count(g, n)


@pytest.mark.parametrize("n", [16000 + 160, 16000 + 1, 116800, 192160, 16077, 201, 480000 + 3200])
def test_tokens_partial_chunks_match_oracle(n):
    for gname in ("moss", "tiny", "whisper_small"):
        g = synth.GEOMETRIES[gname]
        assert sra.tokens(g, n) == oracle.token_count(g, n)


def test_tokens_reject_too_short():
    for gname in ("moss", "whisper_small"):
        assert sra.tokens(synth.GEOMETRIES[gname], 200) == -1
        assert sra.tokens(synth.GEOMETRIES[gname], 0) == -1


@pytest.mark.parametrize("n", [116800, 192160, 16077])
def test_windows_partial_chunks_match_oracle(n):
    g = synth.GEOMETRIES["moss"]
    assert sra.windows(g, n, 3) == oracle.window_partition(g, n, 3).tolist()


@pytest.mark.parametrize("wname", list(synth.WORKLOADS))
def test_windows_match_oracle(wname):
    w = synth.WORKLOADS[wname]
    g = synth.GEOMETRIES[w.geometry]
    cu = sra.windows(g, w.n_samples, w.batch)
    ref = oracle.window_partition(g, w.n_samples, w.batch)
    assert cu == ref.tolist()


def test_windows_capacity_error():
    g = synth.GEOMETRIES["moss"]
    cu = (ctypes.c_int32 * 2)()
    n = ctypes.c_int(2)
    geo = sra.Geometry.of(g)
    rc = sra.lib.asr_enc_windows(ctypes.byref(geo), 480000, 1, cu, ctypes.byref(n))
    assert rc == 1
    assert b"capacity" in sra.lib.asr_enc_last_error(None)


@pytest.mark.parametrize("gname", list(synth.GEOMETRIES))
def test_weight_order_matches_generator(gname):
    g = synth.GEOMETRIES[gname]
    names = sra.weight_names(g)
    specs = [(n, tuple(s)) for n, s, _ in synth.weight_specs(g)]
    assert names == specs


def test_invalid_geometry_rejected():
    bad = synth.GEOMETRIES["moss"].as_dict()
    bad["head_dim"] = 80
    assert sra.lib.asr_enc_weight_count(ctypes.byref(sra.Geometry.of(bad))) == -1
    assert sra.tokens(bad, 16000) == -1
    bad2 = synth.GEOMETRIES["moss"].as_dict()
    bad2["n_fft"] = 512
    with pytest.raises(sra.AsrError):
        sra.windows(bad2, 16000, 1)


def test_null_handle_calls_fail_cleanly():
    assert sra.lib.asr_enc_sync_status(None) == 1
    assert sra.lib.asr_enc_set_taps(None, 1) == 1
    assert sra.lib.asr_enc_workspace_size(None, 16000, 1) == 0
    sra.lib.asr_enc_destroy(None)
    rc = sra.lib.asr_enc_forward(None, None, 16000, 1, None, None, None, 0, None)
    assert rc == 1


def test_documented_limits_are_enforced():
    # Argument validation only: every call below is rejected on the host
    # before anything reaches a device.
    bad = synth.GEOMETRIES["moss"].as_dict()
    bad.update(d_model=192, n_heads=3)                 # d_model must be a multiple of 128
    assert sra.lib.asr_enc_weight_count(ctypes.byref(sra.Geometry.of(bad))) == -1
    big = synth.GEOMETRIES["moss"].as_dict()
    big.update(d_model=2176, n_heads=34)               # d_model must be <= 2048
    assert sra.lib.asr_enc_weight_count(ctypes.byref(sra.Geometry.of(big))) == -1
    # LayerNorm: D a multiple of 128 and at most 2048; NULL operands rejected first.
    assert sra.lib.asr_op_layer_norm(None, None, None, 4, 1280, 1e-5, None, 0, None) == 1
    fake = ctypes.c_void_p(256)                        # never dereferenced: the size check fails first
    for D in (4096, 1000, 2176):
        assert sra.lib.asr_op_layer_norm(fake, fake, fake, 4, D, 1e-5, fake, 0, None) == 1
        assert b"layer_norm" in sra.lib.asr_enc_last_error(None)
    # log-mel: the workspace holds the maxima and the tables
    assert sra.lib.asr_op_log_mel_ws_size(16) >= 16 * 4 + 14 * 1024
    assert sra.lib.asr_op_log_mel_ws_size(0) == 0
