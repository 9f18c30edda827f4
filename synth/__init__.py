"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds data only: the five encoder geometries, a seeded PCM
generator and a seeded weight generator.  It computes nothing of the encoder
itself (no STFT, no convolution, no layer), so that the CPU oracle and the
CUDA path can both draw the same inputs without sharing any of the method's
arithmetic.

Geometries follow the pages:
  * MOSS-Transcribe-preview-2B-GGUF, "Architecture" table: the audio tower
    (32 pre-LN layers, d=1280, 20x64 heads, FFN 5120, windowed attention),
    the conv front-end 1->480->480->480 with conv_out 480*16=7680->1280,
    the head ln_post->proj1 1280->1280->GELU->proj2 1280->2048 and the SwiGLU
    adapter 2048->8192->2048; "Audio" row: 16 kHz, 128 mel bins, n_fft=400,
    hop=160.
  * CrisperWhisper2.0_small-ONNX-timestamped, "What this exports instead":
    whisper-small geometry (12 encoder layers, d_model 768), and "Results":
    1500 encoder frames per 30 s window.
Sizes the pages leave open (the tiny geometry, the 100-frame conv chunk, the
104-token attention window, the FFN width of whisper-small) come from the
benchmark configurations this repository is measured on.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict

import numpy as np
import torch

__all__ = ["Geometry", "GEOMETRIES", "Workload", "WORKLOADS", "pcm_clip", "pcm_batch",
           "weight_specs", "make_weights"]

SAMPLE_RATE = 16000

# Stem kinds.
STEM_CONV2D_CHUNKED = 0   # 3 x Conv2D k3 s2 p1 per 100-frame chunk (MOSS / Qwen3-Omni audio tower)
STEM_CONV1D = 1           # Conv1D k3 s1 p1 then Conv1D k3 s2 p1 (whisper)

# Position modes.
POS_PER_CHUNK = 0
POS_GLOBAL = 1

DTYPE_BF16 = 0
DTYPE_F32 = 1
DTYPE_F16 = 2


@dataclass(frozen=True)
class Geometry:
    """Field-for-field mirror of the C-ABI ``asr_geometry`` struct."""
    stem: int
    n_mels: int
    n_fft: int
    hop: int
    chunk_frames: int
    conv_ch: int
    d_model: int
    n_heads: int
    head_dim: int
    d_ffn: int
    n_layers: int
    window_tokens: int      # 0 = full attention over the clip
    pos_mode: int
    proj1_out: int          # 0 = no head projections (whisper: final LN only)
    proj2_out: int
    adapter_hidden: int     # 0 = no adapter
    adapter_out: int
    ln_eps: float
    dtype: int

    def as_dict(self):
        return asdict(self)

    @property
    def d_out(self) -> int:
        if self.adapter_hidden:
            return self.adapter_out
        if self.proj2_out:
            return self.proj2_out
        return self.d_model


_MOSS = dict(stem=STEM_CONV2D_CHUNKED, n_mels=128, n_fft=400, hop=160, chunk_frames=100,
             conv_ch=480, d_model=1280, n_heads=20, head_dim=64, d_ffn=5120, n_layers=32,
             window_tokens=104, pos_mode=POS_PER_CHUNK, proj1_out=1280, proj2_out=2048,
             adapter_hidden=8192, adapter_out=2048, ln_eps=1e-5, dtype=DTYPE_BF16)

GEOMETRIES = {
    # Tiny encoder, fp32: channels 64, d=256, 2 layers, 4x64 heads, FFN 1024,
    # head 256->256->512, adapter 512->1024->512.
    "tiny": Geometry(**{**_MOSS, "conv_ch": 64, "d_model": 256, "n_heads": 4, "d_ffn": 1024,
                        "n_layers": 2, "proj1_out": 256, "proj2_out": 512,
                        "adapter_hidden": 1024, "adapter_out": 512, "dtype": DTYPE_F32}),
    # MOSS-Transcribe audio tower + head + adapter, bf16 weights.
    "moss": Geometry(**_MOSS),
    # Whisper-small geometry: 80 mels, Conv1D stem, 12 layers d=768, 12x64 heads,
    # FFN 3072, full attention over the 1500 frames of a 30 s window, final LN.
    "whisper_small": Geometry(stem=STEM_CONV1D, n_mels=80, n_fft=400, hop=160, chunk_frames=0,
                              conv_ch=768, d_model=768, n_heads=12, head_dim=64, d_ffn=3072,
                              n_layers=12, window_tokens=0, pos_mode=POS_GLOBAL, proj1_out=0,
                              proj2_out=0, adapter_hidden=0, adapter_out=0, ln_eps=1e-5,
                              dtype=DTYPE_BF16),
}


@dataclass(frozen=True)
class Workload:
    name: str
    geometry: str
    batch: int
    seconds: int
    pcm_seed_base: int
    weight_seed: int
    speech_like: bool = False

    @property
    def n_samples(self) -> int:
        return self.seconds * SAMPLE_RATE


# The five workloads: tiny 1 s; 1 x 30 s; 16 x 30 s (throughput); 1 x 600 s
# speech-like long form; 32 x 30 s whisper-small.
WORKLOADS = {
    "tiny_1x1s": Workload("tiny_1x1s", "tiny", 1, 1, 0, 1234),
    "moss_1x30s": Workload("moss_1x30s", "moss", 1, 30, 1000, 1235),
    "moss_16x30s": Workload("moss_16x30s", "moss", 16, 30, 2000, 1236),
    "moss_1x600s": Workload("moss_1x600s", "moss", 1, 600, 3000, 1237, speech_like=True),
    "whisper_small_32x30s": Workload("whisper_small_32x30s", "whisper_small", 32, 30, 4000, 1238),
}


def pcm_clip(n_samples: int, seed: int, speech_like: bool = False) -> np.ndarray:
    """One seeded synthetic clip, float32 [n_samples] at 16 kHz.

    Three sines with frequencies U(100, 4000) Hz, amplitudes U(0.1, 0.3) and
    phases U(0, 2pi), plus N(0, 0.01) noise.  ``speech_like`` multiplies each
    sine by an envelope 0.5(1 + sin(2 pi f_m t + phi_m)), f_m ~ U(2, 6) Hz, and
    afterwards sets 20 % of the 0.5 s segments (chosen by a seeded
    permutation) to exact zeros.  Draw order is fixed: frequencies, amplitudes,
    phases, [modulation frequencies, modulation phases], noise, [permutation].
    """
    rng = np.random.default_rng(seed)
    freqs = rng.uniform(100.0, 4000.0, 3)
    amps = rng.uniform(0.1, 0.3, 3)
    phases = rng.uniform(0.0, 2.0 * math.pi, 3)
    if speech_like:
        fm = rng.uniform(2.0, 6.0, 3)
        phim = rng.uniform(0.0, 2.0 * math.pi, 3)
    t = np.arange(n_samples, dtype=np.float64) / SAMPLE_RATE
    x = np.zeros(n_samples, dtype=np.float64)
    for i in range(3):
        s = amps[i] * np.sin(2.0 * math.pi * freqs[i] * t + phases[i])
        if speech_like:
            s = s * 0.5 * (1.0 + np.sin(2.0 * math.pi * fm[i] * t + phim[i]))
        x += s
    x += rng.normal(0.0, 0.01, n_samples)
    if speech_like:
        seg = SAMPLE_RATE // 2
        n_seg = n_samples // seg
        silent = rng.permutation(n_seg)[: int(round(0.2 * n_seg))]
        for s_idx in silent:
            x[s_idx * seg:(s_idx + 1) * seg] = 0.0
    return x.astype(np.float32)


def pcm_batch(w: Workload, batch: int | None = None, clips=None) -> np.ndarray:
    """float32 [B, n_samples]; clip b uses seed ``pcm_seed_base + b``."""
    idx = list(range(w.batch if batch is None else batch)) if clips is None else list(clips)
    return np.stack([pcm_clip(w.n_samples, w.pcm_seed_base + b, w.speech_like) for b in idx])


def weight_specs(g: Geometry):
    """Ordered (name, shape, kind) of every weight tensor; kind is 'w' (matrix or
    conv kernel), 'b' (bias), 'g' (LayerNorm gain) or 'beta' (LayerNorm shift).
    Matrices are [out, in] row-major as in torch.nn.Linear; conv kernels are
    [out, in, kh(freq), kw(time)] for Conv2D and [out, in, k] for Conv1D."""
    s = []
    d, C = g.d_model, g.conv_ch
    if g.stem == STEM_CONV2D_CHUNKED:
        f_out = g.n_mels
        for _ in range(3):
            f_out = (f_out - 1) // 2 + 1
        s += [("conv1.w", (C, 1, 3, 3), "w"), ("conv1.b", (C,), "b"),
              ("conv2.w", (C, C, 3, 3), "w"), ("conv2.b", (C,), "b"),
              ("conv3.w", (C, C, 3, 3), "w"), ("conv3.b", (C,), "b"),
              ("conv_out.w", (d, C * f_out), "w")]
    else:
        s += [("conv1.w", (d, g.n_mels, 3), "w"), ("conv1.b", (d,), "b"),
              ("conv2.w", (d, d, 3), "w"), ("conv2.b", (d,), "b")]
    for l in range(g.n_layers):
        p = f"layers.{l}."
        s += [(p + "ln1.g", (d,), "g"), (p + "ln1.b", (d,), "beta"),
              (p + "q.w", (d, d), "w"), (p + "q.b", (d,), "b"),
              (p + "k.w", (d, d), "w"), (p + "k.b", (d,), "b"),
              (p + "v.w", (d, d), "w"), (p + "v.b", (d,), "b"),
              (p + "o.w", (d, d), "w"), (p + "o.b", (d,), "b"),
              (p + "ln2.g", (d,), "g"), (p + "ln2.b", (d,), "beta"),
              (p + "fc1.w", (g.d_ffn, d), "w"), (p + "fc1.b", (g.d_ffn,), "b"),
              (p + "fc2.w", (d, g.d_ffn), "w"), (p + "fc2.b", (d,), "b")]
    s += [("ln_post.g", (d,), "g"), ("ln_post.b", (d,), "beta")]
    if g.proj1_out:
        s += [("proj1.w", (g.proj1_out, d), "w"), ("proj1.b", (g.proj1_out,), "b"),
              ("proj2.w", (g.proj2_out, g.proj1_out), "w"), ("proj2.b", (g.proj2_out,), "b")]
    if g.adapter_hidden:
        a_in = g.proj2_out if g.proj2_out else d
        s += [("adapter.gate.w", (g.adapter_hidden, a_in), "w"),
              ("adapter.up.w", (g.adapter_hidden, a_in), "w"),
              ("adapter.down.w", (g.adapter_out, g.adapter_hidden), "w")]
    return s


def make_weights(g: Geometry, seed: int, affine: bool = False, std: float = 0.02):
    """Seeded random-init weights, an ordered dict name -> torch tensor (CPU).

    Matrices and conv kernels ~ N(0, std) drawn in ``weight_specs`` order from
    ``torch.Generator().manual_seed(seed)``.  By default biases are 0 and
    LayerNorms are identity (gain 1, shift 0).  With ``affine`` the biases are
    N(0, 0.02), LayerNorm gains 1 + N(0, 0.1) and shifts N(0, 0.02), drawn in
    the same stream, so that every bias and LayerNorm path carries signal.
    Values are rounded once to the geometry's dtype (bf16, f16 or fp32); both
    the oracle and the CUDA path consume exactly these rounded values.
    """
    gen = torch.Generator().manual_seed(seed)
    dt = {DTYPE_BF16: torch.bfloat16, DTYPE_F16: torch.float16}.get(g.dtype, torch.float32)
    out = {}
    for name, shape, kind in weight_specs(g):
        if kind == "w":
            t = torch.randn(shape, generator=gen, dtype=torch.float32) * std
        elif kind == "b":
            t = (torch.randn(shape, generator=gen) * 0.02) if affine else torch.zeros(shape)
        elif kind == "g":
            t = (1.0 + torch.randn(shape, generator=gen) * 0.1) if affine else torch.ones(shape)
        else:
            t = (torch.randn(shape, generator=gen) * 0.02) if affine else torch.zeros(shape)
        out[name] = t.to(dt).contiguous()
    return out
